// TMA tensor-map encoding (host).
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace ssd {

enum TmapElem { kTmapBF16 = 0, kTmapF16 = 1, kTmapF32 = 2 };

// 4-D tiled map with 128-byte swizzle, zero fill out of range.  dims[0] is the
// innermost (contiguous) extent; strides_bytes[i] is the byte stride of
// dims[i+1].  Returns false when the driver entry point is unavailable or
// the encoding is rejected.
bool tmap_encode_4d(CUtensorMap *map, const void *base, TmapElem elem, const uint64_t dims[4],
                    const uint64_t strides_bytes[3], const uint32_t box[4]);

// 3-D tiled map without swizzle (the box lands in shared memory row after
// row, box[0] elements per row), zero fill out of range.  Same conventions.
bool tmap_encode_3d_plain(CUtensorMap *map, const void *base, TmapElem elem, const uint64_t dims[3],
                          const uint64_t strides_bytes[2], const uint32_t box[3]);

}  // namespace ssd
