// Host-side construction of TMA tensor maps (cuTensorMapEncodeTiled, reached
// through the runtime's driver entry point so libssd.so needs no link to
// libcuda).  Encoding is pure host work: nothing is enqueued on the GPU.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <mutex>

#include "ssd_tmap.h"

namespace ssd {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_once;

void resolve() {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
}

CUtensorMapDataType tmap_dtype(TmapElem elem) {
    return elem == kTmapBF16  ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
           : elem == kTmapF16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                              : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
}

}  // namespace

bool tmap_encode_3d_plain(CUtensorMap *map, const void *base, TmapElem elem, const uint64_t dims[3],
                          const uint64_t strides_bytes[2], const uint32_t box[3]) {
    std::call_once(g_once, resolve);
    if (!g_encode) return false;
    cuuint64_t gd[3] = {dims[0], dims[1], dims[2]};
    cuuint64_t gs[2] = {strides_bytes[0], strides_bytes[1]};
    cuuint32_t bx[3] = {box[0], box[1], box[2]};
    cuuint32_t es[3] = {1, 1, 1};
    CUresult r = g_encode(map, tmap_dtype(elem), 3, const_cast<void *>(base), gd, gs, bx, es,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool tmap_encode_4d(CUtensorMap *map, const void *base, TmapElem elem, const uint64_t dims[4],
                    const uint64_t strides_bytes[3], const uint32_t box[4]) {
    std::call_once(g_once, resolve);
    if (!g_encode) return false;
    const CUtensorMapDataType dt = tmap_dtype(elem);
    cuuint64_t gd[4] = {dims[0], dims[1], dims[2], dims[3]};
    cuuint64_t gs[3] = {strides_bytes[0], strides_bytes[1], strides_bytes[2]};
    cuuint32_t bx[4] = {box[0], box[1], box[2], box[3]};
    cuuint32_t es[4] = {1, 1, 1, 1};
    CUresult r = g_encode(map, dt, 4, const_cast<void *>(base), gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace ssd
