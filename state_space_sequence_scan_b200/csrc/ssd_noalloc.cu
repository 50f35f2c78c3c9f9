// ssd_chunk_scan_fwd_noalloc: the chunked scan with its scratch in a fixed
// device array that lives inside this library, for callers that cannot
// allocate device memory themselves (for example code running where
// cudaMalloc is not allowed, or a host that hands out only its own input and
// output buffers).  The caller still passes inputs and outputs.
//
// The array below is a file-scope __device__ variable of kNoAllocScratchBytes.
// Every GPU that loads this library holds it until the process exits.  In
// host code its name is only a host-side stand-in, not a device address: the
// device address is looked up once per device with cudaGetSymbolAddress and
// that pointer is what the kernels receive.  The cached address belongs to the
// device's primary context (the runtime's); a cudaDeviceReset or a context
// made current through the driver API invalidates it.
#include <mutex>

#include "../../include/ssd.h"
#include "ssd_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)32 << 20;   // 32 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};

}  // namespace

extern "C" SSD_API ssd_status ssd_chunk_scan_fwd_noalloc(
    const void *x, const float *dt_raw, const float *dt_bias, const float *A, const void *B, const void *C,
    const float *D, const float *init_state, float *y, float *final_state, int64_t batch, int64_t seqlen,
    int64_t nheads, int64_t head_dim, int64_t state_dim, int64_t ngroups, int64_t chunk_size, float dt_lo,
    float dt_hi, int in_dtype, int path, void *stream) {
    size_t need = 0;
    ssd_status st = ssd_chunk_scan_workspace_size(batch, seqlen, nheads, head_dim, state_dim, ngroups, chunk_size,
                                                  in_dtype, path, &need);
    if (st != SSD_OK) return st;
    if (need > kNoAllocScratchBytes) return SSD_ERR_UNSUPPORTED;

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return (ssd_status)ssd::record_cuda_error(e);
    if (dev < 0 || dev >= kMaxDevices) return SSD_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_scratch_addr[dev]) {
            void *p = nullptr;
            e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
            if (e != cudaSuccess) return (ssd_status)ssd::record_cuda_error(e);
            g_scratch_addr[dev] = p;
        }
        scratch = g_scratch_addr[dev];
    }
    return ssd_chunk_scan_fwd(x, dt_raw, dt_bias, A, B, C, D, init_state, y, final_state, batch, seqlen, nheads,
                              head_dim, state_dim, ngroups, chunk_size, dt_lo, dt_hi, in_dtype, path, scratch,
                              kNoAllocScratchBytes, stream);
}
