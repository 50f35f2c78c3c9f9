// Kernel tracing: optional CUDA-event brackets around every kernel the
// library launches, so a caller can read per-kernel device time measured on
// the launching stream.  Off by default; while off, the launch path pays one
// branch.  Events are created by ssd_trace_enable (never on a compute call).
#include <cuda_runtime.h>
#include <mutex>
#include <string.h>

#include "../../include/ssd.h"
#include "ssd_trace.h"

namespace ssd {
namespace {

constexpr int kMaxRecords = 8192;

struct Record {
    int kernel;
    cudaEvent_t beg, end;
};

struct Tracer {
    std::mutex mu;
    bool on = false;
    int capacity = 0;
    int used = 0;
    int dropped = 0;
    Record rec[kMaxRecords];
} g_tr;

const char *kNames[kKernelCount] = {
    "simt_chunk_state", "simt_state_pass", "simt_chunk_out", "decode_step",
    "tc_unit_state", "tc_state_pass", "tc_chunk_out", "tc_dt_prep", "conv1d_silu", "gated_rmsnorm",
    "bwd_dstate", "bwd_dpass", "bwd_cols", "bwd_rows", "bwd_finalize", "bwd_reduce", "bwd_states",
};

}  // namespace

bool trace_on() { return g_tr.on; }

int trace_begin(cudaStream_t s, int kernel) {
    if (!g_tr.on) return -1;
    std::lock_guard<std::mutex> lk(g_tr.mu);
    if (g_tr.used >= g_tr.capacity) {
        ++g_tr.dropped;
        return -1;
    }
    const int i = g_tr.used++;
    g_tr.rec[i].kernel = kernel;
    cudaEventRecord(g_tr.rec[i].beg, s);
    return i;
}

void trace_end(cudaStream_t s, int slot) {
    if (slot < 0) return;
    cudaEventRecord(g_tr.rec[slot].end, s);
}

}  // namespace ssd

using ssd::g_tr;

extern "C" {

SSD_API ssd_status ssd_trace_enable(int max_launches) {
    std::lock_guard<std::mutex> lk(g_tr.mu);
    if (max_launches <= 0) {
        g_tr.on = false;
        return SSD_OK;
    }
    if (max_launches > ssd::kMaxRecords) max_launches = ssd::kMaxRecords;
    for (int i = g_tr.capacity; i < max_launches; ++i) {
        cudaError_t e = cudaEventCreate(&g_tr.rec[i].beg);
        if (e == cudaSuccess) e = cudaEventCreate(&g_tr.rec[i].end);
        if (e != cudaSuccess) {
            g_tr.capacity = i;
            return SSD_ERR_CUDA;
        }
    }
    if (max_launches > g_tr.capacity) g_tr.capacity = max_launches;
    g_tr.used = 0;
    g_tr.dropped = 0;
    g_tr.on = true;
    return SSD_OK;
}

SSD_API ssd_status ssd_trace_read(int kernel, int *launches, double *total_ms) {
    if (!launches || !total_ms || kernel < 0 || kernel >= ssd::kKernelCount) return SSD_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_tr.mu);
    int n = 0;
    double tot = 0.0;
    for (int i = 0; i < g_tr.used; ++i) {
        if (g_tr.rec[i].kernel != kernel) continue;
        cudaError_t e = cudaEventSynchronize(g_tr.rec[i].end);
        float ms = 0.f;
        if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, g_tr.rec[i].beg, g_tr.rec[i].end);
        if (e != cudaSuccess) return SSD_ERR_CUDA;
        tot += ms;
        ++n;
    }
    *launches = n;
    *total_ms = tot;
    return SSD_OK;
}

SSD_API const char *ssd_trace_kernel_name(int kernel) {
    if (kernel < 0 || kernel >= ssd::kKernelCount) return "";
    return ssd::kNames[kernel];
}

SSD_API int ssd_trace_kernel_count(void) { return ssd::kKernelCount; }

}  // extern "C"
