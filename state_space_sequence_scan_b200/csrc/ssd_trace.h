// Internal tracing hooks (see ssd_trace.cu and ssd_trace_enable in ssd.h).
#pragma once

#include <cuda_runtime.h>

namespace ssd {

enum TraceKernel {
    kTrSimtChunkState = 0,
    kTrSimtStatePass = 1,
    kTrSimtChunkOut = 2,
    kTrDecodeStep = 3,
    kTrTcUnitState = 4,
    kTrTcStatePass = 5,
    kTrTcChunkOut = 6,
    kTrTcDtPrep = 7,
    kTrConv1d = 8,
    kTrGatedNorm = 9,
    kTrBwdDstate = 10,
    kTrBwdDpass = 11,
    kTrBwdCols = 12,
    kTrBwdRows = 13,
    kTrBwdFinalize = 14,
    kTrBwdReduce = 15,
    kTrBwdStates = 16,
    kKernelCount = 17,
};

bool trace_on();
int trace_begin(cudaStream_t s, int kernel);   // returns a slot, or -1 when tracing is off/full
void trace_end(cudaStream_t s, int slot);

// RAII bracket: `TraceScope t(stream, kTrX); launch...;`
struct TraceScope {
    cudaStream_t s;
    int slot;
    TraceScope(cudaStream_t st, int kernel) : s(st), slot(trace_begin(st, kernel)) {}
    ~TraceScope() { trace_end(s, slot); }
};

}  // namespace ssd
