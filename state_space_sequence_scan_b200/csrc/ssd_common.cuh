// Device helpers shared by the SSD kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssd {

// Device status word bits (first word of the scan workspace).
enum : unsigned {
    kStatusPrecondition = 1u,   // A > 0 seen
    kStatusTimeout = 2u,        // a bounded wait gave up
    kStatusRange = 4u,          // tensor path: a value outside the fp16 operand range
};

constexpr size_t kStatusBytes = 256;   // status region at the start of the workspace

__device__ __forceinline__ float softplus_f(float z) {
    // log(1 + e^z) in the stable form max(z,0) + log1p(e^-|z|)
    return fmaxf(z, 0.0f) + log1pf(expf(-fabsf(z)));
}

__device__ __forceinline__ float dt_of(float raw, float bias, float lo, float hi) {
    return fminf(fmaxf(softplus_f(raw + bias), lo), hi);
}

// silu(u) = u / (1 + e^-u) with the fast exponential and division.  The
// exponential's error grows with |u| (its argument u log2(e) is rounded to
// fp32 first): about 6e-6 relative at |u| = 100, 1e-6 for |u| < 16; inside
// the fp32 bar of 1e-5 and one bf16 rounding.  For u below about -87, e^-u
// passes 2^126 and the quotient is 0 (silu itself is below 1e-35 there).
// (A reciprocal by Newton steps on the FMA pipe instead of the special
// function unit was measured slower: the conv is issue-bound, not bound by
// that unit.)
__device__ __forceinline__ float silu_f(float u) { return __fdividef(u, 1.0f + __expf(-u)); }

// The causal depthwise conv of one channel at one token, then SiLU:
// silu(bias + sum_{k<K} w[k] x[k]), x[K-1] the current token's input and
// x[0] the oldest.  Two chains of fmas (even k, odd k), added at the end.
// Both arrangements of the conv (split and combined with the scan) evaluate
// exactly this, so they agree bit for bit.
template <int K>
__device__ __forceinline__ float conv_silu(const float (&w)[K], const float (&x)[K], float bias) {
    float a0 = bias, a1 = 0.f;
#pragma unroll
    for (int k = 0; k < K; ++k) {
        if (k & 1) a1 = fmaf(w[k], x[k], a1);
        else a0 = fmaf(w[k], x[k], a0);
    }
    return silu_f(a0 + a1);
}

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) {
    return __bfloat162float(v);
}

__device__ __forceinline__ void flag_status(unsigned *status, unsigned bit) {
    if (status) atomicOr(status, bit);
}

// Inclusive scan of one float per thread across a block of up to 1024 threads
// (blockDim.x a multiple of 32); `total` receives the block-wide sum.
// `warp_tot` is shared scratch of 32 floats.  Fixed combination order:
// deterministic run to run.
__device__ __forceinline__ float block_inclusive_scan(float v, float *warp_tot, float &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        float u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    if (warp == 0) {
        float t = lane < nw ? warp_tot[lane] : 0.0f;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            float u = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += u;
        }
        if (lane < nw) warp_tot[lane] = t;
    }
    __syncthreads();
    if (warp > 0) v += warp_tot[warp - 1];
    total = warp_tot[nw - 1];
    __syncthreads();
    return v;
}

}  // namespace ssd
