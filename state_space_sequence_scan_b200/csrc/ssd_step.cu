// Decode step: one token per (batch, head), state updated in place.
//
// nnterp guide "Mamba-2", section "The state between steps": the update
// writes the new state into the cache and returns only y; no sequence axis.
// Per (b, h):  dt = clamp(softplus(dt_raw + dt_bias)),  S = exp(dt A) S + dt B x^T,
//              y = S^T C + D x.
//
// HBM-bound: every state byte is read once and written once.  One CTA owns
// one (b, h) state of N x P fp32; thread t owns the float4 column quad
// q = t % (P/4) of rows n = t / (P/4) + k * (256 / (P/4)).  All of a
// thread's row loads are issued before any arithmetic (up to 8 x 16 B in
// flight per thread), loads and stores are 128-bit and coalesced along P,
// and the y reduction over n runs in shared memory in a fixed order (bitwise
// reproducible).  CTAs own disjoint states, so the in-place update is
// race-free.
#include "ssd_common.cuh"
#include "ssd_internal.h"
#include "ssd_trace.h"

namespace ssd {
namespace {

constexpr int kStepThreads = 256;
constexpr int kRowBatch = 8;

template <typename T, int P4>
__global__ void __launch_bounds__(kStepThreads)
step_kernel(const T *__restrict__ x, const float *__restrict__ dt_raw,
            const float *__restrict__ dt_bias, const float *__restrict__ A,
            const T *__restrict__ Bm, const T *__restrict__ Cm, const float *__restrict__ D,
            float *__restrict__ state, float *__restrict__ y, int H, int N, int G,
            float lo, float hi) {
    constexpr int P = 4 * P4;
    constexpr int RG = kStepThreads / P4;          // row groups
    extern __shared__ float4 sm4[];
    float *red = reinterpret_cast<float *>(sm4);   // RG * P, float4-accessed: first, 16-byte aligned
    float *sx = red + RG * P;                      // P
    float *sB = sx + P;                            // N
    float *sC = sB + N;                            // N

    const int bh = blockIdx.x;
    const int b = bh / H, h = bh - b * H;
    const int g = h / (H / G);
    const int tid = threadIdx.x;
    const int q = tid % P4, rg = tid / P4;

    for (int i = tid; i < N; i += kStepThreads) {
        sB[i] = to_f(Bm[((size_t)b * G + g) * N + i]);
        sC[i] = to_f(Cm[((size_t)b * G + g) * N + i]);
    }
    for (int i = tid; i < P; i += kStepThreads) sx[i] = to_f(x[(size_t)bh * P + i]);
    const float dt = dt_of(dt_raw[bh], dt_bias[h], lo, hi);
    const float a = expf(dt * A[h]);
    __syncthreads();

    const float4 xq = make_float4(sx[4 * q], sx[4 * q + 1], sx[4 * q + 2], sx[4 * q + 3]);
    float4 *S = reinterpret_cast<float4 *>(state + (size_t)bh * N * P);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);

    for (int n0 = rg; n0 < N; n0 += RG * kRowBatch) {
        float4 v[kRowBatch];
#pragma unroll
        for (int k = 0; k < kRowBatch; ++k) {
            const int n = n0 + k * RG;
            if (n < N) v[k] = __ldcs(&S[(size_t)n * P4 + q]);
        }
#pragma unroll
        for (int k = 0; k < kRowBatch; ++k) {
            const int n = n0 + k * RG;
            if (n < N) {
                const float w = dt * sB[n];
                float4 s = v[k];
                s.x = fmaf(a, s.x, w * xq.x);
                s.y = fmaf(a, s.y, w * xq.y);
                s.z = fmaf(a, s.z, w * xq.z);
                s.w = fmaf(a, s.w, w * xq.w);
                __stcs(&S[(size_t)n * P4 + q], s);
                const float c = sC[n];
                acc.x = fmaf(c, s.x, acc.x);
                acc.y = fmaf(c, s.y, acc.y);
                acc.z = fmaf(c, s.z, acc.z);
                acc.w = fmaf(c, s.w, acc.w);
            }
        }
    }
    reinterpret_cast<float4 *>(red + rg * P)[q] = acc;
    __syncthreads();
    const float Dh = D[h];
    for (int p = tid; p < P; p += kStepThreads) {
        float s = 0.f;
        for (int r = 0; r < RG; ++r) s += red[r * P + p];
        y[(size_t)bh * P + p] = fmaf(Dh, sx[p], s);
    }
}

template <typename T, int P4>
cudaError_t launch_p4(const StepArgs &a, cudaStream_t s) {
    const int P = 4 * P4;
    const int RG = kStepThreads / P4;
    const size_t smem = sizeof(float) * (2 * (size_t)a.N + P + (size_t)RG * P);
    auto kern = step_kernel<T, P4>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const long long blocks = (long long)a.b * a.H;
    {
        TraceScope tr(s, kTrDecodeStep);
        kern<<<(unsigned)blocks, kStepThreads, smem, s>>>(
            (const T *)a.x, a.dt_raw, a.dt_bias, a.A, (const T *)a.B, (const T *)a.C, a.D, a.state, a.y,
            (int)a.H, (int)a.N, (int)a.G, a.dt_lo, a.dt_hi);
    }
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const StepArgs &a, cudaStream_t s) {
    switch (a.P / 4) {
        case 1: return launch_p4<T, 1>(a, s);
        case 2: return launch_p4<T, 2>(a, s);
        case 4: return launch_p4<T, 4>(a, s);
        case 8: return launch_p4<T, 8>(a, s);
        case 16: return launch_p4<T, 16>(a, s);
        case 32: return launch_p4<T, 32>(a, s);
        case 64: return launch_p4<T, 64>(a, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool step_supported(int64_t P, int64_t N) {
    if (P % 4 != 0 || P < 4 || P > 256) return false;
    const int64_t p4 = P / 4;
    if ((p4 & (p4 - 1)) != 0) return false;       // P/4 must divide 256
    return N >= 1 && N <= 4096;
}

cudaError_t step_launch(const StepArgs &a, cudaStream_t s) {
    if (a.b * a.H == 0) return cudaSuccess;
    return a.bf16 ? launch_t<__nv_bfloat16>(a, s) : launch_t<float>(a, s);
}

}  // namespace ssd
