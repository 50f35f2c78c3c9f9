// The steps either side of the scan in a Mamba-2 layer (state-spaces/mamba
// issue on the training/inference paths: causal_conv1d_fn runs before the
// chunk scan; nnterp guide "Mamba-2", table "The values": y is taken before
// the gated norm and out_proj):
//   conv1d_silu_split  causal depthwise conv of width K over the x|B|C
//                      channels, bias, SiLU, written straight into the scan's
//                      separate x, B and C tensors (the split arrangement)
//   gated_rmsnorm      v = y * silu(z), RMS-normalised over groups of
//                      channels, times a per-channel weight
// Both are HBM-bound streams: coalesced vector loads and stores, one pass
// over the data (the norm holds a group in registers; groups that do not
// split evenly over its CTA take a two-pass warp kernel, the second read
// from L1/L2).
#include "../../include/ssd.h"
#include "ssd_common.cuh"
#include "ssd_internal.h"
#include "ssd_trace.h"

namespace ssd {
namespace {

constexpr int kConvThreads = 256;
constexpr int kConvCh = 4;      // channels per thread (one 8- or 16-byte access per token)
constexpr int kConvT = 16;      // tokens per thread (a sliding window in registers)
constexpr int kConvMaxK = 4;

// silu(u) = u / (1 + e^-u) with the fast exponential and division (relative
// error about 1e-6: inside the fp32 bar of 1e-5 and one bf16 rounding).  For
// u below about -87, e^-u is inf and the quotient is the limit, 0.
__device__ __forceinline__ float silu_f(float u) { return __fdividef(u, 1.0f + __expf(-u)); }

// 4 consecutive z values -> floats
__device__ __forceinline__ void load4(const __nv_bfloat16 *p, float (&v)[4]) {
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    v[0] = __uint_as_float(u.x << 16);
    v[1] = __uint_as_float(u.x & 0xFFFF0000u);
    v[2] = __uint_as_float(u.y << 16);
    v[3] = __uint_as_float(u.y & 0xFFFF0000u);
}
__device__ __forceinline__ void load4(const float *p, float (&v)[4]) {
    const float4 a = *reinterpret_cast<const float4 *>(p);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}

__device__ __forceinline__ void store4(__nv_bfloat16 *p, const float (&v)[4]) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), b = __floats2bfloat162_rn(v[2], v[3]);
    *reinterpret_cast<uint2 *>(p) = make_uint2(*reinterpret_cast<const uint32_t *>(&a),
                                               *reinterpret_cast<const uint32_t *>(&b));
}
__device__ __forceinline__ void store4(float *p, const float (&v)[4]) {
    *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
}

// One token tile [t0, t0 + kConvT) of 4 channels from c0 (see conv1d_silu_kernel).
template <typename T, int K>
__device__ __forceinline__ void conv1d_silu_tile(const T *__restrict__ xbc, const float *__restrict__ w,
                                                 const float *__restrict__ bias, T *__restrict__ x,
                                                 T *__restrict__ Bo, T *__restrict__ Co, int L, int Cd, int HP,
                                                 int GN, int c0, int t0, size_t b) {
    float wr[kConvCh][K], bs[kConvCh];
#pragma unroll
    for (int e = 0; e < kConvCh; ++e) {
        bs[e] = bias[c0 + e];
#pragma unroll
        for (int k = 0; k < K; ++k) wr[e][k] = w[(size_t)(c0 + e) * K + k];
    }
    // where these channels go: x [b,L,H*P], B or C [b,L,G*N] (H*P, G*N are multiples of 8)
    T *dst;
    int ld;
    if (c0 < HP) {
        dst = x + c0;
        ld = HP;
    } else if (c0 < HP + GN) {
        dst = Bo + (c0 - HP);
        ld = GN;
    } else {
        dst = Co + (c0 - HP - GN);
        ld = GN;
    }
    const T *src = xbc + b * L * (size_t)Cd + c0;
    dst += b * L * (size_t)ld;
    // rows t0-(K-1) .. t0+kConvT-1, all loaded before any arithmetic or store
    // (dst may not be proven apart from src, so a load after a store would
    // wait for it; 16 + K-1 independent loads keep enough bytes in flight)
    float win[K - 1 + kConvT][kConvCh];
    const int tn = min(kConvT, L - t0);
#pragma unroll
    for (int k = 0; k < K - 1 + kConvT; ++k) {
        const int t = t0 - (K - 1) + k;
        if (t >= 0 && k - (K - 1) < tn) load4(src + (size_t)t * Cd, win[k]);
        else {
#pragma unroll
            for (int e = 0; e < kConvCh; ++e) win[k][e] = 0.f;
        }
    }
#pragma unroll
    for (int j = 0; j < kConvT; ++j) {
        if (j < tn) {
            float o[kConvCh];
#pragma unroll
            for (int e = 0; e < kConvCh; ++e) {
                float acc = bs[e];
#pragma unroll
                for (int k = 0; k < K; ++k) acc = fmaf(wr[e][k], win[j + k][e], acc);
                o[e] = silu_f(acc);
            }
            store4(dst + (size_t)(t0 + j) * ld, o);
        }
    }
}

// grid (ceil(L/kConvT), ceil(Cd/4/256), b): thread = 4 channels x kConvT tokens.
// out[t, c] = silu(bias[c] + sum_k w[c, k] in[t - (K-1) + k, c]), in[t < 0] = 0.
template <typename T, int K>
__global__ void __launch_bounds__(kConvThreads)
conv1d_silu_kernel(const T *__restrict__ xbc, const float *__restrict__ w, const float *__restrict__ bias,
                   T *__restrict__ x, T *__restrict__ Bo, T *__restrict__ Co, int L, int Cd, int HP, int GN) {
    const int c0 = (blockIdx.y * kConvThreads + threadIdx.x) * kConvCh;
    if (c0 >= Cd) return;
    conv1d_silu_tile<T, K>(xbc, w, bias, x, Bo, Co, L, Cd, HP, GN, c0, blockIdx.x * kConvT, blockIdx.z);
}


// One CTA of kNormThreads per (token, group) when the group splits evenly
// into kNormThreads x V float4s: v = y silu(z) stays in registers, one read
// of y and z.  The sum of squares runs in a fixed order (each thread's V
// float4s, then a shuffle tree per warp, then the warps' partials by thread
// 0 in warp order): deterministic.
constexpr int kNormThreads = 128;
constexpr int kNormMaxV = 10;

template <typename Tz, int V>
__global__ void __launch_bounds__(kNormThreads)
gated_rmsnorm_block_kernel(const float *__restrict__ y, const Tz *__restrict__ z, const float *__restrict__ wt,
                           float *__restrict__ out, int D, int group, float eps) {
    __shared__ float s_part[kNormThreads / 32];
    __shared__ float s_r;
    const int ngr = D / group;
    const int64_t t = blockIdx.x / ngr;
    const int g0 = (int)(blockIdx.x % ngr) * group;
    const float *yr = y + t * D + g0;
    const Tz *zr = z + t * D + g0;
    float v[V][4];
    float yv[V][4], zv[V][4];
#pragma unroll
    for (int q = 0; q < V; ++q) {
        const int j = (q * kNormThreads + threadIdx.x) * 4;
        load4(yr + j, yv[q]);
        load4(zr + j, zv[q]);
    }
    float ss = 0.f;
#pragma unroll
    for (int q = 0; q < V; ++q)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            v[q][e] = yv[q][e] * silu_f(zv[q][e]);
            ss = fmaf(v[q][e], v[q][e], ss);
        }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) s_part[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x == 0) {
        float tot = 0.f;
#pragma unroll
        for (int w = 0; w < kNormThreads / 32; ++w) tot += s_part[w];
        s_r = 1.0f / sqrtf(tot / (float)group + eps);
    }
    __syncthreads();
    const float r = s_r;
    float *orow = out + t * D + g0;
    const float *wg = wt + g0;
#pragma unroll
    for (int q = 0; q < V; ++q) {
        const int j = (q * kNormThreads + threadIdx.x) * 4;
        const float4 wv = *reinterpret_cast<const float4 *>(wg + j);
        *reinterpret_cast<float4 *>(orow + j) =
            make_float4(v[q][0] * r * wv.x, v[q][1] * r * wv.y, v[q][2] * r * wv.z, v[q][3] * r * wv.w);
    }
}

// Fallback for groups that do not split evenly: one warp per (token, group);
// 8 warps per block.  Two passes over the group:
// the sum of squares (fixed shuffle order: deterministic), then the output.
template <typename Tz>
__global__ void __launch_bounds__(256)
gated_rmsnorm_kernel(const float *__restrict__ y, const Tz *__restrict__ z, const float *__restrict__ wt,
                     float *__restrict__ out, int64_t rows, int D, int group, float eps) {
    const int64_t gw = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int ngr = D / group;
    if (gw >= rows * ngr) return;
    const int lane = threadIdx.x & 31;
    const int64_t t = gw / ngr;
    const int g0 = (int)(gw % ngr) * group;
    const float *yr = y + t * D + g0;
    const Tz *zr = z + t * D + g0;
    float ss = 0.f;
    for (int j = lane * 4; j < group; j += 128) {
        const float4 yv = *reinterpret_cast<const float4 *>(yr + j);
        float zv[4];
        load4(zr + j, zv);
        const float v0 = yv.x * silu_f(zv[0]), v1 = yv.y * silu_f(zv[1]);
        const float v2 = yv.z * silu_f(zv[2]), v3 = yv.w * silu_f(zv[3]);
        ss = fmaf(v0, v0, fmaf(v1, v1, fmaf(v2, v2, fmaf(v3, v3, ss))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float r = 1.0f / sqrtf(ss / (float)group + eps);
    float *orow = out + t * D + g0;
    const float *wg = wt + g0;
    for (int j = lane * 4; j < group; j += 128) {
        const float4 yv = *reinterpret_cast<const float4 *>(yr + j);
        const float4 wv = *reinterpret_cast<const float4 *>(wg + j);
        float zv[4];
        load4(zr + j, zv);
        *reinterpret_cast<float4 *>(orow + j) =
            make_float4(yv.x * silu_f(zv[0]) * r * wv.x, yv.y * silu_f(zv[1]) * r * wv.y,
                        yv.z * silu_f(zv[2]) * r * wv.z, yv.w * silu_f(zv[3]) * r * wv.w);
    }
}

template <typename T>
cudaError_t conv_launch(const void *xbc, const float *w, const float *bias, void *x, void *B, void *C, int64_t b,
                        int64_t L, int Cd, int HP, int GN, int K, cudaStream_t s) {
    const dim3 g((unsigned)((L + kConvT - 1) / kConvT), (unsigned)((Cd / kConvCh + kConvThreads - 1) / kConvThreads),
                 (unsigned)b);
    TraceScope tr(s, kTrConv1d);
#define SSD_CONV(KK)                                                                                           \
    conv1d_silu_kernel<T, KK><<<g, kConvThreads, 0, s>>>((const T *)xbc, w, bias, (T *)x, (T *)B, (T *)C,     \
                                                         (int)L, Cd, HP, GN)
    switch (K) {
        case 1: SSD_CONV(1); break;
        case 2: SSD_CONV(2); break;
        case 3: SSD_CONV(3); break;
        default: SSD_CONV(4); break;
    }
#undef SSD_CONV
    return cudaGetLastError();
}

bool a16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace ssd

extern "C" SSD_API ssd_status ssd_conv1d_silu_split(const void *xbc, const float *weight, const float *bias,
                                                    void *x, void *B, void *C, int64_t batch, int64_t seqlen,
                                                    int64_t nheads, int64_t head_dim, int64_t ngroups,
                                                    int64_t state_dim, int64_t kernel_width, int in_dtype,
                                                    void *stream) {
    if (batch < 0 || seqlen < 0 || nheads <= 0 || head_dim <= 0 || ngroups <= 0 || state_dim <= 0)
        return SSD_ERR_INVALID_ARG;
    if (kernel_width < 1 || kernel_width > ssd::kConvMaxK) return SSD_ERR_UNSUPPORTED;
    if (in_dtype != SSD_F32 && in_dtype != SSD_BF16) return SSD_ERR_UNSUPPORTED;
    const int64_t HP = nheads * head_dim, GN = ngroups * state_dim, Cd = HP + 2 * GN;
    // grid: token tiles in x, 256-thread channel blocks in y (<= 65535), batch in z
    if (HP % 8 || GN % 8 || Cd > (1 << 24) || batch > 65535 || seqlen > (1ll << 31) - ssd::kConvT)
        return SSD_ERR_UNSUPPORTED;
    if (batch == 0 || seqlen == 0) return SSD_OK;
    if (!xbc || !weight || !bias || !x || !B || !C) return SSD_ERR_INVALID_ARG;
    if (!ssd::a16(xbc) || !ssd::a16(x) || !ssd::a16(B) || !ssd::a16(C)) return SSD_ERR_ALIGNMENT;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const cudaError_t e =
        in_dtype == SSD_BF16
            ? ssd::conv_launch<__nv_bfloat16>(xbc, weight, bias, x, B, C, batch, seqlen, (int)Cd, (int)HP, (int)GN,
                                              (int)kernel_width, s)
            : ssd::conv_launch<float>(xbc, weight, bias, x, B, C, batch, seqlen, (int)Cd, (int)HP, (int)GN,
                                      (int)kernel_width, s);
    return e == cudaSuccess ? SSD_OK : (ssd_status)ssd::record_cuda_error(e);
}

extern "C" SSD_API ssd_status ssd_gated_rmsnorm(const float *y, const void *z, const float *weight, float *out,
                                                int64_t tokens, int64_t dim, int64_t group_size, float eps,
                                                int z_dtype, void *stream) {
    if (tokens < 0 || dim <= 0 || group_size <= 0 || dim % group_size != 0 || !(eps >= 0.0f))
        return SSD_ERR_INVALID_ARG;
    if (z_dtype != SSD_F32 && z_dtype != SSD_BF16) return SSD_ERR_UNSUPPORTED;
    // one warp per (token, group), 8 per block: at most 2^31 blocks
    if (group_size % 4 || dim > (1 << 30) || tokens > (1ll << 40) || tokens * (dim / group_size) > (1ll << 34))
        return SSD_ERR_UNSUPPORTED;
    if (tokens == 0) return SSD_OK;
    if (!y || !z || !weight || !out) return SSD_ERR_INVALID_ARG;
    if (!ssd::a16(y) || !ssd::a16(weight) || !ssd::a16(out) || (reinterpret_cast<uintptr_t>(z) & 7u))
        return SSD_ERR_ALIGNMENT;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t warps = tokens * (dim / group_size);
    const unsigned blocks = (unsigned)((warps + 7) / 8);
    // the single-pass block kernel when a group is kNormThreads x V float4s
    const int64_t V = group_size / (4 * ssd::kNormThreads);
    if (group_size % (4 * ssd::kNormThreads) == 0 && V >= 1 && V <= ssd::kNormMaxV && warps <= 0x7fffffffll) {
        ssd::TraceScope tr(s, ssd::kTrGatedNorm);
        const unsigned nb = (unsigned)warps;
        const __nv_bfloat16 *zb = static_cast<const __nv_bfloat16 *>(z);
        const float *zf = static_cast<const float *>(z);
#define SSD_NORM(VV)                                                                                              \
    if (z_dtype == SSD_BF16)                                                                                      \
        ssd::gated_rmsnorm_block_kernel<__nv_bfloat16, VV><<<nb, ssd::kNormThreads, 0, s>>>(y, zb, weight, out,  \
                                                                                            (int)dim,            \
                                                                                            (int)group_size, eps); \
    else                                                                                                          \
        ssd::gated_rmsnorm_block_kernel<float, VV><<<nb, ssd::kNormThreads, 0, s>>>(y, zf, weight, out, (int)dim, \
                                                                                    (int)group_size, eps)
        switch (V) {
            case 1: SSD_NORM(1); break;
            case 2: SSD_NORM(2); break;
            case 3: SSD_NORM(3); break;
            case 4: SSD_NORM(4); break;
            case 5: SSD_NORM(5); break;
            case 6: SSD_NORM(6); break;
            case 7: SSD_NORM(7); break;
            case 8: SSD_NORM(8); break;
            case 9: SSD_NORM(9); break;
            default: SSD_NORM(10); break;
        }
#undef SSD_NORM
    } else {
        ssd::TraceScope tr(s, ssd::kTrGatedNorm);
        if (z_dtype == SSD_BF16)
            ssd::gated_rmsnorm_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(
                y, static_cast<const __nv_bfloat16 *>(z), weight, out, tokens, (int)dim, (int)group_size, eps);
        else
            ssd::gated_rmsnorm_kernel<float><<<blocks, 256, 0, s>>>(y, static_cast<const float *>(z), weight, out,
                                                                    tokens, (int)dim, (int)group_size, eps);
    }
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SSD_OK : (ssd_status)ssd::record_cuda_error(e);
}
