// The steps either side of the scan in a Mamba-2 layer (state-spaces/mamba
// issue on the training/inference paths: causal_conv1d_fn runs before the
// chunk scan; nnterp guide "Mamba-2", table "The values": y is taken before
// the gated norm and out_proj):
//   conv1d_silu_split  causal depthwise conv of width K over the x|B|C
//                      channels, bias, SiLU, written straight into the scan's
//                      separate x, B and C tensors (the split arrangement)
//   gated_rmsnorm      v = y * silu(z), RMS-normalised over groups of
//                      channels, times a per-channel weight
// Both are HBM-bound streams with one pass over the data.  The conv stages
// its input tiles in shared memory by TMA, several tiles in flight per CTA,
// and stores from registers; its SiLU costs two special-function operations
// an element, so it also needs enough warps to keep that unit busy.  The
// norm holds a group in registers (groups that do not split evenly over its
// CTA take a two-pass warp kernel, the second read from L1/L2).
#include <cuda.h>

#include "../../include/ssd.h"
#include "ssd_common.cuh"
#include "ssd_internal.h"
#include "ssd_tc.cuh"
#include "ssd_tmap.h"
#include "ssd_trace.h"

namespace ssd {
namespace {

constexpr int kConvCh = 4;                    // channels per lane (one 8- or 16-byte access per token)
constexpr int kConvMaxK = 4;
constexpr int kCvWarps = 16;
constexpr int kCvThreads = 32 * kCvWarps;
constexpr int kCvTC = 32 * kConvCh;           // channels per tile: one warp across
constexpr int kCvTokPerWarp = 8;
constexpr int kCvTT = kCvWarps * kCvTokPerWarp;  // tokens per tile
constexpr int kCvHalo = kConvMaxK - 1;        // rows before the tile's first token
constexpr int kCvRows = kCvHalo + kCvTT;      // rows per tile in shared memory
constexpr long long kCvWaitBudget = 1ll << 32;  // clock cycles before a wait gives up (~2 s)
// tiles in flight per CTA: 3 x 33.5 KB (bf16: two 16-warp CTAs per SM, as
// the register file allows at 64 registers a thread), 3 x 67 KB (fp32: one
// CTA per SM by shared memory)
template <typename T> struct CvStages { static constexpr int value = 3; };
template <typename T> constexpr size_t cv_smem_bytes() {
    return (size_t)CvStages<T>::value * kCvRows * kCvTC * sizeof(T) + 8 * CvStages<T>::value;
}

// Status word of the workspace-free kernels (conv1d): kStatusTimeout when a
// bounded wait gave up.  Read and cleared by ssd_read_device_status(NULL, ...).
__device__ unsigned g_front_status = 0;

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

// Persistent conv1d + SiLU over tiles of kCvTT tokens x kCvTC channels.
// Tile rows arrive in shared memory by TMA (a 3-D map over xbc [b, L, Cd],
// box kCvTC x (kCvHalo + kCvTT) x 1, zero fill out of range: the rows before
// token 0 and past L, and the channels past Cd, read as zeros), CvStages
// tiles in flight per CTA.  Shared row r of a tile holds token
// t0 - kCvHalo + r.  Warp w computes tokens [8w, 8w + 8) of the tile,
// lane l channels [4l, 4l + 4), sliding a K-row window down shared memory,
// and stores its outputs straight to x, B or C (8 or 16 bytes per lane, 256
// or 512 bytes per warp and row).  CTA i keeps channel tile i % n_ct for its
// whole life (its weights stay in registers) and walks the (batch, token
// tile) rows i / n_ct, i / n_ct + rows_step, ...
// out[t, c] = silu(bias[c] + sum_k w[c, k] in[t - (K-1) + k, c]), in[t < 0] = 0.
template <typename T, int K>
__global__ void __launch_bounds__(kCvThreads, 2)   // two CTAs per SM: at most 64 registers
conv1d_silu_kernel(const __grid_constant__ CUtensorMap tm, const float *__restrict__ w,
                   const float *__restrict__ bias, T *__restrict__ x, T *__restrict__ Bo, T *__restrict__ Co, int L,
                   int Cd, int HP, int GN, int n_ct, int n_tt, long long n_rows, int rows_step,
                   unsigned *__restrict__ status, long long wait_budget) {
    constexpr int S = CvStages<T>::value;
    constexpr uint32_t kStageBytes = (uint32_t)(kCvRows * kCvTC * sizeof(T));
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + S * kStageBytes);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ct = blockIdx.x % n_ct;
    const long long row0 = blockIdx.x / n_ct;
    if (tid == 0) {
        tc::tma_prefetch_desc(&tm);
        for (int i = 0; i < S; ++i) tc::mbar_init(&full[i], 1);
        tc::fence_mbar_init();
    }
    __syncthreads();
    // request the tile of (batch, token tile) row `row` into stage `st`
    auto request = [&](long long row, int st) {
        const int tt = (int)(row % n_tt), bb = (int)(row / n_tt);
        tc::mbar_arrive_expect_tx(&full[st], kStageBytes);
        tc::tma_load_3d(smem + st * kStageBytes, &tm, &full[st], ct * kCvTC, tt * kCvTT - kCvHalo, bb);
    };
    if (tid == 0)
        for (int i = 0; i < S; ++i)
            if (row0 + (long long)i * rows_step < n_rows) request(row0 + (long long)i * rows_step, i);

    // this lane's 4 channels, their weights and destination
    const int c0 = ct * kCvTC + lane * kConvCh;
    const bool live = c0 < Cd;
    float wr[kConvCh][K], bs[kConvCh];
#pragma unroll
    for (int e = 0; e < kConvCh; ++e) {
        bs[e] = live ? bias[c0 + e] : 0.f;
#pragma unroll
        for (int k = 0; k < K; ++k) wr[e][k] = live ? w[(size_t)(c0 + e) * K + k] : 0.f;
    }
    T *dst = x;
    int ld = HP;
    if (c0 < HP) {
        dst = x + c0;
    } else if (c0 < HP + GN) {
        dst = Bo + (c0 - HP);
        ld = GN;
    } else {
        dst = Co + (c0 - HP - GN);
        ld = GN;
    }

    int it = 0;
    bool timed_out = false;
    for (long long row = row0; row < n_rows; row += rows_step, ++it) {
        const int st = it % S;
        const bool ok = tc::mbar_wait(&full[st], (uint32_t)(it / S) & 1u, wait_budget);
        // one decision for the whole CTA; the barrier also says that every
        // warp is done with the previous tile, whose stage is refilled now
        if (!__syncthreads_and(ok)) {
            timed_out = true;
            break;
        }
        if (tid == 0 && it > 0) {
            const long long nxt = row + (long long)(S - 1) * rows_step;
            if (nxt < n_rows) request(nxt, (it - 1) % S);
        }
        const int tt = (int)(row % n_tt);
        const size_t bb = (size_t)(row / n_tt);
        const int tbase = tt * kCvTT + warp * kCvTokPerWarp;     // first output token of this warp
        const T *src = reinterpret_cast<const T *>(smem + st * kStageBytes) + lane * kConvCh;
        // window of the K input rows of the current output token
        float win[K][kConvCh];
#pragma unroll
        for (int k = 0; k < K - 1; ++k)
            load4(src + (warp * kCvTokPerWarp + kCvHalo - (K - 1) + k) * kCvTC, win[k]);
        T *out = dst + bb * (size_t)L * ld;
#pragma unroll
        for (int j = 0; j < kCvTokPerWarp; ++j) {
            load4(src + (warp * kCvTokPerWarp + kCvHalo + j) * kCvTC, win[K - 1]);
            float o[kConvCh];
#pragma unroll
            for (int e = 0; e < kConvCh; ++e) {
                float xw[K];
#pragma unroll
                for (int k = 0; k < K; ++k) xw[k] = win[k][e];
                o[e] = conv_silu<K>(wr[e], xw, bs[e]);
            }
            if (live && tbase + j < L) store4(out + (size_t)(tbase + j) * ld, o);
#pragma unroll
            for (int k = 0; k < K - 1; ++k)
#pragma unroll
                for (int e = 0; e < kConvCh; ++e) win[k][e] = win[k + 1][e];
        }
    }
    if (timed_out && tid == 0) {
        atomicOr(status, kStatusTimeout);
        // let this CTA's copies still in flight land before its shared memory
        // goes away (each wait bounded again): iterations it .. last were
        // requested and not consumed (the first S at the start, then one
        // S - 1 ahead of each consumed iteration after the first)
        const int last = it == 0 ? S - 1 : it + S - 2;
        for (int j = it; j <= last; ++j)
            if (row0 + (long long)j * rows_step < n_rows)
                tc::mbar_wait(&full[j % S], (uint32_t)(j / S) & 1u, wait_budget);
    }
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

constexpr int kCvMaxDevices = 64;

// SM count and resident conv CTAs per SM on the current device, and the
// shared-memory limit set for the kernel, once per (device, type, width)
template <typename T, int K>
cudaError_t conv_slots(int *slots) {
    static int cached[kCvMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kCvMaxDevices) return cudaErrorInvalidDevice;
    if (!cached[dev]) {
        const int smem = (int)cv_smem_bytes<T>();
        if ((e = cudaFuncSetAttribute(conv1d_silu_kernel<T, K>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
            cudaSuccess)
            return e;
        int sms = 0, per_sm = 0;
        if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, conv1d_silu_kernel<T, K>, kCvThreads,
                                                               smem)) != cudaSuccess)
            return e;
        cached[dev] = sms * (per_sm > 0 ? per_sm : 1);
    }
    *slots = cached[dev];
    return cudaSuccess;
}

cudaError_t front_status_ptr(unsigned **p) {
    static unsigned *cached[kCvMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kCvMaxDevices) return cudaErrorInvalidDevice;
    if (!cached[dev]) {
        void *q = nullptr;
        if ((e = cudaGetSymbolAddress(&q, g_front_status)) != cudaSuccess) return e;
        cached[dev] = static_cast<unsigned *>(q);
    }
    *p = cached[dev];
    return cudaSuccess;
}

template <typename T, int K>
cudaError_t conv_launch_k(const void *xbc, const float *w, const float *bias, void *x, void *B, void *C, int64_t b,
                          int64_t L, int Cd, int HP, int GN, cudaStream_t s) {
    CUtensorMap tm;
    const uint64_t dims[3] = {(uint64_t)Cd, (uint64_t)L, (uint64_t)b};
    const uint64_t strides[2] = {(uint64_t)Cd * sizeof(T), (uint64_t)L * Cd * sizeof(T)};
    const uint32_t box[3] = {(uint32_t)kCvTC, (uint32_t)kCvRows, 1u};
    if (!tmap_encode_3d_plain(&tm, xbc, sizeof(T) == 2 ? kTmapBF16 : kTmapF32, dims, strides, box))
        return cudaErrorInvalidValue;
    int slots = 0;
    unsigned *status = nullptr;
    cudaError_t e = conv_slots<T, K>(&slots);
    if (e == cudaSuccess) e = front_status_ptr(&status);
    if (e != cudaSuccess) return e;
    const int n_ct = (Cd + kCvTC - 1) / kCvTC;
    const int n_tt = (int)((L + kCvTT - 1) / kCvTT);
    const long long n_rows = b * (long long)n_tt;
    long long step = slots / n_ct;
    if (step < 1) step = 1;
    if (step > n_rows) step = n_rows;
    const unsigned grid = (unsigned)(n_ct * step);
    conv1d_silu_kernel<T, K><<<grid, kCvThreads, cv_smem_bytes<T>(), s>>>(
        tm, w, bias, (T *)x, (T *)B, (T *)C, (int)L, Cd, HP, GN, n_ct, n_tt, n_rows, (int)step, status, kCvWaitBudget);
    return cudaGetLastError();
}

template <typename T>
cudaError_t conv_launch(const void *xbc, const float *w, const float *bias, void *x, void *B, void *C, int64_t b,
                        int64_t L, int Cd, int HP, int GN, int K, cudaStream_t s) {
    TraceScope tr(s, kTrConv1d);
    switch (K) {
        case 1: return conv_launch_k<T, 1>(xbc, w, bias, x, B, C, b, L, Cd, HP, GN, s);
        case 2: return conv_launch_k<T, 2>(xbc, w, bias, x, B, C, b, L, Cd, HP, GN, s);
        case 3: return conv_launch_k<T, 3>(xbc, w, bias, x, B, C, b, L, Cd, HP, GN, s);
        default: return conv_launch_k<T, 4>(xbc, w, bias, x, B, C, b, L, Cd, HP, GN, s);
    }
}

bool a16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

// Reads and clears the workspace-free kernels' status word on the current
// device (synchronises the stream).
cudaError_t front_status_read(cudaStream_t s, unsigned *word) {
    unsigned *p = nullptr;
    cudaError_t e = front_status_ptr(&p);
    if (e != cudaSuccess) return e;
    if ((e = cudaMemcpyAsync(word, p, sizeof(unsigned), cudaMemcpyDeviceToHost, s)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(p, 0, sizeof(unsigned), s)) != cudaSuccess) return e;
    return cudaStreamSynchronize(s);
}

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
    // TMA coordinates are 32-bit and the map's strides below 2^40 bytes
    if (HP % 8 || GN % 8 || Cd > (1 << 24) || batch > (1 << 30) || seqlen > (1ll << 31) - 2 * ssd::kCvTT ||
        seqlen * Cd * 4 >= (1ll << 40))
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
