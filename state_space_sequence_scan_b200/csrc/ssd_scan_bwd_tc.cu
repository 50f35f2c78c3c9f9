// Tensor-core pair kernels of the backward (sm_100a: tcgen05 MMAs with TMEM
// accumulators).  They take the place of the fp32 CUDA-core `cols` and
// `rows` kernels of ssd_scan_bwd.cu (same inputs, same outputs in the same
// workspace regions; the launches around them are unchanged), for bf16
// inputs with head_dim 64, state_dim 128 and a chunk size that is a multiple
// of 128, packed rows included (the fp32 kernels' document masks, applied to
// values).  The formulas are those of ssd_scan_bwd.cu's header (the chunked
// form of the forward, "Mamba2" knowledge page); every product of two
// 128-token blocks is an MMA:
//
// cols, per (j block J of a chunk, head, batch), TMEM lane = token j (16 warps:
// lane quarter w % 4, column quarter w / 4):
//   dX_J  = e^{cl-cum_j} B_J G_c             (M=128 j, N=64 p,  K=128 n)
//   dB_J  = e^{cl-cum_j} X_J G_c^T           (M=128 j, N=128 n, K=64 p)
//           (before the scaling, a row dot with B_J gives E_j)
//   for each i block I >= J of the chunk:
//     CB^T = B_J C_I^T,  S^T = X_J dY_I^T    (M=128 j, N=128 i)
//     U^T = CB^T L, V^T = S^T L  (L_ij = e^{cum_i-cum_j}, i >= j), as fp16
//     dX_J += U^T dY_I,  dB_J += V^T C_I     (K=128 i; dB as two N=64 halves)
//   dx_j = dt_j dX_j + D dy_j,  dB_j = dt_j dB_j, and per token the direct
//   d(dt) (row sums of U^T.S^T), the column part of d(cum), E_j, dy_j.x_j.
// rows, per (i block I, head, batch), TMEM lane = token i:
//   dC_I  = e^{cum_i} dY_I H_in^T            (M=128 i, N=128 n, K=64 p)
//           (before the scaling, a row dot with C_I gives T_i)
//   for each j block J <= I: CB = C_I B_J^T, S = dY_I X_J^T,
//     V = S L dt_j (j <= i) as fp16, dC_I += V B_J   (K=128 j; two N=64 halves)
//   and the row part of d(cum): T_i + sum_{j<i} CB_ij V_ij.
//
// Operands are fp16 in 128-byte-swizzled shared-memory tiles, written by the
// threads from the inputs (bf16 B, C, x widen to fp16 exactly inside its
// range; dy, G_c and H_in round to fp16's 11 bits); accumulation is fp32.
// The results carry the forward tensor path's precision: the bf16-input bar
// (2e-2 of RMS) applies, not the fp32 CUDA-core backward's.  A value outside
// fp16's range sets the workspace's range bit (SSD_ERR_PRECONDITION).  Each
// CTA runs its phases in order (copy in, MMA, TMEM math, MMA, ...); every
// wait on an MMA completion is bounded and a timeout sets the status word.
// Sums run in a fixed order (no atomics): deterministic.
#include "ssd_common.cuh"
#include "ssd_internal.h"
#include "ssd_tc.cuh"
#include "ssd_trace.h"

namespace ssd {
namespace {
using namespace tc;

constexpr int kB = 128;                    // tokens per block (MMA M)
constexpr int kNs = 128;                   // state_dim
constexpr int kPh = 64;                    // head_dim
constexpr uint32_t kT = 16384;             // one [128 rows x 64 fp16] swizzled tile
constexpr int kThr = 256;                  // tc_states: 8 warps, lane quarter w % 4, column half w / 4
constexpr int kThrP = 512;                 // pair kernels: 16 warps, lane quarter w % 4, column quarter w / 4
constexpr long long kBudget = 1ll << 32;   // clock cycles before an MMA wait gives up (~2 s)
constexpr float kF16Max = 65504.0f;

// K-step q (16 elements) of a K-major operand 128 wide (two 64-wide tiles)
__device__ __forceinline__ uint32_t kofs128(int q) { return (uint32_t)((q >> 2) * kT + (q & 3) * 32); }

// 8 source values (one 16-byte fp16 chunk's worth) -> floats
template <typename S> struct Raw8;
template <> struct Raw8<__nv_bfloat16> {
    uint4 v;
    __device__ __forceinline__ void load(const __nv_bfloat16 *p) { v = *reinterpret_cast<const uint4 *>(p); }
    __device__ __forceinline__ void zero() { v = make_uint4(0u, 0u, 0u, 0u); }
    __device__ __forceinline__ void get(float (&f)[8]) const {
        f[0] = bf16lo(v.x); f[1] = bf16hi(v.x); f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
        f[4] = bf16lo(v.z); f[5] = bf16hi(v.z); f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
    }
};
template <> struct Raw8<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const float *p) {
        a = *reinterpret_cast<const float4 *>(p);
        b = *reinterpret_cast<const float4 *>(p + 4);
    }
    __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
    __device__ __forceinline__ void get(float (&f)[8]) const {
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    }
};

// Rows 0..127 of a [128 x W] fp16 tile (W = 64 or 128: one or two swizzled
// 64-wide tiles) from `nrows` source rows of `ld` elements (bf16 or fp32),
// each row times scale[r] when `scale` is given; rows past nrows are zero.
// All NT threads; one 16-byte chunk (8 values) per step, consecutive
// threads on consecutive chunks of a row, every load issued before the
// first conversion.
template <int W, int NT, typename S>
__device__ __forceinline__ void fill_tile(uint8_t *tile, const S *src, size_t ld, int nrows, int tid, __half2 &amax,
                                          const float *scale = nullptr) {
    constexpr int cpr = W / 8;             // chunks per row
    constexpr int kIt = kB * cpr / NT;     // chunks per thread
    Raw8<S> raw[kIt];
#pragma unroll
    for (int it = 0; it < kIt; ++it) {
        const int c = tid + it * NT, r = c / cpr, k = c - r * cpr;
        if (r < nrows) raw[it].load(src + (size_t)r * ld + 8 * k);
        else raw[it].zero();
    }
#pragma unroll
    for (int it = 0; it < kIt; ++it) {
        const int c = tid + it * NT, r = c / cpr, k = c - r * cpr;
        float f[8];
        raw[it].get(f);
        if (scale) {
            const float w = scale[r];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] *= w;
        }
        const uint4 o = make_uint4(pack_h2(f[0], f[1]), pack_h2(f[2], f[3]), pack_h2(f[4], f[5]), pack_h2(f[6], f[7]));
        const uint32_t w4[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) amax = __hmax2(amax, __habs2(*reinterpret_cast<const __half2 *>(&w4[i])));
        *reinterpret_cast<uint4 *>(tile + (k >> 3) * kT + sw128_off(r, k & 7)) = o;
    }
}

// Dot of 32 fp32 accumulator values with row `r`, chunks c0..c0+3 of tile
// `half` (32 fp16 values) of a 128-wide swizzled tile
__device__ __forceinline__ float row_dot32(const uint8_t *tile, int r, int half, int c0, const float (&a)[32]) {
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint4 v = *reinterpret_cast<const uint4 *>(tile + half * kT + sw128_off(r, c0 + k));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = unpack_h2(w[e]);
            s = fmaf(f.x, a[8 * k + 2 * e], s);
            s = fmaf(f.y, a[8 * k + 2 * e + 1], s);
        }
    }
    return s;
}

// 32 fp32 values -> fp16 into row `r`, chunks c0..c0+3 of a swizzled tile
__device__ __forceinline__ void store_row32(uint8_t *tile, int r, int c0, const float (&v)[32], __half2 &amax) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            w[e] = pack_h2(v[8 * k + 2 * e], v[8 * k + 2 * e + 1]);
            amax = __hmax2(amax, __habs2(*reinterpret_cast<const __half2 *>(&w[e])));
        }
        *reinterpret_cast<uint4 *>(tile + sw128_off(r, c0 + k)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// Waits for the next completion of `bar` (phase `ph`, then advances it).
// Bounded: false after the budget.
__device__ __forceinline__ bool wait_mma(uint64_t *bar, uint32_t &ph) {
    const bool ok = mbar_wait(bar, ph & 1u, kBudget);
    ++ph;
    tc_fence_after();
    return ok;
}

__device__ __forceinline__ void finish_range(unsigned *status, __half2 amax) {
    const float2 m = __half22float2(amax);
    if (!(m.x <= kF16Max && m.y <= kF16Max)) flag_status(status, kStatusRange);
}

// ---- cols -----------------------------------------------------------------
// shared memory (offsets from a 1024-aligned base)
constexpr uint32_t kCBj = 0, kCXj = 2 * kT, kCG = 3 * kT, kCCi = 4 * kT, kCDYi = 6 * kT, kCU = 7 * kT,
                   kCV = 9 * kT, kCScal = 11 * kT;
// scalars: cum_j, dt_j, dec_j, cum_i, then per column quarter e1[4], zs[4], zo[4], dyx[4], then the
// document counters doc_j, doc_i of packed rows (128 floats each)
constexpr uint32_t kCBar = kCScal + 22 * kB * 4;
constexpr size_t kColsSmem = 1024 + kCBar + 16;
// TMEM columns (each accumulator starts on a multiple of its width, as in
// the forward kernels)
constexpr uint32_t kTmCBt = 0, kTmSt = 128, kTmDB = 256, kTmDX = 384;

template <bool kPacked>
__global__ void __launch_bounds__(kThrP, 1)
tc_cols_kernel(BwdPairArgs a, int L, int H, int G, int Q, int nc) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *s_cumj = reinterpret_cast<float *>(sm + kCScal);
    float *s_dtj = s_cumj + kB, *s_dec = s_dtj + kB, *s_cumi = s_dec + kB;
    float *s_e1 = s_cumi + kB, *s_zs = s_e1 + 4 * kB, *s_zo = s_zs + 4 * kB, *s_dyx = s_zo + 4 * kB;
    float *s_docj = s_dyx + 4 * kB, *s_doci = s_docj + kB;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + kCBar);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar + 1);

    const int nJ = Q / kB;
    const int c = blockIdx.x / nJ, Jb = blockIdx.x - c * nJ;
    const int h = blockIdx.y, b = blockIdx.z;
    const int g = h / (H / G);
    const int t0 = c * Q, q = min(Q, L - t0);
    const int j0 = Jb * kB;
    if (j0 >= q) return;                               // uniform over the CTA
    const int tj = min(kB, q - j0);
    const size_t bh = (size_t)b * H + h;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int lg = warp & 3, ch = warp >> 2, row = 32 * lg + lane;
    __half2 amax = __float2half2_rn(0.f);

    if (warp == 0) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    // j block: B_J, X_J (fp16), G_c (fp16 [n][p]); per-token scalars
    const size_t tokj = (size_t)b * L + t0 + j0;
    fill_tile<128, kThrP>(sm + kCBj, static_cast<const __nv_bfloat16 *>(a.B) + (tokj * G + g) * kNs,
                   (size_t)G * kNs, tj, tid, amax);
    fill_tile<64, kThrP>(sm + kCXj, static_cast<const __nv_bfloat16 *>(a.x) + (tokj * H + h) * kPh,
                  (size_t)H * kPh, tj, tid, amax);
    fill_tile<64, kThrP>(sm + kCG, a.gst + (bh * nc + c) * (size_t)(kNs * kPh), (size_t)kPh, kNs, tid, amax);
    const float cl = a.cum[bh * L + t0 + q - 1];
    // packed rows: dl counts the chunk's document starts; only the last
    // document's tokens write into the state the chunk passes on
    const float dl = kPacked ? a.docc[(size_t)b * L + t0 + q - 1] : 0.f;
    if (tid < kB) {
        const bool v = tid < tj;
        const float cj = v ? a.cum[bh * L + t0 + j0 + tid] : 0.f;
        const float dj = (kPacked && v) ? a.docc[(size_t)b * L + t0 + j0 + tid] : 0.f;
        s_cumj[tid] = cj;
        s_dtj[tid] = v ? a.dtv[bh * L + t0 + j0 + tid] : 0.f;
        s_dec[tid] = (v && dj == dl) ? expf(fminf(cl - cj, 0.f)) : 0.f;
        s_docj[tid] = dj;
    }
    // dy_j . x_j exactly in fp32 (thread: token row, quarter ch of p)
    {
        float d = 0.f;
        if (row < tj) {
            const __nv_bfloat16 *xr = static_cast<const __nv_bfloat16 *>(a.x) + ((tokj + row) * H + h) * kPh + 16 * ch;
            const float *dr = a.dy + ((tokj + row) * H + h) * kPh + 16 * ch;
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const uint4 xv = *reinterpret_cast<const uint4 *>(xr + 8 * k);
                const float4 d0 = *reinterpret_cast<const float4 *>(dr + 8 * k);
                const float4 d1 = *reinterpret_cast<const float4 *>(dr + 8 * k + 4);
                d = fmaf(bf16lo(xv.x), d0.x, d); d = fmaf(bf16hi(xv.x), d0.y, d);
                d = fmaf(bf16lo(xv.y), d0.z, d); d = fmaf(bf16hi(xv.y), d0.w, d);
                d = fmaf(bf16lo(xv.z), d1.x, d); d = fmaf(bf16hi(xv.z), d1.y, d);
                d = fmaf(bf16lo(xv.w), d1.z, d); d = fmaf(bf16hi(xv.w), d1.w, d);
            }
        }
        s_dyx[ch * kB + row] = d;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * lg) << 16);
    const uint32_t sbase = smem_u32(sm);
    uint32_t ph = 0, commits = 0;            // completions waited for; commits issued (thread 0)
    bool ok = true;

    // G_c terms: dX = B_J G_c, dB = X_J G_c^T
    if (tid == 0) {
        const uint64_t dBj = sdesc_sw128(sbase + kCBj, 16, 1024), dXj = sdesc_sw128(sbase + kCXj, 16, 1024);
        const uint64_t dGmn = sdesc_sw128(sbase + kCG, kT, 1024), dGk = sdesc_sw128(sbase + kCG, 16, 1024);
#pragma unroll
        for (int s = 0; s < 8; ++s)
            mma_f16(tmem + kTmDX, dBj + (kofs128(s) >> 4), dGmn + ((s * 2048) >> 4), idesc_f16(128, 64, 0, 1), s > 0);
#pragma unroll
        for (int s = 0; s < 4; ++s)
            mma_f16(tmem + kTmDB, dXj + ((s * 32) >> 4), dGk + ((s * 32) >> 4), idesc_f16(128, 128, 0, 0), s > 0);
        mma_commit(bar);
        ++commits;
    }
    // the first i block's operands while the G_c MMAs run (they read other tiles)
    const int nIb = (q + kB - 1) / kB;
    auto fill_i = [&](int Ib) {
        const int i0 = Ib * kB, ti = min(kB, q - i0);
        const size_t toki = (size_t)b * L + t0 + i0;
        fill_tile<128, kThrP>(sm + kCCi, static_cast<const __nv_bfloat16 *>(a.C) + (toki * G + g) * kNs,
                       (size_t)G * kNs, ti, tid, amax);
        fill_tile<64, kThrP>(sm + kCDYi, a.dy + (toki * H + h) * kPh, (size_t)H * kPh, ti, tid, amax);
        if (tid < kB) {
            s_cumi[tid] = tid < ti ? a.cum[bh * L + t0 + i0 + tid] : 0.f;
            s_doci[tid] = (kPacked && tid < ti) ? a.docc[(size_t)b * L + t0 + i0 + tid] : 0.f;
        }
    };
    fill_i(Jb);
    ok = wait_mma(bar, ph);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
        // E_j's dot (B_J row j with the unscaled dB row), then both accumulators times dec_j
        // (this thread: dB columns [32ch, 32ch+32), dX columns [16ch, 16ch+16))
        const float dec = s_dec[row];
        float t32[32];
        tmem_ld32(lane_addr + kTmDB + 32 * ch, t32);
        s_e1[ch * kB + row] = row_dot32(sm + kCBj, row, ch >> 1, 4 * (ch & 1), t32);
#pragma unroll
        for (int k = 0; k < 32; ++k) t32[k] *= dec;
        tmem_st32(lane_addr + kTmDB + 32 * ch, t32);
        float t16[16];
        tmem_ld16(lane_addr + kTmDX + 16 * ch, t16);
#pragma unroll
        for (int k = 0; k < 16; ++k) t16[k] *= dec;
        tmem_st16(lane_addr + kTmDX + 16 * ch, t16);
    }
    float zs = 0.f, zo = 0.f;                          // this thread's i quarter
    for (int Ib = Jb; Ib < nIb; ++Ib) {
        const int i0 = Ib * kB, ti = min(kB, q - i0);
        // the previous pair's MMAs (which read C_I, DY_I, U, V) are complete
        if (Ib > Jb) fill_i(Ib);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0 && ok) {
            tc_fence_after();
            const uint64_t dBj = sdesc_sw128(sbase + kCBj, 16, 1024), dCi = sdesc_sw128(sbase + kCCi, 16, 1024);
            const uint64_t dXj = sdesc_sw128(sbase + kCXj, 16, 1024), dDY = sdesc_sw128(sbase + kCDYi, 16, 1024);
#pragma unroll
            for (int s = 0; s < 8; ++s)
                mma_f16(tmem + kTmCBt, dBj + (kofs128(s) >> 4), dCi + (kofs128(s) >> 4), idesc_f16(128, 128, 0, 0),
                        s > 0);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_f16(tmem + kTmSt, dXj + ((s * 32) >> 4), dDY + ((s * 32) >> 4), idesc_f16(128, 128, 0, 0), s > 0);
            mma_commit(bar);
            ++commits;
        }
        ok = ok && wait_mma(bar, ph);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
            const float cj = s_cumj[row];
            const int gj = j0 + row;
            {
                const int ib = 32 * ch;                // first i of this thread's quarter
                float cb[32], sv[32];
                tmem_ld32(lane_addr + kTmCBt + ib, cb);
                tmem_ld32(lane_addr + kTmSt + ib, sv);
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    const int il = ib + k, gi = i0 + il;
                    const bool v = il < ti && row < tj && gi >= gj && (!kPacked || s_doci[il] == s_docj[row]);
                    const float lw = v ? expf(fminf(s_cumi[il] - cj, 0.f)) : 0.f;
                    const float u = cb[k] * lw, w = sv[k] * lw;
                    const float z = u * sv[k];
                    zs += z;
                    zo += gi > gj ? z : 0.f;
                    cb[k] = u;
                    sv[k] = w;
                }
                store_row32(sm + kCU + (ch >> 1) * kT, row, 4 * (ch & 1), cb, amax);
                store_row32(sm + kCV + (ch >> 1) * kT, row, 4 * (ch & 1), sv, amax);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0 && ok) {
            tc_fence_after();
            const uint64_t dU = sdesc_sw128(sbase + kCU, 16, 1024), dV = sdesc_sw128(sbase + kCV, 16, 1024);
            const uint64_t dDYmn = sdesc_sw128(sbase + kCDYi, kT, 1024);
#pragma unroll
            for (int s = 0; s < 8; ++s)
                mma_f16(tmem + kTmDX, dU + (kofs128(s) >> 4), dDYmn + ((s * 2048) >> 4), idesc_f16(128, 64, 0, 1), 1u);
            // dB's two 64-column halves, each with one 64-wide MN-major tile of C_I
#pragma unroll
            for (int nh = 0; nh < 2; ++nh) {
                const uint64_t dCmn = sdesc_sw128(sbase + kCCi + nh * kT, kT, 1024);
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_f16(tmem + kTmDB + 64 * nh, dV + (kofs128(s) >> 4), dCmn + ((s * 2048) >> 4),
                            idesc_f16(128, 64, 0, 1), 1u);
            }
            mma_commit(bar);
            ++commits;
        }
        ok = ok && wait_mma(bar, ph);
        ok = __all_sync(0xffffffffu, ok);
    }
    s_zs[ch * kB + row] = zs;
    s_zo[ch * kB + row] = zo;
    __syncthreads();
    // (tcgen05.ld is warp-collective: every lane loads, only the block's own
    // tokens store; `ok` is warp-uniform)
    if (ok) {
        const bool mine = row < tj;
        const float dtj = s_dtj[row];
        const size_t tok = tokj + row;
        const float Dh = a.D[h];
        // this thread: dx columns [16ch, 16ch+16), dB columns [32ch, 32ch+32)
        float t16[16];
        tmem_ld16(lane_addr + kTmDX + 16 * ch, t16);
        float *dxr = a.dx + (tok * H + h) * kPh + 16 * ch;
        const float *dyr = a.dy + (tok * H + h) * kPh + 16 * ch;
        if (mine) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float4 d4 = *reinterpret_cast<const float4 *>(dyr + 4 * k);
                *reinterpret_cast<float4 *>(dxr + 4 * k) =
                    make_float4(fmaf(dtj, t16[4 * k], Dh * d4.x), fmaf(dtj, t16[4 * k + 1], Dh * d4.y),
                                fmaf(dtj, t16[4 * k + 2], Dh * d4.z), fmaf(dtj, t16[4 * k + 3], Dh * d4.w));
            }
        }
        float t32[32];
        tmem_ld32(lane_addr + kTmDB + 32 * ch, t32);
        float *dbr = a.dBh + (tok * H + h) * kNs + 32 * ch;
        if (mine) {
#pragma unroll
            for (int k = 0; k < 8; ++k)
                *reinterpret_cast<float4 *>(dbr + 4 * k) =
                    make_float4(dtj * t32[4 * k], dtj * t32[4 * k + 1], dtj * t32[4 * k + 2], dtj * t32[4 * k + 3]);
        }
        if (mine && ch == 0) {
            // the four column quarters' partials, in quarter order
            auto sum4 = [&](const float *v) { return ((v[row] + v[kB + row]) + v[2 * kB + row]) + v[3 * kB + row]; };
            const float dec = s_dec[row];
            const float e1 = sum4(s_e1);
            const float sdst = dec * e1, E = dtj * sdst;
            const size_t o = bh * L + t0 + j0 + row;
            a.ddt_dir[o] = sdst + sum4(s_zs);
            a.dcum_col[o] = -(dtj * sum4(s_zo)) - E;
            a.E[o] = E;
            a.dyx[o] = sum4(s_dyx);
        }
    }
    if (__any_sync(0xffffffffu, !ok) && lane == 0) flag_status(a.status, kStatusTimeout);
    if (lane == 0) finish_range(a.status, amax);
    // after a timeout, let the last MMAs this CTA issued finish (bounded)
    // before its tensor memory is released
    if (tid == 0 && commits > ph) mbar_wait(bar, (commits - 1) & 1u, kBudget);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---- rows -----------------------------------------------------------------
constexpr uint32_t kRCi = 0, kRDYi = 2 * kT, kRH = 3 * kT, kRBj = 4 * kT, kRXj = 6 * kT, kRV = 7 * kT,
                   kRScal = 9 * kT;
// scalars: cum_i, dec_i, cum_j, dt_j, then per column quarter tv[4], rs[4], then the document
// counters doc_i, doc_j of packed rows (128 floats each)
constexpr uint32_t kRBar = kRScal + 14 * kB * 4;
constexpr size_t kRowsSmem = 1024 + kRBar + 16;
constexpr uint32_t kTmCB = 0, kTmS = 128, kTmDC = 256;

template <bool kPacked>
__global__ void __launch_bounds__(kThrP, 1)
tc_rows_kernel(BwdPairArgs a, int L, int H, int G, int Q, int nc) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *s_cumi = reinterpret_cast<float *>(sm + kRScal);
    float *s_dec = s_cumi + kB, *s_cumj = s_dec + kB, *s_dtj = s_cumj + kB;
    float *s_tv = s_dtj + kB, *s_rs = s_tv + 4 * kB;
    float *s_doci = s_rs + 4 * kB, *s_docj = s_doci + kB;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + kRBar);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar + 1);

    const int nI = Q / kB;
    const int c = blockIdx.x / nI, Ib = blockIdx.x - c * nI;
    const int h = blockIdx.y, b = blockIdx.z;
    const int g = h / (H / G);
    const int t0 = c * Q, q = min(Q, L - t0);
    const int i0 = Ib * kB;
    if (i0 >= q) return;                               // uniform over the CTA
    const int ti = min(kB, q - i0);
    const size_t bh = (size_t)b * H + h;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int lg = warp & 3, ch = warp >> 2, row = 32 * lg + lane;
    __half2 amax = __float2half2_rn(0.f);

    if (warp == 0) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    const size_t toki = (size_t)b * L + t0 + i0;
    fill_tile<128, kThrP>(sm + kRCi, static_cast<const __nv_bfloat16 *>(a.C) + (toki * G + g) * kNs,
                   (size_t)G * kNs, ti, tid, amax);
    fill_tile<64, kThrP>(sm + kRDYi, a.dy + (toki * H + h) * kPh, (size_t)H * kPh, ti, tid, amax);
    fill_tile<64, kThrP>(sm + kRH, a.states + (bh * nc + c) * (size_t)(kNs * kPh), (size_t)kPh, kNs, tid, amax);
    if (tid < kB) {
        const bool v = tid < ti;
        const float ci = v ? a.cum[bh * L + t0 + i0 + tid] : 0.f;
        // packed rows: the entering state reaches only the chunk's first document
        const float di = (kPacked && v) ? a.docc[(size_t)b * L + t0 + i0 + tid] : 0.f;
        s_cumi[tid] = ci;
        s_dec[tid] = (v && di == 0.f) ? expf(fminf(ci, 0.f)) : 0.f;
        s_doci[tid] = di;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * lg) << 16);
    const uint32_t sbase = smem_u32(sm);
    uint32_t ph = 0, commits = 0;            // completions waited for; commits issued (thread 0)
    bool ok = true;

    // H_in term: dC = dY_I H_in^T (M=i, N=n, K=p)
    if (tid == 0) {
        const uint64_t dDY = sdesc_sw128(sbase + kRDYi, 16, 1024), dH = sdesc_sw128(sbase + kRH, 16, 1024);
#pragma unroll
        for (int s = 0; s < 4; ++s)
            mma_f16(tmem + kTmDC, dDY + ((s * 32) >> 4), dH + ((s * 32) >> 4), idesc_f16(128, 128, 0, 0), s > 0);
        mma_commit(bar);
        ++commits;
    }
    // the first j block's operands while the H_in MMAs run (they read other tiles)
    auto fill_j = [&](int Jb) {
        const int j0 = Jb * kB, tj = min(kB, q - j0);
        const size_t tokj = (size_t)b * L + t0 + j0;
        fill_tile<128, kThrP>(sm + kRBj, static_cast<const __nv_bfloat16 *>(a.B) + (tokj * G + g) * kNs,
                       (size_t)G * kNs, tj, tid, amax);
        fill_tile<64, kThrP>(sm + kRXj, static_cast<const __nv_bfloat16 *>(a.x) + (tokj * H + h) * kPh,
                      (size_t)H * kPh, tj, tid, amax);
        if (tid < kB) {
            s_cumj[tid] = tid < tj ? a.cum[bh * L + t0 + j0 + tid] : 0.f;
            s_dtj[tid] = tid < tj ? a.dtv[bh * L + t0 + j0 + tid] : 0.f;
            s_docj[tid] = (kPacked && tid < tj) ? a.docc[(size_t)b * L + t0 + j0 + tid] : 0.f;
        }
    };
    fill_j(0);
    ok = wait_mma(bar, ph);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
        // T_i's dot (C_I row i with the unscaled dC row), then the accumulator times dec_i
        // (this thread: dC columns [32ch, 32ch+32))
        const float dec = s_dec[row];
        float t32[32];
        tmem_ld32(lane_addr + kTmDC + 32 * ch, t32);
        s_tv[ch * kB + row] = row_dot32(sm + kRCi, row, ch >> 1, 4 * (ch & 1), t32);
#pragma unroll
        for (int k = 0; k < 32; ++k) t32[k] *= dec;
        tmem_st32(lane_addr + kTmDC + 32 * ch, t32);
    }
    float rs = 0.f;                                    // sum over this thread's j quarter of CB_ij V_ij, j < i
    const float ci = s_cumi[row];
    const int gi = i0 + row;
    for (int Jb = 0; Jb <= Ib; ++Jb) {
        const int j0 = Jb * kB, tj = min(kB, q - j0);
        // the previous pair's MMAs (which read B_J, V) are complete
        if (Jb > 0) fill_j(Jb);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0 && ok) {
            tc_fence_after();
            const uint64_t dCi = sdesc_sw128(sbase + kRCi, 16, 1024), dBj = sdesc_sw128(sbase + kRBj, 16, 1024);
            const uint64_t dDY = sdesc_sw128(sbase + kRDYi, 16, 1024), dXj = sdesc_sw128(sbase + kRXj, 16, 1024);
#pragma unroll
            for (int s = 0; s < 8; ++s)
                mma_f16(tmem + kTmCB, dCi + (kofs128(s) >> 4), dBj + (kofs128(s) >> 4), idesc_f16(128, 128, 0, 0),
                        s > 0);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_f16(tmem + kTmS, dDY + ((s * 32) >> 4), dXj + ((s * 32) >> 4), idesc_f16(128, 128, 0, 0), s > 0);
            mma_commit(bar);
            ++commits;
        }
        ok = ok && wait_mma(bar, ph);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
            {
                const int jb = 32 * ch;
                float cb[32], sv[32];
                tmem_ld32(lane_addr + kTmCB + jb, cb);
                tmem_ld32(lane_addr + kTmS + jb, sv);
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    const int jl = jb + k, gj = j0 + jl;
                    const bool v = jl < tj && row < ti && gi >= gj && (!kPacked || s_doci[row] == s_docj[jl]);
                    const float w = v ? sv[k] * expf(fminf(ci - s_cumj[jl], 0.f)) * s_dtj[jl] : 0.f;
                    rs += gi > gj ? cb[k] * w : 0.f;
                    sv[k] = w;
                }
                store_row32(sm + kRV + (ch >> 1) * kT, row, 4 * (ch & 1), sv, amax);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0 && ok) {
            tc_fence_after();
            const uint64_t dV = sdesc_sw128(sbase + kRV, 16, 1024);
            // dC's two 64-column halves, each with one 64-wide MN-major tile of B_J
#pragma unroll
            for (int nh = 0; nh < 2; ++nh) {
                const uint64_t dBmn = sdesc_sw128(sbase + kRBj + nh * kT, kT, 1024);
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_f16(tmem + kTmDC + 64 * nh, dV + (kofs128(s) >> 4), dBmn + ((s * 2048) >> 4),
                            idesc_f16(128, 64, 0, 1), 1u);
            }
            mma_commit(bar);
            ++commits;
        }
        ok = ok && wait_mma(bar, ph);
        ok = __all_sync(0xffffffffu, ok);
    }
    s_rs[ch * kB + row] = rs;
    __syncthreads();
    // (tcgen05.ld is warp-collective: every lane loads, only the block's own
    // tokens store; `ok` is warp-uniform)
    if (ok) {
        const bool mine = row < ti;
        const size_t tok = toki + row;
        float *dcr = a.dCh + (tok * H + h) * kNs + 32 * ch;
        float t32[32];
        tmem_ld32(lane_addr + kTmDC + 32 * ch, t32);
        if (mine) {
#pragma unroll
            for (int k = 0; k < 8; ++k)
                *reinterpret_cast<float4 *>(dcr + 4 * k) =
                    make_float4(t32[4 * k], t32[4 * k + 1], t32[4 * k + 2], t32[4 * k + 3]);
        }
        if (mine && ch == 0) {
            // the four column quarters' partials, in quarter order
            auto sum4 = [&](const float *v) { return ((v[row] + v[kB + row]) + v[2 * kB + row]) + v[3 * kB + row]; };
            const float tv = s_dec[row] * sum4(s_tv);
            a.dcum_row[bh * L + t0 + i0 + row] = tv + sum4(s_rs);
        }
    }
    if (__any_sync(0xffffffffu, !ok) && lane == 0) flag_status(a.status, kStatusTimeout);
    if (lane == 0) finish_range(a.status, amax);
    // after a timeout, let the last MMAs this CTA issued finish (bounded)
    // before its tensor memory is released
    if (tid == 0 && commits > ph) mbar_wait(bar, (commits - 1) & 1u, kBudget);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---- states ---------------------------------------------------------------
// per (chunk, head, batch): dt, cum, ell, and the two per-chunk N x P sums,
// block by block of 128 tokens:
//   S_c  += B_k^T (w x)_k     w_j = e^{min(cl-cum_j,0)} dt_j   (M=128 n, N=64 p, K=128 j)
//   dS_c += C_k^T (e dy)_k    e_i = e^{min(cum_i,0)}            (M=128 n, N=64 p, K=128 i)
// (the operand forms of the forward's unit-state MMA: B and C tiles read
// MN-major, the scaled x and dy tiles MN-major).  TMEM lane = state row n.
constexpr int kQMax = 1024;
constexpr uint32_t kSB = 0, kSWX = 2 * kT, kSC = 3 * kT, kSEDY = 5 * kT, kSScal = 6 * kT;
// scalars: dt[kQMax], cum[kQMax], w[128], e[128], warp totals[32]
constexpr uint32_t kSBar = kSScal + (2 * kQMax + 2 * kB + 32) * 4;
constexpr size_t kStatesSmem = 1024 + kSBar + 16;

template <bool kPacked>
__global__ void __launch_bounds__(kThr, 2)
tc_states_kernel(BwdStatesArgs a, int L, int H, int G, int Q, int nc) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *s_dt = reinterpret_cast<float *>(sm + kSScal);
    float *s_cum = s_dt + kQMax, *s_w = s_cum + kQMax, *s_e = s_w + kB, *s_wt = s_e + kB;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + kSBar);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar + 1);

    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int g = h / (H / G);
    const int t0 = c * Q, q = min(Q, L - t0);
    const size_t bh = (size_t)b * H + h;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int lg = warp & 3, ch = warp >> 2, row = 32 * lg + lane;
    const float Ah = a.A[h], bias = a.dt_bias[h];
    __half2 amax = __float2half2_rn(0.f);
    if (tid == 0 && Ah > 0.f) flag_status(a.status, kStatusPrecondition);
    if (warp == 0) {
        tmem_alloc(tslot, 128);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    // dt = clamp(softplus(dt_raw + dt_bias)) and its inclusive cumsum times A (fixed order)
    float carry = 0.f;
    for (int base = 0; base < q; base += kThr) {
        const int i = base + tid;
        const float d = i < q ? dt_of(a.dt_raw[((size_t)b * L + t0 + i) * H + h], bias, a.dt_lo, a.dt_hi) : 0.f;
        float tot;
        const float sc = block_inclusive_scan(d * Ah, s_wt, tot) + carry;
        if (i < q) {
            s_dt[i] = d;
            s_cum[i] = sc;
            a.dtv[bh * L + t0 + i] = d;
            a.cum[bh * L + t0 + i] = sc;
        }
        carry += tot;
    }
    __syncthreads();
    const float cl = s_cum[q - 1];
    // packed rows: a chunk that holds a document start passes no decayed state on
    const float dl = kPacked ? a.docc[(size_t)b * L + t0 + q - 1] : 0.f;
    if (tid == 0) a.ell[bh * nc + c] = dl > 0.f ? -INFINITY : cl;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * lg) << 16);
    const uint32_t sbase = smem_u32(sm);
    uint32_t ph = 0, commits = 0;
    bool ok = true;
    const int nk = (q + kB - 1) / kB;
    for (int kb = 0; kb < nk; ++kb) {
        const int j0 = kb * kB, nr = min(kB, q - j0);
        const size_t tok = (size_t)b * L + t0 + j0;
        if (tid < kB) {
            const bool v = tid < nr;
            // packed rows: only the last document writes the chunk state, only the
            // first reads the entering state
            const float dj = (kPacked && v) ? a.docc[(size_t)b * L + t0 + j0 + tid] : 0.f;
            s_w[tid] = (v && dj == dl) ? expf(fminf(cl - s_cum[j0 + tid], 0.f)) * s_dt[j0 + tid] : 0.f;
            s_e[tid] = (v && dj == 0.f) ? expf(fminf(s_cum[j0 + tid], 0.f)) : 0.f;
        }
        __syncthreads();                               // the previous block's MMAs are complete
        fill_tile<128, kThr>(sm + kSB, static_cast<const __nv_bfloat16 *>(a.B) + (tok * G + g) * kNs,
                       (size_t)G * kNs, nr, tid, amax);
        fill_tile<128, kThr>(sm + kSC, static_cast<const __nv_bfloat16 *>(a.C) + (tok * G + g) * kNs,
                       (size_t)G * kNs, nr, tid, amax);
        fill_tile<64, kThr>(sm + kSWX, static_cast<const __nv_bfloat16 *>(a.x) + (tok * H + h) * kPh,
                            (size_t)H * kPh, nr,
                      tid, amax, s_w);
        fill_tile<64, kThr>(sm + kSEDY, a.dy + (tok * H + h) * kPh, (size_t)H * kPh, nr, tid, amax, s_e);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0 && ok) {
            tc_fence_after();
            const uint64_t dB = sdesc_sw128(sbase + kSB, kT, 1024), dWX = sdesc_sw128(sbase + kSWX, kT, 1024);
            const uint64_t dC = sdesc_sw128(sbase + kSC, kT, 1024), dE = sdesc_sw128(sbase + kSEDY, kT, 1024);
#pragma unroll
            for (int s8 = 0; s8 < 8; ++s8)
                mma_f16(tmem, dB + ((s8 * 2048) >> 4), dWX + ((s8 * 2048) >> 4), idesc_f16(128, 64, 1, 1),
                        (kb > 0 || s8 > 0) ? 1u : 0u);
#pragma unroll
            for (int s8 = 0; s8 < 8; ++s8)
                mma_f16(tmem + 64, dC + ((s8 * 2048) >> 4), dE + ((s8 * 2048) >> 4), idesc_f16(128, 64, 1, 1),
                        (kb > 0 || s8 > 0) ? 1u : 0u);
            mma_commit(bar);
            ++commits;
        }
        ok = ok && wait_mma(bar, ph);
        ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
        // lane n of TMEM is state row n; this thread's 32 of the 64 p columns
        float t32[32];
        const size_t off = (bh * nc + c) * (size_t)(kNs * kPh) + (size_t)row * kPh + 32 * ch;
        tmem_ld32(lane_addr + 32 * ch, t32);
#pragma unroll
        for (int k = 0; k < 8; ++k)
            *reinterpret_cast<float4 *>(a.states + off + 4 * k) =
                make_float4(t32[4 * k], t32[4 * k + 1], t32[4 * k + 2], t32[4 * k + 3]);
        tmem_ld32(lane_addr + 64 + 32 * ch, t32);
#pragma unroll
        for (int k = 0; k < 8; ++k)
            *reinterpret_cast<float4 *>(a.gst + off + 4 * k) =
                make_float4(t32[4 * k], t32[4 * k + 1], t32[4 * k + 2], t32[4 * k + 3]);
    }
    if (__any_sync(0xffffffffu, !ok) && lane == 0) flag_status(a.status, kStatusTimeout);
    if (lane == 0) finish_range(a.status, amax);
    if (tid == 0 && commits > ph) mbar_wait(bar, (commits - 1) & 1u, kBudget);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

}  // namespace

bool bwd_tc_supported(const ScanDims &d, int bf16, int packed) {
    (void)packed;                      // packed rows: value masks from the document counters
    if (!bf16 || d.P != kPh || d.N != kNs || d.Q % kB != 0 || d.Q > kQMax) return false;
    if (d.H > 65535 || d.b > 65535 || d.nc * (d.Q / kB) > 0x7fffffffll) return false;
    return true;
}

cudaError_t bwd_tc_states(const BwdStatesArgs &a, const ScanDims &d, cudaStream_t s) {
    static bool attr_done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_done[dev]) {
        if ((e = cudaFuncSetAttribute(tc_states_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)kStatesSmem)) != cudaSuccess ||
            (e = cudaFuncSetAttribute(tc_states_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)kStatesSmem)) != cudaSuccess)
            return e;
        attr_done[dev] = true;
    }
    TraceScope tr(s, kTrBwdStates);
    const dim3 grid((unsigned)d.nc, (unsigned)d.H, (unsigned)d.b);
    if (a.docc)
        tc_states_kernel<true><<<grid, kThr, kStatesSmem, s>>>(a, (int)d.L, (int)d.H, (int)d.G, (int)d.Q, (int)d.nc);
    else
        tc_states_kernel<false><<<grid, kThr, kStatesSmem, s>>>(a, (int)d.L, (int)d.H, (int)d.G, (int)d.Q, (int)d.nc);
    return cudaGetLastError();
}

cudaError_t bwd_tc_pairs(const BwdPairArgs &a, const ScanDims &d, cudaStream_t s) {
    static bool attr_done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_done[dev]) {
        for (auto k : {tc_cols_kernel<false>, tc_cols_kernel<true>})
            if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kColsSmem)) !=
                cudaSuccess)
                return e;
        for (auto k : {tc_rows_kernel<false>, tc_rows_kernel<true>})
            if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRowsSmem)) !=
                cudaSuccess)
                return e;
        attr_done[dev] = true;
    }
    const dim3 grid((unsigned)(d.nc * (d.Q / kB)), (unsigned)d.H, (unsigned)d.b);
    {
        TraceScope tr(s, kTrBwdCols);
        auto k = a.docc ? tc_cols_kernel<true> : tc_cols_kernel<false>;
        k<<<grid, kThrP, kColsSmem, s>>>(a, (int)d.L, (int)d.H, (int)d.G, (int)d.Q, (int)d.nc);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        TraceScope tr(s, kTrBwdRows);
        auto k = a.docc ? tc_rows_kernel<true> : tc_rows_kernel<false>;
        k<<<grid, kThrP, kRowsSmem, s>>>(a, (int)d.L, (int)d.H, (int)d.G, (int)d.Q, (int)d.nc);
    }
    return cudaGetLastError();
}

}  // namespace ssd
