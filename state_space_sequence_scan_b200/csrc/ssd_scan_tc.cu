// Chunked SSD forward scan on the sm_100a tensor cores (tcgen05 + TMEM).
//
// Scope: bf16 x/B/C, state_dim N = 128, head_dim P = 64, fp32 dt/A/D/state,
// fp32 y.  Every contraction runs as a kind::f16 MMA with fp16 operands
// (bf16 inputs are widened exactly; the decay-weighted operands need fp16's
// 11-bit significand, bf16's 8 bits are not enough for the 2e-2 bar) and
// fp32 accumulation in TMEM.
//
// The sequence of every (batch, head) is cut into 128-token blocks (the MMA
// M extent) and the blocks into `units` of consecutive blocks.  Four
// launches, no kernel waits on another CTA:
//   dt_prep     dt = clamp(softplus(dt_raw + dt_bias)), dA = dt*A, and the
//               inclusive cumsum `cum` of dA inside every 128-token block
//               (warp shuffles, fixed order), transposed to [b, H, L].
//   unit_state  per (unit u, head, batch), units 0..U-2: the state the unit
//               leaves when it starts from zero,
//                 S'_u = sum_{j in u} exp(sum_{r=j+1..end(u)} dA_r) dt_j B_j x_j^T
//               as ONE accumulated MMA over the unit's tokens:
//               D[n,p] += B^T[n,j] (w x)[j,p]  (M=128 n, N=64 p, K=16 per step).
//   state_pass  per (b, h, state element), serial over units:
//               H_in(0) = init (or 0),  H_in(u+1) = exp(ell_u) H_in(u) + S'_u.
//   chunk_out   per (unit, head, batch): starting from H_in(u), for each
//               128-token block in order (state H fp32 in TMEM):
//                 Z   = C H                    (M=128 i, N=64 p, K=128 n)
//                 CB  = C B^T                  (M=128 i, N=128 j, K=128 n)
//                 W   = CB .* exp(cum_i - cum_j) dt_j on j <= i, 0 above
//                 Y   = W X                    (M=128 i, N=64 p, K=128 j)
//                 y_i = Y_i + exp(cum_i) Z_i + D x_i
//                 H   = exp(cum_last) H + B^T (w X),  w_j = exp(cum_last - cum_j) dt_j
//               and the last unit writes final_state.
// This is the chunked form of the scan ("Mamba2" knowledge page: intra-chunk
// parallel in matrix-multiplication form, inter-chunk serial) with the
// intra-chunk quadratic term evaluated on 128-token blocks and the state
// carried on chip between them; it equals the token recurrence up to
// rounding for any chunk size (nnterp guide "Mamba-2", "The state after every
// token").  Exponents are only taken of min(., 0) after the causal select,
// so none can overflow.
#include <stdint.h>

#include "ssd_common.cuh"
#include "ssd_internal.h"
#include "ssd_tc.cuh"
#include "ssd_trace.h"

namespace ssd {
namespace {

using namespace tc;

constexpr int kBlk = 128;                       // tokens per block
constexpr int kN = 128;                         // state_dim
constexpr int kP = 64;                          // head_dim
constexpr int kNP = kN * kP;
constexpr int kTcThreads = 128;
constexpr long long kWaitBudget = 1ll << 32;    // clock cycles before an MMA wait gives up (~2 s)
constexpr float kF16Max = 65504.0f;
constexpr int kUnitTarget = 8 * 148;            // aim for ~8 units per SM across the grid

struct TcWs {
    unsigned *status;
    float *dt;      // [b, H, nblk*128]
    float *cum;     // [b, H, nblk*128]
    float *ell;     // [b, H, U]
    float *states;  // [b, H, U, N, P]
};

struct TcPlan {
    int64_t nblk, U, bpu;
};

TcPlan make_plan(const ScanDims &d) {
    TcPlan p;
    p.nblk = (d.L + kBlk - 1) / kBlk;
    int64_t U = 1;
    while (d.b * d.H * U < kUnitTarget && U < p.nblk) U *= 2;
    if (U > p.nblk) U = p.nblk;
    if (U < 1) U = 1;
    p.bpu = (p.nblk + U - 1) / U;
    p.U = (p.nblk + p.bpu - 1) / p.bpu;
    return p;
}

TcWs carve(const ScanDims &d, const TcPlan &p, void *ws) {
    char *c = static_cast<char *>(ws);
    TcWs w;
    w.status = reinterpret_cast<unsigned *>(c);
    size_t off = kStatusBytes;
    const size_t tok = (size_t)d.b * d.H * p.nblk * kBlk * sizeof(float);
    w.dt = reinterpret_cast<float *>(c + off); off += align256(tok);
    w.cum = reinterpret_cast<float *>(c + off); off += align256(tok);
    w.ell = reinterpret_cast<float *>(c + off); off += align256((size_t)d.b * d.H * p.U * sizeof(float));
    w.states = reinterpret_cast<float *>(c + off);
    return w;
}

size_t ws_bytes(const ScanDims &d, const TcPlan &p) {
    const size_t tok = (size_t)d.b * d.H * p.nblk * kBlk * sizeof(float);
    return kStatusBytes + 2 * align256(tok) + align256((size_t)d.b * d.H * p.U * sizeof(float)) +
           align256((size_t)d.b * d.H * p.U * kNP * sizeof(float));
}

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ uint4 ldg16(const void *p) { return __ldg(reinterpret_cast<const uint4 *>(p)); }

// 8 bf16 (one 16-byte chunk) -> 8 fp16; flags values outside the fp16 range
__device__ __forceinline__ uint4 cvt_chunk(uint4 v, bool &range_ok) {
    const float f[8] = {bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y),
                        bf16lo(v.z), bf16hi(v.z), bf16lo(v.w), bf16hi(v.w)};
#pragma unroll
    for (int i = 0; i < 8; ++i) range_ok &= fabsf(f[i]) <= kF16Max;
    return make_uint4(pack_h2(f[0], f[1]), pack_h2(f[2], f[3]), pack_h2(f[4], f[5]), pack_h2(f[6], f[7]));
}

// 8 bf16 scaled by w -> 8 fp16
__device__ __forceinline__ uint4 cvt_chunk_scaled(uint4 v, float w, bool &range_ok) {
    const float f[8] = {w * bf16lo(v.x), w * bf16hi(v.x), w * bf16lo(v.y), w * bf16hi(v.y),
                        w * bf16lo(v.z), w * bf16hi(v.z), w * bf16lo(v.w), w * bf16hi(v.w)};
#pragma unroll
    for (int i = 0; i < 8; ++i) range_ok &= fabsf(f[i]) <= kF16Max;
    return make_uint4(pack_h2(f[0], f[1]), pack_h2(f[2], f[3]), pack_h2(f[4], f[5]), pack_h2(f[6], f[7]));
}

__device__ __forceinline__ uint4 pack8(const float *f, bool &range_ok) {
#pragma unroll
    for (int i = 0; i < 8; ++i) range_ok &= fabsf(f[i]) <= kF16Max;
    return make_uint4(pack_h2(f[0], f[1]), pack_h2(f[2], f[3]), pack_h2(f[4], f[5]), pack_h2(f[6], f[7]));
}

// ---------------------------------------------------------------------------
// dt_prep: grid (nblk, ceil(H/32), b), 256 threads.
__global__ void __launch_bounds__(256)
dt_prep_kernel(const float *__restrict__ dt_raw, const float *__restrict__ dt_bias,
               const float *__restrict__ A, TcWs ws, int L, int H, int nblk, float lo, float hi) {
    __shared__ float s_dt[kBlk][33];
    __shared__ float s_da[kBlk][33];
    const int blk = blockIdx.x, h0 = blockIdx.y * 32, b = blockIdx.z;
    const int nh = min(32, H - h0);
    for (int e = threadIdx.x; e < kBlk * 32; e += 256) {
        const int tok = e >> 5, hh = e & 31;
        const int t = blk * kBlk + tok;
        float d = 0.f, da = 0.f;
        if (hh < nh && t < L) {
            const int h = h0 + hh;
            d = dt_of(dt_raw[((size_t)b * L + t) * H + h], dt_bias[h], lo, hi);
            da = d * A[h];
        }
        s_dt[tok][hh] = d;
        s_da[tok][hh] = da;
    }
    if (blk == 0 && b == 0 && threadIdx.x < nh && A[h0 + threadIdx.x] > 0.f)
        flag_status(ws.status, kStatusPrecondition);
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int hh = warp; hh < nh; hh += 8) {
        const float v0 = s_da[4 * lane][hh], v1 = s_da[4 * lane + 1][hh];
        const float v2 = s_da[4 * lane + 2][hh], v3 = s_da[4 * lane + 3][hh];
        const float c0 = v0, c1 = c0 + v1, c2 = c1 + v2, c3 = c2 + v3;
        float incl = c3;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float u = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += u;
        }
        const float ex = incl - c3;
        const size_t base = ((size_t)b * H + h0 + hh) * (size_t)nblk * kBlk + (size_t)blk * kBlk + 4 * lane;
        *reinterpret_cast<float4 *>(ws.cum + base) = make_float4(ex + c0, ex + c1, ex + c2, ex + c3);
        *reinterpret_cast<float4 *>(ws.dt + base) =
            make_float4(s_dt[4 * lane][hh], s_dt[4 * lane + 1][hh], s_dt[4 * lane + 2][hh], s_dt[4 * lane + 3][hh]);
    }
}

// ---------------------------------------------------------------------------
// unit_state: grid (H, U-1, b), 128 threads.
constexpr size_t kUsSmem = 1024 + 32768 + 16384 + 128 * 4 + 4096 * 4 + 64;

__global__ void __launch_bounds__(kTcThreads)
unit_state_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ Bm, TcWs ws, int L,
                  int H, int G, int nblk, int U, int bpu) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    uint8_t *sB = sm;                                          // [128 j][128 n] fp16
    uint8_t *sWX = sm + 32768;                                 // [128 j][64 p] fp16
    float *s_w = reinterpret_cast<float *>(sm + 49152);        // 128
    float *s_suf = s_w + kBlk;                                 // bpu (<= 4096)
    uint64_t *mbar = reinterpret_cast<uint64_t *>(s_suf + 4096);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(mbar + 1);

    const int h = blockIdx.x, u = blockIdx.y, b = blockIdx.z;
    const int g = h / (H / G);
    const int tid = threadIdx.x, warp = tid >> 5;
    const size_t bh = (size_t)b * H + h;
    const int kb0 = u * bpu, kb1 = min(nblk, kb0 + bpu);
    const float *cum = ws.cum + bh * (size_t)nblk * kBlk;
    const float *dtv = ws.dt + bh * (size_t)nblk * kBlk;

    if (warp == 0) {
        tmem_alloc(tslot, 64);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(mbar, 1);
        fence_mbar_init();
        float acc = 0.f;
        for (int k = kb1 - 1; k >= kb0; --k) {    // suffix sums of the block totals
            s_suf[k - kb0] = acc;
            acc += cum[(size_t)k * kBlk + kBlk - 1];
        }
        ws.ell[bh * U + u] = acc;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;

    bool ok = true, range_ok = true;
    uint32_t phase = 0;
    const uint32_t idesc = idesc_f16(128, 64, 1, 1);
    for (int k = kb0; k < kb1; ++k) {
        const int t0 = k * kBlk;
        {
            const float e = cum[t0 + kBlk - 1] - cum[t0 + tid] + s_suf[k - kb0];
            s_w[tid] = expf(fminf(e, 0.f)) * dtv[t0 + tid];
        }
        __syncthreads();
        for (int c = tid; c < kBlk * 16; c += kTcThreads) {
            const int r = c >> 4, kk = c & 15, t = t0 + r;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (t < L) v = ldg16(Bm + (((size_t)b * L + t) * G + g) * kN + kk * 8);
            *reinterpret_cast<uint4 *>(sB + (kk >> 3) * 16384 + sw128_off(r, kk & 7)) = cvt_chunk(v, range_ok);
        }
        for (int c = tid; c < kBlk * 8; c += kTcThreads) {
            const int r = c >> 3, kk = c & 7, t = t0 + r;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (t < L) v = ldg16(x + (((size_t)b * L + t) * H + h) * kP + kk * 8);
            *reinterpret_cast<uint4 *>(sWX + sw128_off(r, kk)) = cvt_chunk_scaled(v, s_w[r], range_ok);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
            const uint32_t b_base = smem_u32(sB), w_base = smem_u32(sWX);
#pragma unroll
            for (int s = 0; s < 8; ++s)
                mma_f16(tmem, sdesc_sw128(b_base + s * 2048, 16384, 1024), sdesc_sw128(w_base + s * 2048, 16384, 1024),
                        idesc, (k > kb0 || s > 0) ? 1u : 0u);
            mma_commit(mbar);
        }
        ok = __syncthreads_and(mbar_wait(mbar, phase, kWaitBudget));
        phase ^= 1u;
        if (!ok) break;
        tc_fence_after();
    }
    if (!ok) {
        if (tid == 0) flag_status(ws.status, kStatusTimeout);
    } else {
        float *dst = ws.states + (bh * U + u) * (size_t)kNP + (size_t)tid * kP;
        const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float v[32];
            tmem_ld32(lane_addr + half * 32, v);
#pragma unroll
            for (int q = 0; q < 8; ++q)
                *reinterpret_cast<float4 *>(dst + half * 32 + 4 * q) =
                    make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
    }
    if (!__syncthreads_and(range_ok) && tid == 0) flag_status(ws.status, kStatusRange);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 64);
}

// ---------------------------------------------------------------------------
// state_pass: grid (N*P/256, H, b), 256 threads.
__global__ void __launch_bounds__(256)
tc_state_pass_kernel(TcWs ws, const float *__restrict__ init, int H, int U) {
    const int e = blockIdx.x * 256 + threadIdx.x;
    const size_t bh = (size_t)blockIdx.z * H + blockIdx.y;
    float hs = init ? init[bh * kNP + e] : 0.f;
    float *S = ws.states + bh * (size_t)U * kNP + e;
    const float *ell = ws.ell + bh * U;
    for (int u = 0; u + 1 < U; ++u) {
        const float s = S[(size_t)u * kNP];
        S[(size_t)u * kNP] = hs;                  // state entering unit u
        hs = fmaf(expf(fminf(ell[u], 0.f)), hs, s);
    }
    S[(size_t)(U - 1) * kNP] = hs;
}

// ---------------------------------------------------------------------------
// chunk_out: grid (H, U, b), 128 threads, 2 CTAs per SM.
constexpr size_t kCoSmem = 1024 + 32768 * 2 + 16384 * 2 + 2 * kBlk * 4 + 64;

__global__ void __launch_bounds__(kTcThreads, 2)
chunk_out_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ Bm,
                 const __nv_bfloat16 *__restrict__ Cm, const float *__restrict__ D,
                 const float *__restrict__ init, float *__restrict__ y, float *__restrict__ final_state, TcWs ws,
                 int L, int H, int G, int nblk, int U, int bpu, int states_from_ws) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    uint8_t *sCW = sm;                      // C tile [128 i][128 n], then W tile [128 i][128 j]
    uint8_t *sB = sm + 32768;               // B tile [128 j][128 n]
    uint8_t *sX = sm + 65536;               // X tile [128 j][64 p]
    uint8_t *sHW = sm + 81920;              // fp16 state [128 n][64 p], then w.X [128 j][64 p]
    float *s_dt = reinterpret_cast<float *>(sm + 98304);
    float *s_cum = s_dt + kBlk;
    uint64_t *mbar = reinterpret_cast<uint64_t *>(s_cum + kBlk);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(mbar + 1);

    const int h = blockIdx.x, u = blockIdx.y, b = blockIdx.z;
    const int g = h / (H / G);
    const int tid = threadIdx.x, warp = tid >> 5;
    const size_t bh = (size_t)b * H + h;
    const int kb0 = u * bpu, kb1 = min(nblk, kb0 + bpu);
    const float *cum = ws.cum + bh * (size_t)nblk * kBlk;
    const float *dtv = ws.dt + bh * (size_t)nblk * kBlk;

    if (warp == 0) {
        tmem_alloc(tslot, 256);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(mbar, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    const uint32_t tH = 0, tZ = 64, tCB = 128;   // TMEM columns: state, C.H, C.B^T then Y
    bool range_ok = true;

    // state entering the unit -> TMEM (fp32) and sHW (fp16); thread tid owns row n = tid
    {
        const float *src = states_from_ws ? ws.states + (bh * U + u) * (size_t)kNP
                                          : (init ? init + bh * kNP : nullptr);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float v[32];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                float4 f = src ? *reinterpret_cast<const float4 *>(src + (size_t)tid * kP + half * 32 + 4 * q)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
                v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
            }
            tmem_st32(lane_addr + tH + half * 32, v);
#pragma unroll
            for (int q = 0; q < 4; ++q)
                *reinterpret_cast<uint4 *>(sHW + sw128_off(tid, half * 4 + q)) = pack8(v + 8 * q, range_ok);
        }
    }

    bool ok = true;
    uint32_t phase = 0;
    const uint32_t idesc_z = idesc_f16(128, 64, 0, 1);    // A=C K-major, B=H MN-major
    const uint32_t idesc_cb = idesc_f16(128, 128, 0, 0);  // A=C K-major, B=B K-major
    const uint32_t idesc_y = idesc_f16(128, 64, 0, 1);    // A=W K-major, B=X MN-major
    const uint32_t idesc_s = idesc_f16(128, 64, 1, 1);    // A=B^T MN-major, B=wX MN-major
    const float Dh = D[h];

    for (int k = kb0; k < kb1 && ok; ++k) {
        const int t0 = k * kBlk;
        s_dt[tid] = dtv[t0 + tid];
        s_cum[tid] = cum[t0 + tid];
        for (int c = tid; c < kBlk * 16; c += kTcThreads) {
            const int r = c >> 4, kk = c & 15, t = t0 + r;
            uint4 vc = make_uint4(0u, 0u, 0u, 0u), vb = vc;
            if (t < L) {
                const size_t off = (((size_t)b * L + t) * G + g) * kN + kk * 8;
                vc = ldg16(Cm + off);
                vb = ldg16(Bm + off);
            }
            const uint32_t o = (kk >> 3) * 16384 + sw128_off(r, kk & 7);
            *reinterpret_cast<uint4 *>(sCW + o) = cvt_chunk(vc, range_ok);
            *reinterpret_cast<uint4 *>(sB + o) = cvt_chunk(vb, range_ok);
        }
        for (int c = tid; c < kBlk * 8; c += kTcThreads) {
            const int r = c >> 3, kk = c & 7, t = t0 + r;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (t < L) v = ldg16(x + (((size_t)b * L + t) * H + h) * kP + kk * 8);
            *reinterpret_cast<uint4 *>(sX + sw128_off(r, kk)) = cvt_chunk(v, range_ok);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        if (tid == 0) {
            const uint32_t c_base = smem_u32(sCW), b_base = smem_u32(sB), h_base = smem_u32(sHW);
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const uint64_t ad = sdesc_sw128(c_base + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024);
                mma_f16(tmem + tZ, ad, sdesc_sw128(h_base + s * 2048, 16384, 1024), idesc_z, s > 0);
                mma_f16(tmem + tCB, ad, sdesc_sw128(b_base + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024), idesc_cb,
                        s > 0);
            }
            mma_commit(mbar);
        }
        ok = __syncthreads_and(mbar_wait(mbar, phase, kWaitBudget));
        phase ^= 1u;
        if (!ok) break;
        tc_fence_after();

        // W row i = tid (K-major over j), w.X row j = tid, state scaled by the block decay
        {
            const int i = tid;
            const float ci = s_cum[i];
#pragma unroll
            for (int c32 = 0; c32 < 4; ++c32) {
                uint4 out[4];
                if (c32 <= warp) {                       // warp-uniform: rows 32w.. see columns < 32(w+1)
                    float v[32];
                    tmem_ld32(lane_addr + tCB + c32 * 32, v);
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        const int j = c32 * 32 + jj;
                        v[jj] = (j <= i) ? v[jj] * expf(fminf(ci - s_cum[j], 0.f)) * s_dt[j] : 0.f;
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q) out[q] = pack8(v + 8 * q, range_ok);
                } else {
#pragma unroll
                    for (int q = 0; q < 4; ++q) out[q] = make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<uint4 *>(sCW + (c32 >> 1) * 16384 + sw128_off(i, (c32 & 1) * 4 + q)) = out[q];
            }
            const float clast = s_cum[kBlk - 1];
            const float wj = expf(fminf(clast - s_cum[tid], 0.f)) * s_dt[tid];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint4 xv = *reinterpret_cast<const uint4 *>(sX + sw128_off(tid, q));
                float f[8];
                const float2 a0 = unpack_h2(xv.x), a1 = unpack_h2(xv.y), a2 = unpack_h2(xv.z), a3 = unpack_h2(xv.w);
                f[0] = wj * a0.x; f[1] = wj * a0.y; f[2] = wj * a1.x; f[3] = wj * a1.y;
                f[4] = wj * a2.x; f[5] = wj * a2.y; f[6] = wj * a3.x; f[7] = wj * a3.y;
                *reinterpret_cast<uint4 *>(sHW + sw128_off(tid, q)) = pack8(f, range_ok);
            }
            const float decay = expf(fminf(clast, 0.f));
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float v[32];
                tmem_ld32(lane_addr + tH + half * 32, v);
#pragma unroll
                for (int q = 0; q < 32; ++q) v[q] *= decay;
                tmem_st32(lane_addr + tH + half * 32, v);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        if (tid == 0) {
            const uint32_t w_base = smem_u32(sCW), x_base = smem_u32(sX), b_base = smem_u32(sB),
                           wx_base = smem_u32(sHW);
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                mma_f16(tmem + tCB, sdesc_sw128(w_base + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024),
                        sdesc_sw128(x_base + s * 2048, 16384, 1024), idesc_y, s > 0);
                mma_f16(tmem + tH, sdesc_sw128(b_base + s * 2048, 16384, 1024),
                        sdesc_sw128(wx_base + s * 2048, 16384, 1024), idesc_s, 1u);
            }
            mma_commit(mbar);
        }
        ok = __syncthreads_and(mbar_wait(mbar, phase, kWaitBudget));
        phase ^= 1u;
        if (!ok) break;
        tc_fence_after();

        // y_i = Y_i + exp(cum_i) Z_i + D x_i ; next block's fp16 state
        {
            const int i = tid, t = t0 + i;
            const float ei = expf(fminf(s_cum[i], 0.f));
            float *yrow = y + (((size_t)b * L + t) * H + h) * kP;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float yv[32], zv[32];
                tmem_ld32(lane_addr + tCB + half * 32, yv);
                tmem_ld32(lane_addr + tZ + half * 32, zv);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint4 xv = *reinterpret_cast<const uint4 *>(sX + sw128_off(i, half * 4 + q));
                    const float2 a0 = unpack_h2(xv.x), a1 = unpack_h2(xv.y), a2 = unpack_h2(xv.z),
                                 a3 = unpack_h2(xv.w);
                    const float xs[8] = {a0.x, a0.y, a1.x, a1.y, a2.x, a2.y, a3.x, a3.y};
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int p = q * 8 + e;
                        yv[p] = fmaf(Dh, xs[e], fmaf(ei, zv[p], yv[p]));
                    }
                }
                if (t < L) {
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        *reinterpret_cast<float4 *>(yrow + half * 32 + 4 * q) =
                            make_float4(yv[4 * q], yv[4 * q + 1], yv[4 * q + 2], yv[4 * q + 3]);
                }
            }
            const bool last = (k + 1 == kb1);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float v[32];
                tmem_ld32(lane_addr + tH + half * 32, v);
                if (!last) {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        *reinterpret_cast<uint4 *>(sHW + sw128_off(tid, half * 4 + q)) = pack8(v + 8 * q, range_ok);
                } else if (final_state && u == U - 1) {
                    float *dst = final_state + bh * kNP + (size_t)tid * kP + half * 32;
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        *reinterpret_cast<float4 *>(dst + 4 * q) =
                            make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    if (!ok && tid == 0) flag_status(ws.status, kStatusTimeout);
    if (!__syncthreads_and(range_ok) && tid == 0) flag_status(ws.status, kStatusRange);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

}  // namespace

bool tc_supported(const ScanDims &d, int bf16) {
    if (!bf16 || d.N != kN || d.P != kP) return false;
    if (d.Q != 64 && d.Q != 128 && d.Q != 256) return false;
    if (d.H > 65535 || d.b > 65535) return false;
    const TcPlan p = make_plan(d);
    return p.U <= 65535 && p.nblk <= 0x7fffffff && p.bpu <= 4096;
}

size_t tc_workspace_bytes(const ScanDims &d) { return ws_bytes(d, make_plan(d)); }

cudaError_t tc_scan(const ScanArgs &a, const ScanDims &d, void *wsp, cudaStream_t s) {
    const TcPlan p = make_plan(d);
    TcWs ws = carve(d, p, wsp);
    cudaError_t e;
    static bool attr_done = false;
    if (!attr_done) {
        if ((e = cudaFuncSetAttribute(unit_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)kUsSmem)) != cudaSuccess)
            return e;
        if ((e = cudaFuncSetAttribute(chunk_out_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)kCoSmem)) != cudaSuccess)
            return e;
        attr_done = true;
    }
    const __nv_bfloat16 *x = static_cast<const __nv_bfloat16 *>(a.x);
    const __nv_bfloat16 *Bm = static_cast<const __nv_bfloat16 *>(a.B);
    const __nv_bfloat16 *Cm = static_cast<const __nv_bfloat16 *>(a.C);
    {
        TraceScope tr(s, kTrTcDtPrep);
        dt_prep_kernel<<<dim3((unsigned)p.nblk, (unsigned)((d.H + 31) / 32), (unsigned)d.b), 256, 0, s>>>(
            a.dt_raw, a.dt_bias, a.A, ws, (int)d.L, (int)d.H, (int)p.nblk, a.dt_lo, a.dt_hi);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (p.U > 1) {
        {
            TraceScope tr(s, kTrTcUnitState);
            unit_state_kernel<<<dim3((unsigned)d.H, (unsigned)(p.U - 1), (unsigned)d.b), kTcThreads, kUsSmem, s>>>(
                x, Bm, ws, (int)d.L, (int)d.H, (int)d.G, (int)p.nblk, (int)p.U, (int)p.bpu);
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        {
            TraceScope tr(s, kTrTcStatePass);
            tc_state_pass_kernel<<<dim3(kNP / 256, (unsigned)d.H, (unsigned)d.b), 256, 0, s>>>(ws, a.init_state,
                                                                                               (int)d.H, (int)p.U);
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        TraceScope tr(s, kTrTcChunkOut);
        chunk_out_kernel<<<dim3((unsigned)d.H, (unsigned)p.U, (unsigned)d.b), kTcThreads, kCoSmem, s>>>(
            x, Bm, Cm, a.D, a.init_state, a.y, a.final_state, ws, (int)d.L, (int)d.H, (int)d.G, (int)p.nblk,
            (int)p.U, (int)p.bpu, p.U > 1 ? 1 : 0);
    }
    return cudaGetLastError();
}

}  // namespace ssd
