// Chunked SSD forward scan on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Scope: bf16 x/B/C, state_dim N = 128, head_dim P = 64, fp32 dt/A/D/state,
// fp32 y.  Every contraction runs as a kind::f16 MMA with fp16 operands and
// fp32 accumulation in TMEM.  bf16 -> fp16 is exact for inputs within fp16
// range; the decay-weighted operands are formed in fp16, whose 11-bit
// significand the 2e-2 bar needs (bf16's 8 bits are not enough).  Tiles
// arrive by TMA already in the 128-byte-swizzled operand layout.
//
// The sequence of every (batch, head) is cut into 128-token blocks (the MMA
// M extent) and the blocks into `units` of consecutive blocks.  Four
// launches; no CTA ever waits on another CTA:
//   prep        dt = clamp(softplus(dt_raw + dt_bias)), dA = dt*A, and the
//               inclusive cumsum `cum` of dA inside every 128-token block
//               (warp shuffles, fixed order), transposed to [b, H, L]; and an
//               fp16 copy of B and C (zero-padded to whole blocks), made once
//               per call because every head of a group reads them.
//   unit_state  per (head, unit u < U-1, batch): the state the unit leaves
//               when it starts from zero,
//                 S'_u = sum_{j in u} exp(sum_{r=j+1..end(u)} dA_r) dt_j B_j x_j^T,
//               as ONE accumulated MMA over the unit's tokens,
//               D[n,p] += B^T[n,j] (w x)[j,p]  (M=128 n, N=64 p, K=16 per
//               instruction), with a two-stage TMA pipeline.
//   state_pass  per (b, h, state element), serial over units:
//               H_in(0) = init (or 0),  H_in(u+1) = exp(ell_u) H_in(u) + S'_u.
//   chunk_out   per (head, unit, batch): from H_in(u), for each 128-token
//               block in order (state H fp32 in TMEM):
//                 Z   = C H                    (M=128 i, N=64 p, K=128 n)
//                 CB  = C B^T                  (M=128 i, N=128 j, K=128 n)
//                 W   = CB .* exp(cum_i - cum_j) dt_j on j <= i, 0 above
//                 Y   = W X                    (M=128 i, N=64 p, K=128 j)
//                 y_i = Y_i + exp(cum_i) Z_i + D x_i      (TMA store)
//                 H   = exp(cum_last) H + B^T (w X),  w_j = exp(cum_last - cum_j) dt_j
//               and the last unit writes final_state.
// This is the chunked form of the scan ("Mamba2" knowledge page: intra-chunk
// parallel in matrix-multiplication form, inter-chunk serial) with the
// intra-chunk quadratic term evaluated on 128-token blocks and the state
// carried on chip between them; it equals the token recurrence up to
// rounding for any chunk size (nnterp guide "Mamba-2", "The state after every
// token").  Every exponent is of min(., 0), taken after the causal select,
// so none can overflow.  Below the diagonal 32x32 sub-blocks the decay
// factors through the row group's first row m:
//   exp(cum_i - cum_j) = exp(cum_i - cum_m) * exp(cum_m - cum_j),  j <= m <= i,
// both factors <= 1, so W there costs two multiplies instead of an exp.
#include <stdint.h>

#include "ssd_common.cuh"
#include "ssd_internal.h"
#include "ssd_tc.cuh"
#include "ssd_tmap.h"
#include "ssd_trace.h"

namespace ssd {
namespace {

using namespace tc;

constexpr int kBlk = 128;                       // tokens per block
constexpr int kN = 128;                         // state_dim
constexpr int kP = 64;                          // head_dim
constexpr int kNP = kN * kP;
constexpr int kThreads = 256;                   // 8 warps; warps w and w+4 share TMEM lanes 32*(w%4)..
constexpr long long kWaitBudget = 1ll << 32;    // clock cycles before a wait gives up (~2 s)
constexpr float kF16Max = 65504.0f;
constexpr int kUnitTarget = 8 * 148;            // aim for ~8 units per SM across the grid
constexpr uint32_t kTileBytes = 16384;          // one 128-row x 128-byte swizzled tile

struct TcWs {
    unsigned *status;
    float *dt;       // [b, H, nblk*128]
    float *cum;      // [b, H, nblk*128]
    float *ell;      // [b, H, U]
    float *states;   // [b, H, U, N, P]
    __half *Bh;      // [b, nblk*128, G, N]  fp16 copy of B, zero rows past L
    __half *Ch;      // [b, nblk*128, G, N]  fp16 copy of C
};

struct TcPlan {
    int64_t nblk, U, bpu;
};

struct TcMaps {
    CUtensorMap x, B, C, y;
};

TcPlan make_plan(const ScanDims &d) {
    TcPlan p;
    p.nblk = (d.L + kBlk - 1) / kBlk;
    if (p.nblk < 1 || d.b < 1) {          // no tokens: nothing is launched
        p.nblk = 0;
        p.U = 1;
        p.bpu = 1;
        return p;
    }
    int64_t U = 1;
    while (d.b * d.H * U < kUnitTarget && U < p.nblk) U *= 2;
    if (U > p.nblk) U = p.nblk;
    p.bpu = (p.nblk + U - 1) / U;
    p.U = (p.nblk + p.bpu - 1) / p.bpu;
    return p;
}

size_t bc_bytes(const ScanDims &d, const TcPlan &p) {
    return (size_t)d.b * p.nblk * kBlk * d.G * kN * sizeof(__half);
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
    w.states = reinterpret_cast<float *>(c + off); off += align256((size_t)d.b * d.H * p.U * kNP * sizeof(float));
    w.Bh = reinterpret_cast<__half *>(c + off); off += align256(bc_bytes(d, p));
    w.Ch = reinterpret_cast<__half *>(c + off);
    return w;
}

size_t ws_bytes(const ScanDims &d, const TcPlan &p) {
    const size_t tok = (size_t)d.b * d.H * p.nblk * kBlk * sizeof(float);
    return kStatusBytes + 2 * align256(tok) + align256((size_t)d.b * d.H * p.U * sizeof(float)) +
           align256((size_t)d.b * d.H * p.U * kNP * sizeof(float)) + 2 * align256(bc_bytes(d, p));
}

// Tensor maps (4-D, innermost first) with 128-token boxes: x bf16 [b,L,H,P]
// and the fp16 B/C copies [b,Lp,G,N] in 64 x 1 x 128 x 1 boxes (one 16 KB
// swizzled tile); y fp32 [b,L,H,P] in 32 x 1 x 128 x 1 boxes.
bool make_maps(const ScanArgs &a, const ScanDims &d, const TcPlan &p, const TcWs &w, TcMaps *m) {
    const uint64_t b = d.b, L = d.L, H = d.H, G = d.G, Lp = p.nblk * kBlk;
    const uint32_t box_h[4] = {64, 1, kBlk, 1};
    const uint32_t box_y[4] = {32, 1, kBlk, 1};
    {
        const uint64_t dims[4] = {kP, H, L, b};
        const uint64_t st[3] = {kP * 2, H * kP * 2, L * H * kP * 2};
        if (!tmap_encode_4d(&m->x, a.x, kTmapBF16, dims, st, box_h)) return false;
    }
    {
        const uint64_t dims[4] = {kN, G, Lp, b};
        const uint64_t st[3] = {kN * 2, G * kN * 2, Lp * G * kN * 2};
        if (!tmap_encode_4d(&m->B, w.Bh, kTmapF16, dims, st, box_h)) return false;
        if (!tmap_encode_4d(&m->C, w.Ch, kTmapF16, dims, st, box_h)) return false;
    }
    {
        const uint64_t dims[4] = {kP, H, L, b};
        const uint64_t st[3] = {kP * 4, H * kP * 4, L * H * kP * 4};
        if (!tmap_encode_4d(&m->y, a.y, kTmapF32, dims, st, box_y)) return false;
    }
    return true;
}

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// 8 floats -> 8 fp16 (one 16-byte chunk); `amax` tracks the largest magnitude
__device__ __forceinline__ uint4 pack8(const float *f, float &amax) {
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
    return make_uint4(pack_h2(f[0], f[1]), pack_h2(f[2], f[3]), pack_h2(f[4], f[5]), pack_h2(f[6], f[7]));
}

__device__ __forceinline__ void bf16_chunk_to_f32(uint4 v, float *f) {
    f[0] = bf16lo(v.x); f[1] = bf16hi(v.x); f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
    f[4] = bf16lo(v.z); f[5] = bf16hi(v.z); f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
}

__device__ __forceinline__ void f16_chunk_to_f32(uint4 v, float *f) {
    const float2 a0 = unpack_h2(v.x), a1 = unpack_h2(v.y), a2 = unpack_h2(v.z), a3 = unpack_h2(v.w);
    f[0] = a0.x; f[1] = a0.y; f[2] = a1.x; f[3] = a1.y; f[4] = a2.x; f[5] = a2.y; f[6] = a3.x; f[7] = a3.y;
}

// ---------------------------------------------------------------------------
// prep: grid (nblk, ceil(H/32) + G, b), 256 threads.  y-slices below
// ceil(H/32) do dt/cum for 32 heads; the rest convert B and C of one group.
__global__ void __launch_bounds__(256)
prep_kernel(const float *__restrict__ dt_raw, const float *__restrict__ dt_bias, const float *__restrict__ A,
            const __nv_bfloat16 *__restrict__ Bm, const __nv_bfloat16 *__restrict__ Cm, TcWs ws, int L, int H,
            int G, int nblk, float lo, float hi) {
    __shared__ float s_dt[kBlk][33];
    __shared__ float s_da[kBlk][33];
    const int blk = blockIdx.x, b = blockIdx.z;
    const int nhy = (H + 31) / 32;
    if ((int)blockIdx.y >= nhy) {
        const int g = blockIdx.y - nhy;
        const int t0 = blk * kBlk;
        const size_t Lp = (size_t)nblk * kBlk;
        float amax = 0.f;
#pragma unroll 4
        for (int c = threadIdx.x; c < 2 * kBlk * 16; c += 256) {
            const int which = c >> 11, r = (c >> 4) & (kBlk - 1), kk = c & 15;
            const int t = t0 + r;
            const __nv_bfloat16 *src = which ? Cm : Bm;
            __half *dst = which ? ws.Ch : ws.Bh;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (t < L) v = __ldg(reinterpret_cast<const uint4 *>(src + (((size_t)b * L + t) * G + g) * kN + kk * 8));
            float f[8];
            bf16_chunk_to_f32(v, f);
            *reinterpret_cast<uint4 *>(dst + (((size_t)b * Lp + t) * G + g) * kN + kk * 8) = pack8(f, amax);
        }
        if (!(amax <= kF16Max)) flag_status(ws.status, kStatusRange);
        return;
    }
    const int h0 = blockIdx.y * 32;
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
// unit_state: grid (H, U-1, b), 256 threads, two TMA stages of (B fp16, X bf16).
// Units 0..U-2 never hold the sequence's ragged tail (it is in the last
// unit), so every block here is a full 128 tokens.
constexpr uint32_t kUsStage = 3 * kTileBytes;                 // B (2 tiles) + X (1 tile)
constexpr size_t kUsSmem = 1024 + 2 * kUsStage + 2 * kBlk * 4 + 64;

__global__ void __launch_bounds__(kThreads, 2)
unit_state_kernel(const __grid_constant__ TcMaps maps, TcWs ws, int H, int G, int nblk, int U, int bpu) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    float *s_w = reinterpret_cast<float *>(sm + 2 * kUsStage);   // [2][128]
    uint64_t *bar = reinterpret_cast<uint64_t *>(s_w + 2 * kBlk); // tma[2], mma[2]
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar + 4);

    const int h = blockIdx.x, u = blockIdx.y, b = blockIdx.z;
    const int g = h / (H / G);
    const int tid = threadIdx.x, warp = tid >> 5;
    const size_t bh = (size_t)b * H + h;
    const int kb0 = u * bpu, kb1 = min(nblk, kb0 + bpu);
    const int nk = kb1 - kb0;
    const float *cum = ws.cum + bh * (size_t)nblk * kBlk;
    const float *dtv = ws.dt + bh * (size_t)nblk * kBlk;

    if (warp == 0) {
        tmem_alloc(tslot, 64);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(bar + i, 1);
        fence_mbar_init();
        for (int i = 0; i < 2 && i < nk; ++i) {
            uint8_t *st = sm + i * kUsStage;
            const int t0 = (kb0 + i) * kBlk;
            mbar_arrive_expect_tx(bar + i, kUsStage);
            tma_load_4d(st, &maps.B, bar + i, 0, g, t0, b);
            tma_load_4d(st + kTileBytes, &maps.B, bar + i, 64, g, t0, b);
            tma_load_4d(st + 2 * kTileBytes, &maps.x, bar + i, 0, h, t0, b);
        }
    }
    // suffix: the unit's log decay after the current block (sum of later block totals)
    float suffix = 0.f;
    for (int k = kb0 + 1; k < kb1; ++k) suffix += cum[(size_t)k * kBlk + kBlk - 1];
    if (tid == 0) ws.ell[bh * U + u] = suffix + cum[(size_t)kb0 * kBlk + kBlk - 1];
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;

    bool ok = true;
    float amax = 0.f;
    uint32_t tma_par = 0, mma_par = 0;              // per-stage phase bits
    const uint32_t idesc = idesc_f16(128, 64, 1, 1);
    for (int k = kb0; k < kb1; ++k) {
        const int i = k - kb0, s = i & 1;
        uint8_t *st = sm + s * kUsStage;
        float *w = s_w + s * kBlk;
        if (tid < kBlk) {
            const float e = cum[(size_t)k * kBlk + kBlk - 1] - cum[(size_t)k * kBlk + tid] + suffix;
            w[tid] = expf(fminf(e, 0.f)) * dtv[(size_t)k * kBlk + tid];
        }
        if (k + 1 < kb1) suffix -= cum[(size_t)(k + 1) * kBlk + kBlk - 1];
        ok = mbar_wait(bar + s, (tma_par >> s) & 1u, kWaitBudget);
        tma_par ^= 1u << s;
        __syncthreads();                            // w[] visible
        // X (bf16) -> w.X (fp16) in place; the row of a chunk is offset / 128
        uint8_t *sx = st + 2 * kTileBytes;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int c = tid + r * kThreads;
            uint4 *p = reinterpret_cast<uint4 *>(sx + c * 16);
            float f[8];
            bf16_chunk_to_f32(*p, f);
            const float wr = w[c >> 3];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] *= wr;
            *p = pack8(f, amax);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        ok = __syncthreads_and(ok);
        tc_fence_after();
        if (!ok) break;
        if (tid == 0) {
            const uint32_t b_base = smem_u32(st), x_base = smem_u32(sx);
#pragma unroll
            for (int q = 0; q < 8; ++q)
                mma_f16(tmem, sdesc_sw128(b_base + q * 2048, kTileBytes, 1024),
                        sdesc_sw128(x_base + q * 2048, kTileBytes, 1024), idesc, (i > 0 || q > 0) ? 1u : 0u);
            mma_commit(bar + 2 + s);
            // refill this stage with block k+2 once these MMAs have read it
            if (k + 2 < kb1) {
                const bool done = mbar_wait(bar + 2 + s, (mma_par >> s) & 1u, kWaitBudget);
                mma_par ^= 1u << s;
                if (done) {
                    const int t0 = (k + 2) * kBlk;
                    mbar_arrive_expect_tx(bar + s, kUsStage);
                    tma_load_4d(st, &maps.B, bar + s, 0, g, t0, b);
                    tma_load_4d(st + kTileBytes, &maps.B, bar + s, 64, g, t0, b);
                    tma_load_4d(st + 2 * kTileBytes, &maps.x, bar + s, 0, h, t0, b);
                } else {
                    flag_status(ws.status, kStatusTimeout);
                }
            }
        }
    }
    // wait for the last block's MMAs (the stage it used still has that commit pending)
    if (ok && tid == 0 && nk > 0) {
        const int s = (nk - 1) & 1;
        ok = mbar_wait(bar + 2 + s, (mma_par >> s) & 1u, kWaitBudget);
    }
    ok = __syncthreads_and(ok);
    tc_fence_after();
    if (!ok) {
        if (tid == 0) flag_status(ws.status, kStatusTimeout);
    } else {
        // 8 warps: lanes 32*(warp%4).., columns 32*(warp/4)..
        const int n = 32 * (warp & 3) + (tid & 31), ch = warp >> 2;
        float v[32];
        tmem_ld32(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + ch * 32, v);
        float *dst = ws.states + (bh * U + u) * (size_t)kNP + (size_t)n * kP + ch * 32;
#pragma unroll
        for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4 *>(dst + 4 * q) = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
    if (!__syncthreads_and(amax <= kF16Max) && tid == 0) flag_status(ws.status, kStatusRange);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 64);
}

// ---------------------------------------------------------------------------
// state_pass: grid (N*P/4/256, H, b), 256 threads; each thread owns one
// float4 of the state and issues its loads for a batch of units before the
// serial combine.
constexpr int kSpBatch = 8;

__global__ void __launch_bounds__(256)
tc_state_pass_kernel(TcWs ws, const float *__restrict__ init, int H, int U) {
    const int e4 = blockIdx.x * 256 + threadIdx.x;
    const size_t bh = (size_t)blockIdx.z * H + blockIdx.y;
    float4 hs = init ? reinterpret_cast<const float4 *>(init + bh * kNP)[e4] : make_float4(0.f, 0.f, 0.f, 0.f);
    float4 *S = reinterpret_cast<float4 *>(ws.states + bh * (size_t)U * kNP) + e4;
    const float *ell = ws.ell + bh * U;
    for (int u0 = 0; u0 + 1 < U; u0 += kSpBatch) {
        const int n = min(kSpBatch, U - 1 - u0);
        float4 s[kSpBatch];
        float a[kSpBatch];
#pragma unroll
        for (int i = 0; i < kSpBatch; ++i) {
            if (i < n) {
                s[i] = S[(size_t)(u0 + i) * (kNP / 4)];
                a[i] = expf(fminf(ell[u0 + i], 0.f));
            }
        }
#pragma unroll
        for (int i = 0; i < kSpBatch; ++i) {
            if (i < n) {
                S[(size_t)(u0 + i) * (kNP / 4)] = hs;   // state entering unit u0+i
                hs.x = fmaf(a[i], hs.x, s[i].x);
                hs.y = fmaf(a[i], hs.y, s[i].y);
                hs.z = fmaf(a[i], hs.z, s[i].z);
                hs.w = fmaf(a[i], hs.w, s[i].w);
            }
        }
    }
    S[(size_t)(U - 1) * (kNP / 4)] = hs;
}

// ---------------------------------------------------------------------------
// chunk_out: grid (H, U, b), 256 threads, 2 CTAs per SM.
constexpr size_t kCoSmem = 1024 + 6 * kTileBytes + (3 * kBlk + 3 * kBlk) * 4 + 64;

__global__ void __launch_bounds__(kThreads, 2)
chunk_out_kernel(const __grid_constant__ TcMaps maps, const float *__restrict__ D,
                 const float *__restrict__ init, float *__restrict__ final_state, TcWs ws, int L, int H, int G,
                 int nblk, int U, int bpu, int states_from_ws) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    uint8_t *sCW = sm;                              // C tile -> W tile -> y staging (2 tiles)
    uint8_t *sB = sm + 2 * kTileBytes;              // B tile (2 tiles)
    uint8_t *sX = sm + 4 * kTileBytes;              // X tile
    uint8_t *sHW = sm + 5 * kTileBytes;             // fp16 state [n][p], then w.X [j][p]
    float *s_dt = reinterpret_cast<float *>(sm + 6 * kTileBytes);
    float *s_cum = s_dt + kBlk;
    float *s_w = s_cum + kBlk;
    float *s_v = s_w + kBlk;                        // [3][128] pivot factors for row groups 1..3
    uint64_t *bar = reinterpret_cast<uint64_t *>(s_v + 3 * kBlk);  // [0] TMA, [1] MMA
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar + 2);

    const int h = blockIdx.x, u = blockIdx.y, b = blockIdx.z;
    const int g = h / (H / G);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int w4 = warp & 3;                        // row group: rows 32*w4 .. 32*w4+31
    const int row = 32 * w4 + lane;                 // TMEM lane / tile row of this thread
    const int ch = warp >> 2;                       // which 32-column half it handles
    const size_t bh = (size_t)b * H + h;
    const int kb0 = u * bpu, kb1 = min(nblk, kb0 + bpu);
    const float *cum = ws.cum + bh * (size_t)nblk * kBlk;
    const float *dtv = ws.dt + bh * (size_t)nblk * kBlk;

    if (warp == 0) {
        tmem_alloc(tslot, 256);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init(bar + 1, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * w4) << 16);
    const uint32_t tH = 0, tZ = 64, tCB = 128;   // TMEM columns: state, C.H, C.B^T then Y
    float amax = 0.f;

    // state entering the unit -> TMEM (fp32) and sHW (fp16): row n = `row`, columns 32*ch..
    {
        const float *src = states_from_ws ? ws.states + (bh * U + u) * (size_t)kNP
                                          : (init ? init + bh * kNP : nullptr);
        float v[32];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float4 f = src ? *reinterpret_cast<const float4 *>(src + (size_t)row * kP + ch * 32 + 4 * q)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
            v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
        }
        tmem_st32(lane_addr + tH + ch * 32, v);
#pragma unroll
        for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4 *>(sHW + sw128_off(row, ch * 4 + q)) = pack8(v + 8 * q, amax);
    }

    bool ok = true;
    uint32_t tma_par = 0, mma_par = 0;
    const uint32_t idesc_z = idesc_f16(128, 64, 0, 1);    // A=C K-major, B=H MN-major
    const uint32_t idesc_cb = idesc_f16(128, 128, 0, 0);  // A=C K-major, B=B K-major
    const uint32_t idesc_y = idesc_f16(128, 64, 0, 1);    // A=W K-major, B=X MN-major
    const uint32_t idesc_s = idesc_f16(128, 64, 1, 1);    // A=B^T MN-major, B=wX MN-major
    const float Dh = D[h];

    for (int k = kb0; k < kb1; ++k) {
        const int t0 = k * kBlk;
        if (tid == 0) {
            tma_store_wait_read();                 // the previous y store has left sCW
            mbar_arrive_expect_tx(bar, 5 * kTileBytes);
            tma_load_4d(sCW, &maps.C, bar, 0, g, t0, b);
            tma_load_4d(sCW + kTileBytes, &maps.C, bar, 64, g, t0, b);
            tma_load_4d(sB, &maps.B, bar, 0, g, t0, b);
            tma_load_4d(sB + kTileBytes, &maps.B, bar, 64, g, t0, b);
            tma_load_4d(sX, &maps.x, bar, 0, h, t0, b);
        }
        if (tid < kBlk) s_dt[tid] = dtv[(size_t)t0 + tid];
        else s_cum[tid - kBlk] = cum[(size_t)t0 + tid - kBlk];
        __syncthreads();                           // s_dt, s_cum visible
        // decay to the block's last real token (padding carries dA = 0 but its
        // cumsum may round differently)
        const float clast = s_cum[min(kBlk - 1, L - 1 - t0)];
        if (tid < kBlk) s_w[tid] = expf(fminf(clast - s_cum[tid], 0.f)) * s_dt[tid];
        for (int idx = tid; idx < 3 * kBlk; idx += kThreads) {   // pivot factors, row groups 1..3
            const int gm = idx >> 7, j = idx & (kBlk - 1);
            const int m = 32 * (gm + 1) - 1;
            if (j <= m) s_v[idx] = expf(fminf(s_cum[m] - s_cum[j], 0.f)) * s_dt[j];
        }
        ok = mbar_wait(bar, tma_par, kWaitBudget);
        tma_par ^= 1u;
        // X: bf16 -> fp16 in place (C and B arrive as fp16)
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            uint4 *p = reinterpret_cast<uint4 *>(sX + (tid + r * kThreads) * 16);
            float f[8];
            bf16_chunk_to_f32(*p, f);
            *p = pack8(f, amax);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        ok = __syncthreads_and(ok);
        tc_fence_after();
        if (!ok) break;

        if (tid == 0) {
            const uint32_t c_base = smem_u32(sCW), b_base = smem_u32(sB), h_base = smem_u32(sHW);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint64_t ad = sdesc_sw128(c_base + (q >> 2) * kTileBytes + (q & 3) * 32, 16, 1024);
                mma_f16(tmem + tZ, ad, sdesc_sw128(h_base + q * 2048, kTileBytes, 1024), idesc_z, q > 0);
                mma_f16(tmem + tCB, ad, sdesc_sw128(b_base + (q >> 2) * kTileBytes + (q & 3) * 32, 16, 1024),
                        idesc_cb, q > 0);
            }
            mma_commit(bar + 1);
        }
        ok = __syncthreads_and(mbar_wait(bar + 1, mma_par, kWaitBudget));
        mma_par ^= 1u;
        if (!ok) break;
        tc_fence_after();

        // W (row `row`, columns 64*ch..64*ch+63) into sCW; w.X into sHW; the
        // state scaled by the block decay
        {
            const float ci = s_cum[row];
            const float ui = w4 > 0 ? expf(fminf(ci - s_cum[32 * w4 - 1], 0.f)) : 0.f;
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int c32 = 2 * ch + cc;
                uint4 out[4];
                if (c32 < w4) {                          // below the diagonal: factored decay
                    float v[32];
                    tmem_ld32(lane_addr + tCB + c32 * 32, v);
                    const float4 *vf = reinterpret_cast<const float4 *>(s_v + (w4 - 1) * kBlk + c32 * 32);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 f = vf[q];
                        v[4 * q] *= f.x * ui;
                        v[4 * q + 1] *= f.y * ui;
                        v[4 * q + 2] *= f.z * ui;
                        v[4 * q + 3] *= f.w * ui;
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q) out[q] = pack8(v + 8 * q, amax);
                } else if (c32 == w4) {                  // diagonal 32x32: masked, exact exponent
                    float v[32];
                    tmem_ld32(lane_addr + tCB + c32 * 32, v);
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        const int j = c32 * 32 + jj;
                        v[jj] = (jj <= lane) ? v[jj] * expf(fminf(ci - s_cum[j], 0.f)) * s_dt[j] : 0.f;
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q) out[q] = pack8(v + 8 * q, amax);
                } else {
#pragma unroll
                    for (int q = 0; q < 4; ++q) out[q] = make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<uint4 *>(sCW + ch * kTileBytes + sw128_off(row, cc * 4 + q)) = out[q];
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) {                // 1024 chunks of w.X
                const int c = tid + r * kThreads;
                const int j = c >> 3, q = c & 7;
                float f[8];
                f16_chunk_to_f32(*reinterpret_cast<const uint4 *>(sX + sw128_off(j, q)), f);
                const float wj = s_w[j];
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] *= wj;
                *reinterpret_cast<uint4 *>(sHW + sw128_off(j, q)) = pack8(f, amax);
            }
            const float decay = expf(fminf(clast, 0.f));
            float v[32];
            tmem_ld32(lane_addr + tH + ch * 32, v);
#pragma unroll
            for (int q = 0; q < 32; ++q) v[q] *= decay;
            tmem_st32(lane_addr + tH + ch * 32, v);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        if (tid == 0) {
            const uint32_t w_base = smem_u32(sCW), x_base = smem_u32(sX), b_base = smem_u32(sB),
                           wx_base = smem_u32(sHW);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                mma_f16(tmem + tCB, sdesc_sw128(w_base + (q >> 2) * kTileBytes + (q & 3) * 32, 16, 1024),
                        sdesc_sw128(x_base + q * 2048, kTileBytes, 1024), idesc_y, q > 0);
                mma_f16(tmem + tH, sdesc_sw128(b_base + q * 2048, kTileBytes, 1024),
                        sdesc_sw128(wx_base + q * 2048, kTileBytes, 1024), idesc_s, 1u);
            }
            mma_commit(bar + 1);
        }
        ok = __syncthreads_and(mbar_wait(bar + 1, mma_par, kWaitBudget));
        mma_par ^= 1u;
        if (!ok) break;
        tc_fence_after();

        // y_i = Y_i + exp(cum_i) Z_i + D x_i -> staging (sCW, two 32-column
        // fp32 tiles) -> TMA store; the next block's fp16 state into sHW
        {
            const float ei = expf(fminf(s_cum[row], 0.f));
            float yv[32], zv[32];
            tmem_ld32(lane_addr + tCB + ch * 32, yv);
            tmem_ld32(lane_addr + tZ + ch * 32, zv);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float xs[8];
                f16_chunk_to_f32(*reinterpret_cast<const uint4 *>(sX + sw128_off(row, ch * 4 + q)), xs);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int p = q * 8 + e;
                    yv[p] = fmaf(Dh, xs[e], fmaf(ei, zv[p], yv[p]));
                }
            }
            uint8_t *stg = sCW + ch * kTileBytes;
#pragma unroll
            for (int q = 0; q < 8; ++q)
                *reinterpret_cast<float4 *>(stg + sw128_off(row, q)) =
                    make_float4(yv[4 * q], yv[4 * q + 1], yv[4 * q + 2], yv[4 * q + 3]);
            const bool last = (k + 1 == kb1);
            float v[32];
            tmem_ld32(lane_addr + tH + ch * 32, v);
            if (!last) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<uint4 *>(sHW + sw128_off(row, ch * 4 + q)) = pack8(v + 8 * q, amax);
            } else if (final_state && u == U - 1) {
                float *dst = final_state + bh * kNP + (size_t)row * kP + ch * 32;
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    *reinterpret_cast<float4 *>(dst + 4 * q) = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
            tma_store_4d(&maps.y, sCW, 0, h, t0, b);
            tma_store_4d(&maps.y, sCW + kTileBytes, 32, h, t0, b);
            tma_store_commit();
        }
    }
    if (tid == 0) tma_store_wait_all();
    if (!ok && tid == 0) flag_status(ws.status, kStatusTimeout);
    if (!__syncthreads_and(amax <= kF16Max) && tid == 0) flag_status(ws.status, kStatusRange);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

}  // namespace

bool tc_supported(const ScanDims &d, int bf16) {
    if (!bf16 || d.N != kN || d.P != kP) return false;
    if (d.Q != 64 && d.Q != 128 && d.Q != 256) return false;
    if (d.H > 65535 || d.b > 65535 || d.L > 0x7fffffffll - kBlk) return false;
    const TcPlan p = make_plan(d);
    return p.U <= 65535 && (d.H + 31) / 32 + d.G <= 65535;
}

size_t tc_workspace_bytes(const ScanDims &d) { return ws_bytes(d, make_plan(d)); }

cudaError_t tc_scan(const ScanArgs &a, const ScanDims &d, void *wsp, cudaStream_t s) {
    const TcPlan p = make_plan(d);
    if (p.nblk == 0) return cudaSuccess;
    TcWs ws = carve(d, p, wsp);
    TcMaps maps;
    if (!make_maps(a, d, p, ws, &maps)) return cudaErrorInvalidValue;
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
    {
        TraceScope tr(s, kTrTcDtPrep);
        const unsigned ny = (unsigned)((d.H + 31) / 32 + d.G);
        prep_kernel<<<dim3((unsigned)p.nblk, ny, (unsigned)d.b), 256, 0, s>>>(
            a.dt_raw, a.dt_bias, a.A, static_cast<const __nv_bfloat16 *>(a.B), static_cast<const __nv_bfloat16 *>(a.C),
            ws, (int)d.L, (int)d.H, (int)d.G, (int)p.nblk, a.dt_lo, a.dt_hi);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (p.U > 1) {
        {
            TraceScope tr(s, kTrTcUnitState);
            unit_state_kernel<<<dim3((unsigned)d.H, (unsigned)(p.U - 1), (unsigned)d.b), kThreads, kUsSmem, s>>>(
                maps, ws, (int)d.H, (int)d.G, (int)p.nblk, (int)p.U, (int)p.bpu);
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        {
            TraceScope tr(s, kTrTcStatePass);
            tc_state_pass_kernel<<<dim3(kNP / 4 / 256, (unsigned)d.H, (unsigned)d.b), 256, 0, s>>>(
                ws, a.init_state, (int)d.H, (int)p.U);
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        TraceScope tr(s, kTrTcChunkOut);
        chunk_out_kernel<<<dim3((unsigned)d.H, (unsigned)p.U, (unsigned)d.b), kThreads, kCoSmem, s>>>(
            maps, a.D, a.init_state, a.final_state, ws, (int)d.L, (int)d.H, (int)d.G, (int)p.nblk, (int)p.U,
            (int)p.bpu, p.U > 1 ? 1 : 0);
    }
    return cudaGetLastError();
}

}  // namespace ssd
