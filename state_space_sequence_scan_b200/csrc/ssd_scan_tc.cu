// Chunked SSD forward scan on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Scope: bf16 x/B/C, state_dim N = 128, head_dim P = 64, fp32 dt/A/D/state,
// fp32 y.  Every contraction runs as a kind::f16 MMA with fp32 accumulation
// in TMEM.  C.B^T, the state terms B^T (w x) and C H take fp16 operands
// (bf16 -> fp16 is exact for inputs within fp16 range; the decay-weighted
// w x and the carried state need fp16's 11-bit significand, bf16's 8 bits
// are not enough).  W.X takes the x tile as the TMA delivers it (bf16) and
// the decay-weighted W as a bf16 high/low pair (two MMAs, about 16
// significant bits): y is heavy-tailed and its largest elements are single
// W.X terms, whose fp16 rounding alone exceeds the 2e-2 bar.  Tiles arrive by
// TMA already in the 128-byte-swizzled operand layout.
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

#include <atomic>

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
constexpr long long kWaitBudget = 1ll << 32;    // clock cycles before a wait gives up (~2 s)
constexpr long long kTestWaitBudget = 1ll << 21;  // the same under the test fault (~1 ms)
constexpr float kF16Max = 65504.0f;
constexpr int kSMs = 148;                       // B200 streaming multiprocessors
// Relative cost of the unit decomposition, in chunk_out block-times (one
// 128-token block of one CTA; chunk_out runs one CTA per SM): unit_state runs
// two CTAs per SM at about this fraction of a chunk_out block, and the
// state pass costs about this many block-times.
// A CTA also pays about kCtaStartRel block-times to start its pipeline.
constexpr double kUnitStateRel = 0.35;
constexpr double kStatePassRel = 5.0;
constexpr double kCtaStartRel = 2.0;
constexpr int64_t kMaxUnits = 4096;
constexpr int kMaxAttrDevices = 64;
constexpr uint32_t kTileBytes = 16384;          // one 128-row x 128-byte swizzled tile
constexpr int kConvK = 4;                        // conv width of the combined arrangement
constexpr int kXRaw = kBlk + kConvK - 1;         // input rows of a block's conv (3 before it)
constexpr uint32_t kXRawBytes = kXRaw * 128;     // 16768: the raw X tile, 128 bytes a row

struct TcWs {
    unsigned *status;
    float *dt;       // [b, H, nblk*128]
    float *cum;      // [b, H, nblk*128]
    float *ell;      // [b, H, U]
    float *states;   // [b, H, U, N, P]
    __half *Bh;      // [b, nblk*128, G, N]  fp16 copy of B, zero rows past L
    __half *Ch;      // [b, nblk*128, G, N]  fp16 copy of C
    int *rs;         // [b, nblk*128] packed rows: the last document start at or before
                     // each token within its 128-token block (block offset), -1 if none
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
    // Split every (batch, head) chain into U units of bpu blocks so that the
    // grid's waves times the blocks per unit, plus the passes that carry the
    // state between units, is smallest (ties: fewer units).  A function of
    // the shape alone, so the workspace size is known before the launch.
    const int64_t chains = d.b * d.H;
    double best = 0.0;
    p.U = 1;
    p.bpu = p.nblk;
    for (int64_t U = 1; U <= p.nblk && U <= kMaxUnits; ++U) {
        const int64_t bpu = (p.nblk + U - 1) / U;
        if ((p.nblk + bpu - 1) / bpu != U) continue;         // same split as a smaller U
        double cost = (double)((chains * U + kSMs - 1) / kSMs) * ((double)bpu + kCtaStartRel);
        if (U > 1)
            cost += (double)((chains * (U - 1) + 2 * kSMs - 1) / (2 * kSMs)) * ((double)bpu + kCtaStartRel) *
                        kUnitStateRel +
                    kStatePassRel;
        if (U == 1 || cost < best) {
            best = cost;
            p.U = U;
            p.bpu = bpu;
        }
    }
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
    w.Ch = reinterpret_cast<__half *>(c + off); off += align256(bc_bytes(d, p));
    w.rs = reinterpret_cast<int *>(c + off);
    return w;
}

size_t ws_bytes(const ScanDims &d, const TcPlan &p) {
    const size_t tok = (size_t)d.b * d.H * p.nblk * kBlk * sizeof(float);
    return kStatusBytes + 2 * align256(tok) + align256((size_t)d.b * d.H * p.U * sizeof(float)) +
           align256((size_t)d.b * d.H * p.U * kNP * sizeof(float)) + 2 * align256(bc_bytes(d, p)) +
           align256((size_t)d.b * p.nblk * kBlk * sizeof(int));
}

// Tensor maps (4-D, innermost first) with 128-token boxes: x bf16 [b,L,H,P]
// and the fp16 B/C copies [b,Lp,G,N] in 64 x 1 x 128 x 1 boxes (one 16 KB
// swizzled tile); y fp32 [b,L,H,P] in 32 x 1 x 128 x 1 boxes.
bool make_maps(const ScanArgs &a, const ScanDims &d, const TcPlan &p, const TcWs &w, TcMaps *m) {
    const uint64_t b = d.b, L = d.L, H = d.H, G = d.G, Lp = p.nblk * kBlk;
    const uint32_t box_h[4] = {64, 1, kBlk, 1};
    const uint32_t box_y[4] = {32, 1, kBlk, 1};
    if (a.conv_w) {
        // combined arrangement: the x channels of xbc [b, L, Cd], a block's 128
        // tokens and the conv's 3 rows before them
        const uint64_t Cd = a.Cd;
        const uint32_t box_x[4] = {64, 1, (uint32_t)kXRaw, 1};
        const uint64_t dims[4] = {kP, H, L, b};
        const uint64_t st[3] = {kP * 2, Cd * 2, L * Cd * 2};
        if (!tmap_encode_4d(&m->x, a.x, kTmapBF16, dims, st, box_x)) return false;
    } else {
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

// 8 floats -> 8 fp16 (one 16-byte chunk).  `hmax` tracks the largest packed
// magnitude as a half2 (an out-of-range value rounds to inf and stays there).
__device__ __forceinline__ uint4 pack8(const float *f, __half2 &hmax) {
    const uint4 o = make_uint4(pack_h2(f[0], f[1]), pack_h2(f[2], f[3]), pack_h2(f[4], f[5]), pack_h2(f[6], f[7]));
    const uint32_t w[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) hmax = __hmax2(hmax, __habs2(*reinterpret_cast<const __half2 *>(&w[i])));
    return o;
}

__device__ __forceinline__ bool in_f16_range(__half2 hmax) {
    const float2 m = __half22float2(hmax);
    return m.x <= kF16Max && m.y <= kF16Max;
}

__device__ __forceinline__ void bf16_chunk_to_f32(uint4 v, float *f) {
    f[0] = bf16lo(v.x); f[1] = bf16hi(v.x); f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
    f[4] = bf16lo(v.z); f[5] = bf16hi(v.z); f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
}

// ---- the combined arrangement: conv1d + SiLU inside the scan's kernels
// A value the split conv would store as bf16, back in fp32.
__device__ __forceinline__ float bf16_round(float v) { return __bfloat162float(__float2bfloat16_rn(v)); }

// Channels 4q..4q+3 of the bf16 row r of an X-type tile (128-byte-swizzled,
// 64 channels a row): the 8-byte half (q & 1) of chunk q >> 1.
__device__ __forceinline__ uint32_t xq_off(int r, int q) {
    return (uint32_t)r * 128u + ((((uint32_t)q >> 1) ^ ((uint32_t)r & 7u)) << 4) + ((uint32_t)q & 1u) * 8u;
}


// In place on a 64-channel X tile that holds kXRaw raw input rows (row r' =
// token t0 - 3 + r'): row r becomes conv1d + SiLU of token t0 + r, rounded to
// bf16 (as the split conv stores x).  kScaled false (chunk_out): stored as
// bf16; rows at or past L become 0 (as the TMA fills x there).  kScaled true
// (unit_state): times w[r] in fp32, stored as fp16 (the w.X operand), the
// largest magnitude tracked in `amax`.  256 threads take 4 channels x 8 rows
// each: all read their 11 input rows, meet at named barrier 1, then write.
// `wb` holds the 64 channels' weights (float4 each) then their biases.  Every
// thread of the barrier calls this; `ok` false skips the reads and writes.
template <bool kScaled>
__device__ __forceinline__ void conv_x_tile(uint8_t *sx, const float4 *wb, int tid, int t0, int L, bool ok,
                                            const float *w_row = nullptr, __half2 *amax = nullptr) {
    const int q = tid & 15, rg = tid >> 4;
    uint2 rw[8 + kConvK - 1];
    if (ok) {
#pragma unroll
        for (int j = 0; j < 8 + kConvK - 1; ++j) rw[j] = *reinterpret_cast<const uint2 *>(sx + xq_off(8 * rg + j, q));
    }
    named_bar_sync(256);
    if (!ok) return;
    float w[4][kConvK], bias[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float4 v = wb[4 * q + e];
        w[e][0] = v.x; w[e][1] = v.y; w[e][2] = v.z; w[e][3] = v.w;
    }
    {
        const float4 v = wb[64 + q];
        bias[0] = v.x; bias[1] = v.y; bias[2] = v.z; bias[3] = v.w;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int r = 8 * rg + j;
        float o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float xw[kConvK];
#pragma unroll
            for (int k = 0; k < kConvK; ++k) {
                const uint32_t u = (e < 2) ? rw[j + k].x : rw[j + k].y;
                xw[k] = (e & 1) ? bf16hi(u) : bf16lo(u);
            }
            o[e] = conv_silu<kConvK>(w[e], xw, bias[e]);
        }
        uint2 out;
        if (kScaled) {
            const float wr = w_row[r];
            const uint32_t h0 = pack_h2(bf16_round(o[0]) * wr, bf16_round(o[1]) * wr);
            const uint32_t h1 = pack_h2(bf16_round(o[2]) * wr, bf16_round(o[3]) * wr);
            *amax = __hmax2(*amax, __habs2(*reinterpret_cast<const __half2 *>(&h0)));
            *amax = __hmax2(*amax, __habs2(*reinterpret_cast<const __half2 *>(&h1)));
            out = make_uint2(h0, h1);
        } else {
            const bool live = t0 + r < L;
            const __nv_bfloat162 a = __floats2bfloat162_rn(live ? o[0] : 0.f, live ? o[1] : 0.f);
            const __nv_bfloat162 c = __floats2bfloat162_rn(live ? o[2] : 0.f, live ? o[3] : 0.f);
            out = make_uint2(*reinterpret_cast<const uint32_t *>(&a), *reinterpret_cast<const uint32_t *>(&c));
        }
        *reinterpret_cast<uint2 *>(sx + xq_off(r, q)) = out;
    }
}

// The 64 x channels of head h: weights [64][4] then biases [64] into `wb`
// (a float4 each for the weights, 16 float4s of biases)
__device__ __forceinline__ void conv_load_weights(float4 *wb, const float *cw, const float *cb, int h, int tid,
                                                  int nthreads) {
    for (int i = tid; i < 64 + 16; i += nthreads)
        wb[i] = i < 64 ? *reinterpret_cast<const float4 *>(cw + ((size_t)h * kP + i) * kConvK)
                       : *reinterpret_cast<const float4 *>(cb + (size_t)h * kP + 4 * (i - 64));
}

// ---------------------------------------------------------------------------
// prep: grid (nblk, ceil(H/8) + 4 G, b), 256 threads.  y-slices below
// ceil(H/8) do dt/cum for 8 heads of one 128-token block; the rest convert a
// 32-row quarter of the block's B and C of one group.  Small slices keep many
// CTAs in flight: every thread issues its few loads before any arithmetic.
constexpr int kPrepHeads = 8;

template <bool kConv>
__global__ void __launch_bounds__(256)
prep_kernel(const float *__restrict__ dt_raw, const float *__restrict__ dt_bias, const float *__restrict__ A,
            const __nv_bfloat16 *__restrict__ Bm, const __nv_bfloat16 *__restrict__ Cm,
            const int32_t *__restrict__ seq_idx, TcWs ws, int L, int H, int G, int nblk, float lo, float hi,
            const float *__restrict__ cw, const float *__restrict__ cb, int Cd) {
    __shared__ float s_dt[kPrepHeads][kBlk + 4];
    __shared__ float s_da[kPrepHeads][kBlk + 4];
    pdl_launch_dependents();                     // the next kernel waits for this one's writes itself
    const int blk = blockIdx.x, b = blockIdx.z;
    const int nhy = (H + kPrepHeads - 1) / kPrepHeads;
    if ((int)blockIdx.y >= nhy) {
        const int g = (blockIdx.y - nhy) >> 2, quarter = (blockIdx.y - nhy) & 3;
        const int t0 = blk * kBlk + 32 * quarter;
        const size_t Lp = (size_t)nblk * kBlk;
        __half2 amax = __float2half2_rn(0.f);
        if constexpr (kConv) {
            // combined arrangement: B and C are conv1d + SiLU of xbc's channels
            // H*P + g*N.. (B) and H*P + G*N + g*N.. (C), rounded to bf16 as the
            // split conv stores them.  Thread: one tensor, one 8-channel chunk,
            // 4 consecutive rows, from a window of the 3 rows before them too
            const int HP = Cd - 2 * G * kN;
            const int which = threadIdx.x >> 7, kk = threadIdx.x & 15, r0 = 4 * ((threadIdx.x >> 4) & 7);
            const size_t ch0 = (size_t)HP + (size_t)which * G * kN + (size_t)g * kN + kk * 8;
            uint4 v[4 + kConvK - 1];
#pragma unroll
            for (int j = 0; j < 4 + kConvK - 1; ++j) {
                const int tt = t0 + r0 - (kConvK - 1) + j;
                v[j] = make_uint4(0u, 0u, 0u, 0u);
                if (tt >= 0 && tt < L)
                    v[j] = __ldg(reinterpret_cast<const uint4 *>(Bm + ((size_t)b * L + tt) * Cd + ch0));
            }
            float4 wv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) wv[e] = __ldg(reinterpret_cast<const float4 *>(cw + (ch0 + e) * kConvK));
            const float4 b0 = __ldg(reinterpret_cast<const float4 *>(cb + ch0));
            const float4 b1 = __ldg(reinterpret_cast<const float4 *>(cb + ch0 + 4));
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
            float xin[4 + kConvK - 1][8];
#pragma unroll
            for (int j = 0; j < 4 + kConvK - 1; ++j) bf16_chunk_to_f32(v[j], xin[j]);
            __half *dst = which ? ws.Ch : ws.Bh;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int t = t0 + r0 + j;
                float f[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float w4[kConvK] = {wv[e].x, wv[e].y, wv[e].z, wv[e].w};
                    const float xw[kConvK] = {xin[j][e], xin[j + 1][e], xin[j + 2][e], xin[j + 3][e]};
                    f[e] = t < L ? bf16_round(conv_silu<kConvK>(w4, xw, bv[e])) : 0.f;
                }
                *reinterpret_cast<uint4 *>(dst + (((size_t)b * Lp + t) * G + g) * kN + kk * 8) = pack8(f, amax);
            }
            if (!in_f16_range(amax)) flag_status(ws.status, kStatusRange);
            return;
        }
        // 2 tensors x 32 rows x 16 chunks of 8: four chunks per thread, all loads first
        uint4 v[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int c = threadIdx.x + 256 * r;
            const int which = c >> 9, row = (c >> 4) & 31, kk = c & 15;
            const int t = t0 + row;
            const __nv_bfloat16 *src = which ? Cm : Bm;
            v[r] = make_uint4(0u, 0u, 0u, 0u);
            if (t < L) v[r] = __ldg(reinterpret_cast<const uint4 *>(src + (((size_t)b * L + t) * G + g) * kN + kk * 8));
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int c = threadIdx.x + 256 * r;
            const int which = c >> 9, row = (c >> 4) & 31, kk = c & 15;
            const int t = t0 + row;
            __half *dst = which ? ws.Ch : ws.Bh;
            float f[8];
            bf16_chunk_to_f32(v[r], f);
            *reinterpret_cast<uint4 *>(dst + (((size_t)b * Lp + t) * G + g) * kN + kk * 8) = pack8(f, amax);
        }
        if (!in_f16_range(amax)) flag_status(ws.status, kStatusRange);
        return;
    }
    const int h0 = blockIdx.y * kPrepHeads;
    const int nh = min(kPrepHeads, H - h0);
    {
        // thread -> head hh = tid % 8, tokens tid / 8 + 32 r: all 4 loads in flight first
        const int hh = threadIdx.x & (kPrepHeads - 1);
        const bool hv = hh < nh;
        const float bias = hv ? dt_bias[h0 + hh] : 0.f, Ah = hv ? A[h0 + hh] : 0.f;
        float raw[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int t = blk * kBlk + (threadIdx.x >> 3) + 32 * r;
            raw[r] = (hv && t < L) ? dt_raw[((size_t)b * L + t) * H + h0 + hh] : 0.f;
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int tok = (threadIdx.x >> 3) + 32 * r;
            const int t = blk * kBlk + tok;
            float d = 0.f;
            if (hv && t < L) d = dt_of(raw[r], bias, lo, hi);
            s_dt[hh][tok] = d;
            s_da[hh][tok] = d * Ah;
        }
    }
    if (blk == 0 && b == 0 && threadIdx.x < nh && A[h0 + threadIdx.x] > 0.f)
        flag_status(ws.status, kStatusPrecondition);
    __syncthreads();
    // warp w: inclusive cumsum of dA over the block for head w (four tokens per lane, fixed order)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp < nh) {
        const float4 da = *reinterpret_cast<const float4 *>(&s_da[warp][4 * lane]);
        const float c0 = da.x, c1 = c0 + da.y, c2 = c1 + da.z, c3 = c2 + da.w;
        float incl = c3;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float u = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += u;
        }
        const float ex = incl - c3;
        const size_t base = ((size_t)b * H + h0 + warp) * (size_t)nblk * kBlk + (size_t)blk * kBlk + 4 * lane;
        *reinterpret_cast<float4 *>(ws.cum + base) = make_float4(ex + c0, ex + c1, ex + c2, ex + c3);
        *reinterpret_cast<float4 *>(ws.dt + base) = *reinterpret_cast<const float4 *>(&s_dt[warp][4 * lane]);
    }
    // packed rows: the first head slice also records, for each token of the
    // block, the last document start at or before it (an inclusive max-scan
    // of the start positions; a start is a token whose id differs from the
    // previous token's, tokens past L start nothing)
    if (seq_idx && blockIdx.y == 0) {
        __shared__ int s_wmax[4];
        const int t = blk * kBlk + threadIdx.x;
        int v = -1;
        if (threadIdx.x < kBlk && t > 0 && t < L && seq_idx[(size_t)b * L + t] != seq_idx[(size_t)b * L + t - 1])
            v = threadIdx.x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v = max(v, u);
        }
        if (lane == 31 && warp < 4) s_wmax[warp] = v;
        __syncthreads();
        if (threadIdx.x < kBlk) {
            for (int w2 = 0; w2 < warp; ++w2) v = max(v, s_wmax[w2]);
            ws.rs[(size_t)b * nblk * kBlk + (size_t)blk * kBlk + threadIdx.x] = v;
        }
    }
}

// ---------------------------------------------------------------------------
// unit_state: grid (H, U-1, b), 8 compute warps + 1 control warp, 2 CTAs per
// SM, two TMA stages of (B fp16, X bf16, dt, cum), and x of the two blocks
// after them requested into L2.  The control warp's lane 0
// issues the TMA copies and the MMAs; the compute warps only widen X (scaled
// by w) and signal.  Units 0..U-2 never hold the sequence's ragged tail (it
// is in the last unit), so every block here is a full 128 tokens.
constexpr int kUsCompute = 256;
constexpr int kUsPrefetch = 2;   // blocks of x requested into L2 ahead of the two stages
constexpr int kUsThreads = kUsCompute + 32;
// stage: B (2 tiles), X (1 tile; kXRaw rows in the combined arrangement), dt, cum
template <bool kConv> struct UsLayout {
    static constexpr uint32_t kXBytes = kConv ? kXRawBytes : kTileBytes;
    static constexpr uint32_t kTx = 2 * kTileBytes + kXBytes + 2 * kBlk * 4;    // bytes a stage receives
    static constexpr uint32_t kStage = (kTx + 1023) & ~1023u;                  // 1024-aligned stages
    static constexpr uint32_t kOffW = 2 * kStage;                              // w [2][128]
    static constexpr uint32_t kOffCw = kOffW + 2 * kBlk * 4;                   // conv weights [80] float4
    static constexpr uint32_t kOffBar = kOffCw + (kConv ? 80 * 16 : 0);        // tma[2], mma[2], converted[2]
    static constexpr size_t kSmem = 1024 + kOffBar + 6 * 8 + 16;
};

template <bool kConv>
__global__ void __launch_bounds__(kUsThreads, 2)
unit_state_kernel(const __grid_constant__ TcMaps maps, TcWs ws, int H, int G, int nblk, int U, int bpu,
                  int packed, const float *__restrict__ cw, const float *__restrict__ cb) {
    using Lay = UsLayout<kConv>;
    constexpr uint32_t kUsStage = Lay::kStage, kUsOffW = Lay::kOffW, kUsOffBar = Lay::kOffBar;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    // per stage: [0,1] TMA landed, [2,3] MMAs done, [4,5] X converted.  One barrier of
    // each kind per stage keeps every waiter within one phase of its signaller.
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + kUsOffBar);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar + 6);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);

    const int h = blockIdx.x, u = blockIdx.y, b = blockIdx.z;
    const int g = h / (H / G);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t bh = (size_t)b * H + h;
    const int kb0 = u * bpu, kb1 = min(nblk, kb0 + bpu);
    const int nk = kb1 - kb0;
    const float *cumg = ws.cum + bh * (size_t)nblk * kBlk;
    const float *dtg = ws.dt + bh * (size_t)nblk * kBlk;
    auto stage = [&](int s) { return sm + s * kUsStage; };

    if (warp == 0) {
        tmem_alloc(tslot, 64);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 6; ++i) mbar_init(bar + i, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    pdl_launch_dependents();
    pdl_wait_prerequisites();                    // dt, cum and the fp16 B come from prep

    if (warp == kUsCompute / 32) {
        // ------------------------------ control warp --------------------------
        if (lane == 0) {
            auto load = [&](int s, int k) {
                uint8_t *st = stage(s);
                const int t0 = k * kBlk;
                mbar_arrive_expect_tx(bar + s, Lay::kTx);
                tma_load_4d(st, &maps.B, bar + s, 0, g, t0, b);
                tma_load_4d(st + kTileBytes, &maps.B, bar + s, 64, g, t0, b);
                tma_load_4d(st + 2 * kTileBytes, &maps.x, bar + s, 0, h, kConv ? t0 - (kConvK - 1) : t0, b);
                bulk_load(st + 2 * kTileBytes + Lay::kXBytes, dtg + (size_t)t0, kBlk * 4, bar + s);
                bulk_load(st + 2 * kTileBytes + Lay::kXBytes + kBlk * 4, cumg + (size_t)t0, kBlk * 4, bar + s);
            };
            // x of block k into L2 (x is the kernel's DRAM stream; B comes from L2, where
            // the group's heads share it): two blocks beyond the two stages, so more of
            // the row's reads are in flight than the stages hold
            auto prefetch_x = [&](int k) {
                if (k < kb1) tma_prefetch_4d(&maps.x, 0, h, kConv ? k * kBlk - (kConvK - 1) : k * kBlk, b);
            };
            const uint32_t idesc = idesc_f16(128, 64, 1, 1);
            bool ok = true;
            for (int i = 0; i < 2 && i < nk; ++i) load(i, kb0 + i);
            for (int i = 2; i < 2 + kUsPrefetch; ++i) prefetch_x(kb0 + i);
            for (int i = 0; i < nk && ok; ++i) {
                const int s = i & 1;
                ok = mbar_wait_abortable(bar + 4 + s, ((uint32_t)i >> 1) & 1u, kWaitBudget, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t b_base = smem_u32(stage(s)), x_base = smem_u32(stage(s) + 2 * kTileBytes);
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    mma_f16(tmem, sdesc_sw128(b_base + q * 2048, kTileBytes, 1024),
                            sdesc_sw128(x_base + q * 2048, kTileBytes, 1024), idesc, (i > 0 || q > 0) ? 1u : 0u);
                mma_commit(bar + 2 + s);
                if (i + 2 < nk) {       // refill stage s once these MMAs have read it
                    ok = mbar_wait_abortable(bar + 2 + s, ((uint32_t)i >> 1) & 1u, kWaitBudget, abort_flag);
                    if (ok) {
                        load(s, kb0 + i + 2);
                        prefetch_x(kb0 + i + 2 + kUsPrefetch);
                    }
                }
            }
        }
        __syncwarp();
    } else {
        // ------------------------------ compute warps -------------------------
        __half2 amax = __float2half2_rn(0.f);
        bool ok = true;
        float4 *cwb = reinterpret_cast<float4 *>(sm + Lay::kOffCw);
        if (kConv) conv_load_weights(cwb, cw, cb, h, tid, kUsCompute);   // visible after the first barrier below
        // the unit's log decay after the current block (sum of later block totals);
        // packed rows: how many later blocks of the unit hold a document start
        const int *rsb = ws.rs + (size_t)b * nblk * kBlk;
        float suffix = 0.f;
        int later = 0;
        if (tid < kBlk)
            for (int k = kb0 + 1; k < kb1; ++k) {
                suffix += cumg[(size_t)k * kBlk + kBlk - 1];
                if (packed) later += rsb[(size_t)k * kBlk + kBlk - 1] >= 0;
            }
        if (tid == 0) {
            const bool starts = packed && (later > 0 || rsb[(size_t)kb0 * kBlk + kBlk - 1] >= 0);
            // a unit that holds a document start passes no decayed state on
            ws.ell[bh * U + u] = starts ? -INFINITY : suffix + cumg[(size_t)kb0 * kBlk + kBlk - 1];
        }
        for (int i = 0; i < nk; ++i) {
            const int s = i & 1;
            uint8_t *st = stage(s);
            const float *dt = reinterpret_cast<const float *>(st + 2 * kTileBytes + Lay::kXBytes);
            const float *cum = dt + kBlk;
            float *w = reinterpret_cast<float *>(sm + kUsOffW) + s * kBlk;
            ok = ok && mbar_wait_abortable(bar + s, ((uint32_t)i >> 1) & 1u, kWaitBudget, abort_flag);
            if (ok && tid < kBlk) {
                // packed rows: only the unit's last document writes into its state
                const bool cut = packed && (later > 0 || tid < rsb[(size_t)(kb0 + i) * kBlk + kBlk - 1]);
                w[tid] = cut ? 0.f : expf(fminf(cum[kBlk - 1] - cum[tid] + suffix, 0.f)) * dt[tid];
            }
            if (tid < kBlk && kb0 + i + 1 < kb1) {
                suffix -= cumg[(size_t)(kb0 + i + 1) * kBlk + kBlk - 1];
                if (packed) later -= rsb[(size_t)(kb0 + i + 1) * kBlk + kBlk - 1] >= 0;
            }
            named_bar_sync(kUsCompute);                 // w[] visible
            if (kConv) {
                // w.X (fp16) straight from the raw rows: conv1d + SiLU, bf16, times w
                conv_x_tile<true>(st + 2 * kTileBytes, cwb, tid, 0, 0, ok, w, &amax);
            } else if (ok) {
                uint8_t *sx = st + 2 * kTileBytes;      // X (bf16) -> w.X (fp16); row = offset / 128
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int c = tid + r * kUsCompute;
                    uint4 *p = reinterpret_cast<uint4 *>(sx + c * 16);
                    float f[8];
                    bf16_chunk_to_f32(*p, f);
                    const float wr = w[c >> 3];
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] *= wr;
                    *p = pack8(f, amax);
                }
            }
            fence_proxy_async_smem();
            named_bar_sync(kUsCompute);
            if (tid == 0) mbar_arrive(bar + 4 + s);
        }
        // the accumulated state: wait for the last block's MMAs
        const int sl = (nk - 1) & 1;
        ok = __all_sync(0xffffffffu, ok && mbar_wait_abortable(bar + 2 + sl, ((uint32_t)(nk - 1) >> 1) & 1u,
                                                                   kWaitBudget, abort_flag));
        tc_fence_after();
        if (ok) {
            // 8 warps: lanes 32*(warp%4).., columns 32*(warp/4)..
            const int n = 32 * (warp & 3) + lane, ch = warp >> 2;
            float v[32];
            tmem_ld32(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + ch * 32, v);
            float *dst = ws.states + (bh * U + u) * (size_t)kNP + (size_t)n * kP + ch * 32;
#pragma unroll
            for (int q = 0; q < 8; ++q)
                *reinterpret_cast<float4 *>(dst + 4 * q) =
                    make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
        if (__any_sync(0xffffffffu, !in_f16_range(amax)) && lane == 0) flag_status(ws.status, kStatusRange);
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) flag_status(ws.status, kStatusTimeout);
    if (warp == 0) tmem_dealloc(tmem, 64);
}

// ---------------------------------------------------------------------------
// state_pass: grid (N*P/4/256, H, b), 256 threads; each thread owns one
// float4 of the state and issues its loads for a batch of units before the
// serial combine.
constexpr int kSpBatch = 8;

__global__ void __launch_bounds__(256)
tc_state_pass_kernel(TcWs ws, const float *__restrict__ init, int H, int U) {
    pdl_launch_dependents();
    pdl_wait_prerequisites();                    // the unit states come from unit_state
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
// chunk_out: grid (H, U, b), one CTA per SM: 8 compute warps, an MMA warp and
// a TMA warp.
//
// The MMA warp's lane 0 issues every tcgen05.mma, the TMA warp's lane 0
// every bulk copy; both only wait on mbarriers, so the compute warps never
// stall on an issue (a tcgen05.mma holds its issuing thread for about as
// long as it runs).  Per 128-token block k the compute warps run:
//   [1] C.B^T(k) done -> W(k) into TMEM (bf16 high and low parts, the A
//       operands of W.X)              -> MMA: Y(k) = W_hi(k) X(k) + W_lo(k) X(k),
//                                        then C.B^T(k+1)
//   [2] x/dt/cum(k+1) landed -> decay factors of block k+1
//   [3] S(k), Z(k) done -> H_in(k+1) = a_k H_in(k) + S(k) in registers, its
//       fp16 copy, and w.X(k+1)       -> MMA: Z(k+1) = C(k+1) H_in(k+1) and
//                                        S(k+1) = B^T (w.X(k+1))
// S(k+1) needs no W, so it runs a whole block before [3] of k+1 reads it.
//   [4] Y(k) done -> y(k) = Y + exp(cum) Z(k) + D x, staged in block k's B tiles
//                                     -> TMA: store y(k); x/dt/cum(k+3), C/B(k+2)
// while the MMA warp issues C.B^T(k+1) as soon as C/B(k+1) have landed.  C
// and B (fp16 copies) are double-buffered by block parity; x with dt and cum
// rotates through three slots, so it is fetched more than a block ahead.
// Compute warp w owns TMEM lanes 32*(w%4).. (its rows) and column half w/4:
// C.B^T column slices w/4 and w/4+2, and 32 of the 64 Y/Z/S/state columns.
constexpr int kCoCompute = 256;                                 // 8 compute warps
constexpr int kCoWarps = kCoCompute / 32;
constexpr int kCoMmaWarp = kCoWarps, kCoTmaWarp = kCoWarps + 1;
constexpr int kCoThreads = kCoCompute + 64;                     // + MMA warp + TMA warp
constexpr uint32_t kCoCB = 4 * kTileBytes;                      // C(2 tiles) B(2 tiles) of one block
// x slot: X (kXRaw rows: room for the combined arrangement's raw rows), dt[128], cum[128]
constexpr uint32_t kCoXS = (kXRawBytes + 1024 + 1023) & ~1023u;
constexpr int kCoXSlots = 3;
constexpr uint32_t kCoOffXS = 2 * kCoCB;                        // x ring
constexpr uint32_t kCoOffWX = kCoOffXS + kCoXSlots * kCoXS;     // w.X fp16
constexpr uint32_t kCoOffH16 = kCoOffWX + kTileBytes;           // fp16 entering state [n][p]
constexpr uint32_t kCoFactors = 320;                            // w[128], v0[32], v1[64], v2[96]
constexpr uint32_t kCoOffF = kCoOffH16 + kTileBytes;            // factors [2][320] floats
constexpr uint32_t kCoOffG = kCoOffF + 2 * kCoFactors * 4;      // diagonal fast-path flags [2][4]
constexpr uint32_t kCoOffMask = kCoOffG + 8 * 4;                // causal masks of the diagonal [4][32 lanes] x 16 B
constexpr uint32_t kCoOffIss = kCoOffMask + 32 * 16 * 4;        // issue counters (drain after an abort)
constexpr uint32_t kCoOffCw = kCoOffIss + 16 * 4;               // conv weights [64] + biases [16] float4
constexpr uint32_t kCoOffBar = kCoOffCw + 80 * 16;              // mbarriers, TMEM slot, abort flag
constexpr int kCoBars = 13;
constexpr size_t kCoSmem = 1024 + kCoOffBar + kCoBars * 8 + 16;
constexpr float kDiagExpCap = 64.0f;                            // largest exponent on the diagonal fast path
constexpr double kL2Bytes = 126e6;                              // B200 L2
static_assert(kCoXS % 1024 == 0 && kCoCB % 1024 == 0, "tiles must stay 1024-byte aligned");
static_assert(kCoSmem <= 232448, "chunk_out shared memory exceeds the per-CTA limit");

// TMEM columns (512 allocated)
constexpr uint32_t kTmCB = 0;      // C.B^T fp32, 128 columns
constexpr uint32_t kTmW = 128;     // W bf16 pairs, the high part (W truncated to bf16), 64 columns
constexpr uint32_t kTmY = 192;     // W.X fp32, 64 columns
constexpr uint32_t kTmS = 256;     // B^T.(w.X) fp32, 64 columns
constexpr uint32_t kTmZ = 320;     // C.H fp32, two buffers of 64 columns (block parity)
constexpr uint32_t kTmWlo = 448;   // W bf16 pairs, the low part (W - high, rounded), 64 columns

// "Block done" has one barrier per C/B stage: block k+2 cannot finish before
// the TMA warp has seen block k finish and loaded k+2's tiles, so that waiter
// never falls two phases behind.
enum CoBar { kBarTcb0 = 0, kBarTcb1 = 1, kBarTx0 = 2, kBarTx1 = 3, kBarTx2 = 4,       // copies landed
             kBarCB = 5, kBarS = 6, kBarY = 7, kBarZ = 8,                            // MMAs done
             kBarW = 9, kBarH16 = 10, kBarFree0 = 11, kBarFree1 = 12 };              // compute -> issuers
constexpr int kFirstComputeBar = kBarW;

// v_g (pivot m = 32g+31, j <= m) starts at this factor index; w is v_3.
__host__ __device__ constexpr int voff(int g) { return g == 3 ? 0 : 128 + 16 * g * (g + 1); }

struct CoSmem {
    uint8_t *base;
    __device__ uint8_t *C(int s) const { return base + s * kCoCB; }
    __device__ uint8_t *B(int s) const { return base + s * kCoCB + 2 * kTileBytes; }
    __device__ uint8_t *X(int r) const { return base + kCoOffXS + r * kCoXS; }
    __device__ float *dt(int r) const { return reinterpret_cast<float *>(X(r) + kXRawBytes); }
    __device__ float *cum(int r) const { return dt(r) + kBlk; }
    __device__ uint8_t *WX() const { return base + kCoOffWX; }
    __device__ uint8_t *H16() const { return base + kCoOffH16; }
    __device__ float *F(int s) const { return reinterpret_cast<float *>(base + kCoOffF) + s * kCoFactors; }
    __device__ int *G(int s) const { return reinterpret_cast<int *>(base + kCoOffG) + s * 4; }
    __device__ uint4 *Mask() const { return reinterpret_cast<uint4 *>(base + kCoOffMask); }
    __device__ int *issued() const { return reinterpret_cast<int *>(base + kCoOffIss); }
    __device__ float4 *Cw() const { return reinterpret_cast<float4 *>(base + kCoOffCw); }
    __device__ uint64_t *bar(int i) const { return reinterpret_cast<uint64_t *>(base + kCoOffBar) + i; }
    __device__ uint32_t *tslot() const { return reinterpret_cast<uint32_t *>(bar(kCoBars)); }
    __device__ volatile int *abort_flag() const { return reinterpret_cast<volatile int *>(bar(kCoBars)) + 1; }
};

// Shared-memory descriptors advance by (byte offset >> 4) in their low field
// (smem addresses stay below 2^18, so the 14-bit field never carries).
__device__ __forceinline__ uint64_t dadd(uint64_t desc, uint32_t bytes) { return desc + (bytes >> 4); }

// TMA: C and B (fp16 copies) of block k into stage s
__device__ __forceinline__ void co_load_cb(const CoSmem &S, const TcMaps &maps, int s, int k, int g, int b) {
    const int t0 = k * kBlk;
    uint64_t *bar = S.bar(kBarTcb0 + s);
    mbar_arrive_expect_tx(bar, kCoCB);
    tma_load_4d(S.C(s), &maps.C, bar, 0, g, t0, b);
    tma_load_4d(S.C(s) + kTileBytes, &maps.C, bar, 64, g, t0, b);
    tma_load_4d(S.B(s), &maps.B, bar, 0, g, t0, b);
    tma_load_4d(S.B(s) + kTileBytes, &maps.B, bar, 64, g, t0, b);
    ++S.issued()[kBarTcb0 + s];
}

// TMA: C and B (fp16 copies) of block k into L2 a block ahead of their load
// into shared memory (the heads of a group read them at about the same time,
// so the first request would otherwise wait for DRAM with the rest behind it)
__device__ __forceinline__ void co_prefetch_cb(const TcMaps &maps, int k, int g, int b) {
    const int t0 = k * kBlk;
    tma_prefetch_4d(&maps.C, 0, g, t0, b);
    tma_prefetch_4d(&maps.C, 64, g, t0, b);
    tma_prefetch_4d(&maps.B, 0, g, t0, b);
    tma_prefetch_4d(&maps.B, 64, g, t0, b);
}

// TMA: X (bf16), dt and cum rows of block k into x slot r.  Combined
// arrangement: the raw x channels of xbc for the block's tokens and the 3
// before them (zero before token 0).
template <bool kConv>
__device__ __forceinline__ void co_load_x(const CoSmem &S, const TcMaps &maps, const float *dtv, const float *cum,
                                          int r, int k, int h, int b) {
    const int t0 = k * kBlk;
    uint64_t *bar = S.bar(kBarTx0 + r);
    mbar_arrive_expect_tx(bar, (kConv ? kXRawBytes : kTileBytes) + 2 * kBlk * 4);
    tma_load_4d(S.X(r), &maps.x, bar, 0, h, kConv ? t0 - (kConvK - 1) : t0, b);
    bulk_load(S.dt(r), dtv + (size_t)t0, kBlk * 4, bar);
    bulk_load(S.cum(r), cum + (size_t)t0, kBlk * 4, bar);
    ++S.issued()[kBarTx0 + r];
}

// Per-block decay factors into F(f), from the dt/cum of x slot r (all
// exponents clamped as stated):
//   v_g[j] = exp(min(cum_m - cum_j, 0)) dt_j,  m = 32g+31, j <= m, g = 0..2
//   w[j]   = v_3[j] = exp(min(cum_last - cum_j, 0)) dt_j         (state update)
// Row group g uses v_{g-1} below its diagonal sub-block and v_g on it; the
// flag says the diagonal may use the factored form (its total decay is
// below exp(-cap), so no row factor there exceeds exp(cap)).
__device__ __forceinline__ void co_factors(const CoSmem &S, int r, int f, int last_valid, int tid) {
    const float *cum = S.cum(r), *dt = S.dt(r);
    float *F = S.F(f);
    const float clast = cum[last_valid];
    for (int idx = tid; idx < (int)kCoFactors; idx += kCoCompute) {
        float cm;
        int j;
        if (idx < kBlk) {
            cm = clast;
            j = idx;
        } else {
            const int q = idx - kBlk, g = q < 32 ? 0 : (q < 96 ? 1 : 2);
            j = q - 16 * g * (g + 1);
            cm = cum[32 * g + 31];
        }
        F[idx] = expf(fminf(cm - cum[j], 0.f)) * dt[j];
    }
    if (tid < 4) S.G(f)[tid] = (cum[32 * tid] - cum[32 * tid + 31]) <= kDiagExpCap ? 1 : 0;
}

// w.X (fp16) of the X tile of slot r (bf16, as the TMA delivered it) into
// WX, same swizzled layout (a chunk's row is its offset / 128 whatever the
// swizzle): products in fp32, rounded to fp16 once.  Packed rows: tokens
// before the block's last document start (rs_last; -1 for none) write nothing
// into the state the block passes on.
//
// chunk_out tracks no fp16 range per operand: a value beyond +-65504 in an
// fp16 operand it forms (w.X, the entering state) rounds to inf, and each
// reaches y or the final state through a product and a sum, where inf stays
// inf or turns NaN (inf * 0).  One finiteness check on y and the final state
// (co_nonfinite) therefore reports it, off the W path.  W itself is carried
// in bf16 (hi/lo), which cannot overflow.
__device__ __forceinline__ void co_form_wx(const CoSmem &S, int r, int f, int tid, int rs_last) {
    const float *w = S.F(f);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int c = tid + q * kCoCompute;
        float xv[8];
        bf16_chunk_to_f32(*reinterpret_cast<const uint4 *>(S.X(r) + c * 16), xv);
        const float wj = (c >> 3) >= rs_last ? w[c >> 3] : 0.f;
        const float2 w2 = make_float2(wj, wj);
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 m = __fmul2_rn(make_float2(xv[2 * e], xv[2 * e + 1]), w2);
            o[e] = pack_h2(m.x, m.y);
        }
        *reinterpret_cast<uint4 *>(S.WX() + c * 16) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// A compute warp hands its shared-memory and TMEM writes to the issuing
// warps: one arrival per warp on `bar` (initialised with kCoWarps).
__device__ __forceinline__ void co_arrive(uint64_t *bar, int lane) {
    fence_proxy_async_smem();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar);
}

// The same for TMEM writes only (tcgen05.st, already waited for): no
// generic-to-async proxy fence is needed for them.
__device__ __forceinline__ void co_arrive_tmem(uint64_t *bar, int lane) {
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar);
}

// 16 floats -> 8 fp16 pairs
__device__ __forceinline__ void pack16(const float *v, uint32_t *o) {
#pragma unroll
    for (int q = 0; q < 8; ++q) o[q] = pack_h2(v[2 * q], v[2 * q + 1]);
}

// Accumulates v*0 over 32 floats: the sum stays 0 unless a value is inf or NaN.
__device__ __forceinline__ void co_nonfinite(const float *v, int n, float2 &acc) {
    const float2 z = make_float2(0.f, 0.f);
#pragma unroll
    for (int q = 0; q < 16; ++q)
        if (2 * q < n) acc = __ffma2_rn(make_float2(v[2 * q], v[2 * q + 1]), z, acc);
}

// W for one 32-column slice cq <= lg of this thread's row i (see co_factors),
// stored as two bf16 pairs per column: the high part (W truncated to bf16)
// and the low part (the rest, rounded to bf16).  Y = W_hi X + W_lo X then
// carries W to about 16 significant bits: y is heavy-tailed (single W.X
// terms of 50 to 60 times the output RMS), and the 11 bits of an fp16 W
// leave those terms' rounding above the 2e-2 RMS bar.
// Packed rows: rs_i is the last document start at or before row i in the
// block (-1 for none); columns before it drop out of the row.
__device__ __forceinline__ void co_w_slice(const CoSmem &S, int r, int f, uint32_t lane_addr, int lg, int cq,
                                           int lane, float ci, int rs_i) {
    const float *cum = S.cum(r);
    const float *F = S.F(f);
    float v[32];
    tmem_ld32(lane_addr + kTmCB + cq * 32, v);
    uint32_t oh[16], ol[16];                         // W as bf16 pairs: high part, low part
    if (cq < lg) {                                   // below the diagonal: pivot at row 32*lg-1
        const float ui = expf(fminf(ci - cum[32 * lg - 1], 0.f));
        const float2 u2 = make_float2(ui, ui);
        const float4 *vf = reinterpret_cast<const float4 *>(F + voff(lg - 1) + cq * 32);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float4 f4 = vf[q];
            const float2 m0 = __fmul2_rn(make_float2(v[4 * q], v[4 * q + 1]), __fmul2_rn(make_float2(f4.x, f4.y), u2));
            const float2 m1 =
                __fmul2_rn(make_float2(v[4 * q + 2], v[4 * q + 3]), __fmul2_rn(make_float2(f4.z, f4.w), u2));
            split_bf16x2(m0.x, m0.y, oh[2 * q], ol[2 * q]);
            split_bf16x2(m1.x, m1.y, oh[2 * q + 1], ol[2 * q + 1]);
        }
    } else {                                         // diagonal 32x32: pivot at its last row m
        if (S.G(f)[lg]) {
            // exp(cum_i - cum_j) = exp(cum_i - cum_m) exp(cum_m - cum_j); the first
            // factor is >= 1 and at most exp(cap) (flag), the second <= 1
            const float ud = expf(fminf(ci - cum[32 * lg + 31], kDiagExpCap));
            const float2 u2 = make_float2(ud, ud);
            const float4 *vf = reinterpret_cast<const float4 *>(F + voff(lg) + cq * 32);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 f4 = vf[q];
                const float2 m0 =
                    __fmul2_rn(__fmul2_rn(make_float2(v[4 * q], v[4 * q + 1]), make_float2(f4.x, f4.y)), u2);
                const float2 m1 =
                    __fmul2_rn(__fmul2_rn(make_float2(v[4 * q + 2], v[4 * q + 3]), make_float2(f4.z, f4.w)), u2);
                v[4 * q] = m0.x;
                v[4 * q + 1] = m0.y;
                v[4 * q + 2] = m1.x;
                v[4 * q + 3] = m1.y;
            }
        } else {                                     // steep decay: one exp per element
            const float *dts = S.dt(r) + cq * 32, *cj = cum + cq * 32;
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) {
                v[jj] = v[jj] * expf(fminf(ci - cj[jj], 0.f)) * dts[jj];
                asm volatile("" ::: "memory");       // one element at a time: keeps the loads from piling up
            }
        }
        // causal select on the packed pairs (j <= i kept), both parts
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
            const uint4 m4 = S.Mask()[q4 * 32 + lane];
            const uint32_t mw[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int q = 4 * q4 + e;
                split_bf16x2(v[2 * q], v[2 * q + 1], oh[q], ol[q]);
                oh[q] &= mw[e];
                ol[q] &= mw[e];
            }
        }
    }
    const int j0 = 32 * cq;
    if (rs_i > j0) {
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            const uint32_t keep =
                (j0 + 2 * q >= rs_i ? 0x0000FFFFu : 0u) | (j0 + 2 * q + 1 >= rs_i ? 0xFFFF0000u : 0u);
            oh[q] &= keep;
            ol[q] &= keep;
        }
    }
    tmem_st16u(lane_addr + kTmW + 16 * cq, oh);
    tmem_st16u(lane_addr + kTmWlo + 16 * cq, ol);
}

// kPacked: packed rows (the document starts of ws.rs mask W, the C.H term,
// w.X and the block decay); the unpacked instantiation carries none of it.
template <bool kPacked, bool kConv>
__global__ void __launch_bounds__(kCoThreads, 1)
chunk_out_kernel(const __grid_constant__ TcMaps maps, const float *__restrict__ D,
                 const float *__restrict__ init, float *__restrict__ final_state, TcWs ws,
                 int L, int H, int G, int nblk, int U, int bpu, int states_from_ws, int prefetch_cb,
                 float *__restrict__ chunk_states, int bpc, int nc, long long wait_budget, int test_fault,
                 const float *__restrict__ cw, const float *__restrict__ cb) {
    extern __shared__ uint8_t smem_raw[];
    CoSmem S;
    S.base = align1024(smem_raw);
    volatile int *abort_flag = S.abort_flag();

    const int h = blockIdx.x, u = blockIdx.y, b = blockIdx.z;
    const int g = h / (H / G);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t bh = (size_t)b * H + h;
    const int kb0 = u * bpu, kb1 = min(nblk, kb0 + bpu);
    const float *cumg = ws.cum + bh * (size_t)nblk * kBlk;
    const float *dtg = ws.dt + bh * (size_t)nblk * kBlk;

    if (warp == 0) {
        tmem_alloc(S.tslot(), 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < kCoBars; ++i) {
            mbar_init(S.bar(i), i < kFirstComputeBar ? 1 : kCoWarps);
            S.issued()[i] = 0;
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *S.tslot();
    pdl_wait_prerequisites();                    // prep (and the unit passes) wrote what follows reads

    if (warp == kCoMmaWarp) {
        // ------------------------------ MMA warp ------------------------------
        if (lane == 0) {
            const uint32_t idesc_cb = idesc_f16(128, 128, 0, 0);  // A=C K-major, B=B K-major
            const uint32_t idesc_z = idesc_f16(128, 64, 0, 1);    // A=C K-major, B=H MN-major
            const uint32_t idesc_y = idesc_bf16(128, 64, 0, 1);   // A=W hi/lo (TMEM) bf16, B=X (bf16) MN-major
            const uint32_t idesc_s = idesc_f16(128, 64, 1, 1);    // A=B^T MN-major, B=wX MN-major
            // per-stage / per-slot descriptors are the first one's plus a byte offset
            // (no arrays: a dynamically indexed one would live in local memory)
            const uint64_t dC0 = sdesc_sw128(smem_u32(S.C(0)), 16, 1024);
            const uint64_t dBk0 = sdesc_sw128(smem_u32(S.B(0)), 16, 1024);
            const uint64_t dBm0 = sdesc_sw128(smem_u32(S.B(0)), kTileBytes, 1024);
            const uint64_t dX0 = sdesc_sw128(smem_u32(S.X(0)), kTileBytes, 1024);
            const uint64_t dWX = sdesc_sw128(smem_u32(S.WX()), kTileBytes, 1024);
            const uint64_t dH = sdesc_sw128(smem_u32(S.H16()), kTileBytes, 1024);
            auto st = [](int s) { return (uint32_t)s * kCoCB; };
            auto xs = [](int r) { return (uint32_t)r * kCoXS; };
            // K-major K-step q of a 128-wide tile: column block q/4, 32 bytes per step inside it
            auto kofs = [](int q) { return (uint32_t)((q >> 2) * kTileBytes + (q & 3) * 32); };
            auto issue_cb = [&](int s) {
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    mma_f16(tmem + kTmCB, dadd(dC0, st(s) + kofs(q)), dadd(dBk0, st(s) + kofs(q)), idesc_cb, q > 0);
                mma_commit(S.bar(kBarCB));
                ++S.issued()[kBarCB];
            };
            auto issue_z = [&](int s, int zb) {
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    mma_f16(tmem + kTmZ + 64u * zb, dadd(dC0, st(s) + kofs(q)), dadd(dH, q * 2048), idesc_z, q > 0);
                mma_commit(S.bar(kBarZ));
                ++S.issued()[kBarZ];
            };
            auto issue_s = [&](int s) {
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    mma_f16(tmem + kTmS, dadd(dBm0, st(s) + q * 2048), dadd(dWX, q * 2048), idesc_s, q > 0);
                mma_commit(S.bar(kBarS));
                ++S.issued()[kBarS];
            };
            auto issue_y = [&](int r) {
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    mma_f16_ts(tmem + kTmY, tmem + kTmW + 8u * q, dadd(dX0, xs(r) + q * 2048), idesc_y, q > 0);
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    mma_f16_ts(tmem + kTmY, tmem + kTmWlo + 8u * q, dadd(dX0, xs(r) + q * 2048), idesc_y, 1u);
                mma_commit(S.bar(kBarY));
                ++S.issued()[kBarY];
            };
            // "fp16 state ready" also means w.X of that block is formed
            bool ok = mbar_wait_abortable(S.bar(kBarTcb0), 0, wait_budget, abort_flag);
            tc_fence_after();
            if (ok) issue_cb(0);
            ok = ok && mbar_wait_abortable(S.bar(kBarH16), 0, wait_budget, abort_flag);
            tc_fence_after();
            if (ok) {
                issue_z(0, 0);
                issue_s(0);
            }
            for (int k = kb0; k < kb1 && ok; ++k) {
                const int i = k - kb0, s1 = (i & 1) ^ 1;
                const uint32_t par = (uint32_t)i & 1u, par1 = (uint32_t)(i + 1) & 1u;
                ok = mbar_wait_abortable(S.bar(kBarW), par, wait_budget, abort_flag);
                if (!ok) break;
                tc_fence_after();
                issue_y(i % kCoXSlots);
                if (k + 1 < kb1) {
                    // C.B^T(k+1) once its tiles have landed (W(k) has read C.B^T(k))
                    ok = mbar_wait_abortable(S.bar(kBarTcb0 + s1), ((uint32_t)(i + 1) >> 1) & 1u, wait_budget,
                                             abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    issue_cb(s1);
                    // Z(k+1), S(k+1) once the fp16 state and w.X of k+1 are formed (S(k)
                    // and Z(k) have been read by then)
                    ok = mbar_wait_abortable(S.bar(kBarH16), par1, wait_budget, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    issue_z(s1, (int)par1);
                    issue_s(s1);
                }
            }
            if (!ok) *abort_flag = 1;
        }
        __syncwarp();
    } else if (warp == kCoTmaWarp) {
        // ------------------------------ TMA warp ------------------------------
        if (lane == 0) {
            // test_fault 1: the first C/B stage is never requested, so every wait
            // that depends on it runs out of budget (the timeout path)
            for (int q = 0; q < 2 && kb0 + q < kb1; ++q)
                if (q > 0 || test_fault != 1) co_load_cb(S, maps, q, kb0 + q, g, b);
            for (int q = 0; q < kCoXSlots && kb0 + q < kb1; ++q)
                co_load_x<kConv>(S, maps, dtg, cumg, q, kb0 + q, h, b);
            if (prefetch_cb && kb0 + 2 < kb1) co_prefetch_cb(maps, kb0 + 2, g, b);
            for (int k = kb0; k < kb1; ++k) {
                const int i = k - kb0, s = i & 1;
                if (!mbar_wait_abortable(S.bar(kBarFree0 + s), ((uint32_t)i >> 1) & 1u, wait_budget, abort_flag))
                    break;
                // block k is done with its x slot; its y sits in its B tiles
                if (k + kCoXSlots < kb1) co_load_x<kConv>(S, maps, dtg, cumg, i % kCoXSlots, k + kCoXSlots, h, b);
                if (prefetch_cb && k + 3 < kb1) co_prefetch_cb(maps, k + 3, g, b);
                tma_store_4d(&maps.y, S.B(s), 0, h, k * kBlk, b);
                tma_store_4d(&maps.y, S.B(s) + kTileBytes, 32, h, k * kBlk, b);
                tma_store_commit();
                if (k + 2 < kb1) {
                    tma_store_wait_read();
                    co_load_cb(S, maps, s, k + 2, g, b);
                }
            }
            tma_store_wait_all();
        }
        __syncwarp();
    } else {
        // ------------------------------ compute warps -------------------------
        const int lg = warp & 3;                    // row group: rows 32*lg .. 32*lg+31
        const int row = 32 * lg + lane;             // TMEM lane / tile row of this thread
        const int ch = warp >> 2;                   // column half 0..1
        const uint32_t lane_addr = tmem + ((uint32_t)(32 * lg) << 16);
        const float Dh = D[h];
        float2 nonfinite = make_float2(0.f, 0.f);  // stays 0 unless y or the final state is inf or NaN
        bool ok = true;

        // entering state of the unit, row `row`, columns 32*ch..: registers and fp16 copy
        float hv[32];
        {
            const float *src = states_from_ws ? ws.states + (bh * U + u) * (size_t)kNP
                                              : (init ? init + bh * kNP : nullptr);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 f4 = src ? *reinterpret_cast<const float4 *>(src + (size_t)row * kP + ch * 32 + 4 * q)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
                hv[4 * q] = f4.x; hv[4 * q + 1] = f4.y; hv[4 * q + 2] = f4.z; hv[4 * q + 3] = f4.w;
            }
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t o[8];
                pack16(hv + 16 * hh, o);
#pragma unroll
                for (int q = 0; q < 2; ++q)
                    *reinterpret_cast<uint4 *>(S.H16() + sw128_off(row, 4 * ch + 2 * hh + q)) =
                        make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
            }
            // W above the diagonal sub-blocks stays zero for the whole kernel
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                const int cq = ch + 2 * t;
                if (cq > lg) {
                    uint32_t z[16];
#pragma unroll
                    for (int q = 0; q < 16; ++q) z[q] = 0u;
                    tmem_st16u(lane_addr + kTmW + 16 * cq, z);
                    tmem_st16u(lane_addr + kTmWlo + 16 * cq, z);
                }
            }
            // causal masks of a diagonal sub-block: lane l keeps columns jj <= l;
            // word q holds jj = 2q (low half) and 2q+1 (high half)
            if (tid < 128) {
                const int ml = tid & 31, q4 = tid >> 5;
                uint32_t mw[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int q = 4 * q4 + e;
                    mw[e] = (2 * q + 1 <= ml ? 0xFFFF0000u : 0u) | (2 * q <= ml ? 0x0000FFFFu : 0u);
                }
                S.Mask()[q4 * 32 + ml] = make_uint4(mw[0], mw[1], mw[2], mw[3]);
            }
        }
        if (kConv) conv_load_weights(S.Cw(), cw, cb, h, tid, kCoCompute);
        // block kb0: x landed -> factors, w.X; then "state ready"
        ok = mbar_wait_abortable(S.bar(kBarTx0), 0, wait_budget, abort_flag);
        if (ok) co_factors(S, 0, 0, min(kBlk - 1, L - 1 - kb0 * kBlk), tid);
        // combined arrangement: x of the first two blocks now, then each block's
        // two blocks ahead while W.X runs (the conv weights are read after
        // conv_x_tile's own barrier)
        if (kConv) {
            conv_x_tile<false>(S.X(0), S.Cw(), tid, kb0 * kBlk, L, ok);
            if (kb0 + 1 < kb1) {
                ok = ok && mbar_wait_abortable(S.bar(kBarTx0 + 1), 0, wait_budget, abort_flag);
                conv_x_tile<false>(S.X(1), S.Cw(), tid, (kb0 + 1) * kBlk, L, ok);
            }
        }
        named_bar_sync(kCoCompute);                 // factors and masks visible to every compute warp
        // packed rows: document starts of each block (ws.rs, written by prep)
        const int *rsb = ws.rs + (size_t)b * nblk * kBlk;
        if (ok) co_form_wx(S, 0, 0, tid, kPacked ? rsb[(size_t)kb0 * kBlk + kBlk - 1] : -1);
        co_arrive(S.bar(kBarH16), lane);

        // every compute warp runs every iteration (and so every named barrier);
        // after an abort the waits return at once and the work is skipped
        for (int k = kb0; k < kb1; ++k) {
            const int i = k - kb0, f = i & 1, f1 = f ^ 1;
            const int r = i % kCoXSlots, r1 = (i + 1) % kCoXSlots;
            const uint32_t par = (uint32_t)i & 1u;
            const int t0 = k * kBlk;
            const float *cum = S.cum(r);
            const int rs_row = kPacked ? rsb[(size_t)t0 + row] : -1;
            const int rs_last = kPacked ? rsb[(size_t)t0 + kBlk - 1] : -1;
            const int rs_last1 = (kPacked && k + 1 < kb1) ? rsb[(size_t)t0 + 2 * kBlk - 1] : -1;

            // [1] C.B^T(k) done -> W(k) (fp16 pairs) into TMEM
            ok = ok && mbar_wait_abortable(S.bar(kBarCB), par, wait_budget, abort_flag);
            ok = __all_sync(0xffffffffu, ok);        // warp-uniform before tcgen05.ld
            tc_fence_after();
            if (ok) {
                const float ci = cum[row];
                if (ch <= lg) co_w_slice(S, r, f, lane_addr, lg, ch, lane, ci, rs_row);
                if (ch + 2 <= lg) co_w_slice(S, r, f, lane_addr, lg, ch + 2, lane, ci, rs_row);
            }
            co_arrive_tmem(S.bar(kBarW), lane);

            // [2] block k+1: x landed -> factors (overlaps S(k), Y(k))
            if (k + 1 < kb1) {
                ok = ok && mbar_wait_abortable(S.bar(kBarTx0 + r1), ((uint32_t)(i + 1) / kCoXSlots) & 1u,
                                               wait_budget, abort_flag);
                if (ok) co_factors(S, r1, f1, min(kBlk - 1, L - 1 - (k + 1) * kBlk), tid);
                named_bar_sync(kCoCompute);          // factors (and x) of block k+1 visible
            }

            // [3] S(k) done (and Z(k), which read the fp16 copy) -> H_in(k+1), w.X(k+1)
            ok = ok && mbar_wait_abortable(S.bar(kBarS), par, wait_budget, abort_flag);
            ok = ok && mbar_wait_abortable(S.bar(kBarZ), par, wait_budget, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
            if (ok) {
                float sv[32];
                tmem_ld32(lane_addr + kTmS + ch * 32, sv);
                // a block that holds a document start passes no decayed state on
                const float a = rs_last >= 0 ? 0.f : expf(fminf(cum[min(kBlk - 1, L - 1 - t0)], 0.f));
                const float2 a2 = make_float2(a, a);
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const float2 rr = __ffma2_rn(a2, make_float2(hv[2 * q], hv[2 * q + 1]),
                                                 make_float2(sv[2 * q], sv[2 * q + 1]));
                    hv[2 * q] = rr.x;
                    hv[2 * q + 1] = rr.y;
                }
                if (k + 1 < kb1) {
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        uint32_t o[8];
                        pack16(hv + 16 * hh, o);
#pragma unroll
                        for (int q = 0; q < 2; ++q)
                            *reinterpret_cast<uint4 *>(S.H16() + sw128_off(row, 4 * ch + 2 * hh + q)) =
                                make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
                    }
                    co_form_wx(S, r1, f1, tid, rs_last1);
                } else if (final_state && u == U - 1) {
                    float *dst = final_state + bh * kNP + (size_t)row * kP + ch * 32;
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        *reinterpret_cast<float4 *>(dst + 4 * q) =
                            make_float4(hv[4 * q], hv[4 * q + 1], hv[4 * q + 2], hv[4 * q + 3]);
                    co_nonfinite(hv, 32, nonfinite);
                }
                // block k ends chunk k / bpc (the last block ends the last chunk)
                if (chunk_states && ((k + 1) % bpc == 0 || k == nblk - 1)) {
                    float *dst =
                        chunk_states + (((size_t)b * nc + k / bpc) * H + h) * kNP + (size_t)row * kP + ch * 32;
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        *reinterpret_cast<float4 *>(dst + 4 * q) =
                            make_float4(hv[4 * q], hv[4 * q + 1], hv[4 * q + 2], hv[4 * q + 3]);
                }
            }
            if (k + 1 < kb1) co_arrive(S.bar(kBarH16), lane);

            // [3b] combined arrangement: x of block k+2 (its slot was block k-1's)
            // while Y(k) runs; read by the compute warps after the next [2]
            // barrier, and by the MMAs after the next "state ready" arrival
            if (kConv && k + 2 < kb1) {
                const int r2 = (i + 2) % kCoXSlots;
                ok = ok && mbar_wait_abortable(S.bar(kBarTx0 + r2), ((uint32_t)(i + 2) / kCoXSlots) & 1u, wait_budget,
                                               abort_flag);
                conv_x_tile<false>(S.X(r2), S.Cw(), tid, (k + 2) * kBlk, L, ok);
            }

            // [4] Y(k) done -> y_i = Y_i + exp(cum_i) Z_i + D x_i -> staging in block k's B tiles
            ok = ok && mbar_wait_abortable(S.bar(kBarY), par, wait_budget, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
            if (ok) {
                // the entering state reaches a row only before the block's first document start
                const float ei = rs_row >= 0 ? 0.f : expf(fminf(cum[row], 0.f));
                const float2 e2 = make_float2(ei, ei), d2 = make_float2(Dh, Dh);
                uint8_t *stg = S.B(i & 1) + ch * kTileBytes;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float yv[16], zv[16];
                    tmem_ld16x2(lane_addr + kTmY + ch * 32 + 16 * hh, yv,
                                lane_addr + kTmZ + 64u * par + ch * 32 + 16 * hh, zv);
                    float xv[16];
                    bf16_chunk_to_f32(*reinterpret_cast<const uint4 *>(S.X(r) + sw128_off(row, 4 * ch + 2 * hh)),
                                      xv);
                    bf16_chunk_to_f32(
                        *reinterpret_cast<const uint4 *>(S.X(r) + sw128_off(row, 4 * ch + 2 * hh + 1)), xv + 8);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        float2 rr = __ffma2_rn(e2, make_float2(zv[2 * q], zv[2 * q + 1]),
                                               make_float2(yv[2 * q], yv[2 * q + 1]));
                        rr = __ffma2_rn(d2, make_float2(xv[2 * q], xv[2 * q + 1]), rr);
                        yv[2 * q] = rr.x;
                        yv[2 * q + 1] = rr.y;
                    }
                    co_nonfinite(yv, 16, nonfinite);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        *reinterpret_cast<float4 *>(stg + sw128_off(row, 4 * hh + q)) =
                            make_float4(yv[4 * q], yv[4 * q + 1], yv[4 * q + 2], yv[4 * q + 3]);
                }
            }
            co_arrive(S.bar(kBarFree0 + f), lane);
        }
        // an fp16 operand out of range (see co_form_wx) or a non-finite input
        if (__any_sync(0xffffffffu, !(nonfinite.x == 0.f && nonfinite.y == 0.f)) && lane == 0)
            flag_status(ws.status, kStatusRange);
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) {
        // let every copy and MMA already issued finish before the CTA
        // releases its shared memory and TMEM (bounded waits)
        for (int q = 0; q < kFirstComputeBar; ++q) {
            const int cnt = S.issued()[q];
            if (cnt) mbar_wait(S.bar(q), (uint32_t)((cnt - 1) & 1), wait_budget);
        }
        flag_status(ws.status, kStatusTimeout);
    }
    if (warp == 0) {
        __syncwarp();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace

namespace {
std::atomic<int> g_test_fault{0};
}  // namespace

void tc_set_test_fault(int kind) { g_test_fault.store(kind); }
int tc_test_fault() { return g_test_fault.load(); }

bool tc_supported(const ScanDims &d, int bf16) {
    if (!bf16 || d.N != kN || d.P != kP) return false;
    if (d.Q != 64 && d.Q != 128 && d.Q != 256) return false;
    if (d.H > 65535 || d.b > 65535 || d.L > 0x7fffffffll - kBlk) return false;
    const TcPlan p = make_plan(d);
    return p.U <= 65535 && (d.H + kPrepHeads - 1) / kPrepHeads + 4 * d.G <= 65535;
}

size_t tc_workspace_bytes(const ScanDims &d) { return ws_bytes(d, make_plan(d)); }

cudaError_t tc_scan(const ScanArgs &a, const ScanDims &d, void *wsp, cudaStream_t s) {
    const TcPlan p = make_plan(d);
    if (p.nblk == 0) return cudaSuccess;
    TcWs ws = carve(d, p, wsp);
    TcMaps maps;
    if (!make_maps(a, d, p, ws, &maps)) return cudaErrorInvalidValue;
    cudaError_t e;
    // the shared-memory limits are set once per device
    static bool attr_done[kMaxAttrDevices] = {};
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxAttrDevices) return cudaErrorInvalidDevice;
    if (!attr_done[dev]) {
        if ((e = cudaFuncSetAttribute(unit_state_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)UsLayout<false>::kSmem)) != cudaSuccess)
            return e;
        if ((e = cudaFuncSetAttribute(unit_state_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)UsLayout<true>::kSmem)) != cudaSuccess)
            return e;
        if ((e = cudaFuncSetAttribute(chunk_out_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)kCoSmem)) != cudaSuccess)
            return e;
        if ((e = cudaFuncSetAttribute(chunk_out_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)kCoSmem)) != cudaSuccess)
            return e;
        if ((e = cudaFuncSetAttribute(chunk_out_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)kCoSmem)) != cudaSuccess)
            return e;
        attr_done[dev] = true;
    }
    const bool conv = a.conv_w != nullptr;
    {
        TraceScope tr(s, kTrTcDtPrep);
        // a plain launch: it overwrites the workspace the previous call's kernels read
        // (combined arrangement: B and C come from xbc, through the conv)
        const unsigned ny = (unsigned)((d.H + kPrepHeads - 1) / kPrepHeads + 4 * d.G);
        auto prep = conv ? prep_kernel<true> : prep_kernel<false>;   // the split path compiles without the conv
        prep<<<dim3((unsigned)p.nblk, ny, (unsigned)d.b), 256, 0, s>>>(
            a.dt_raw, a.dt_bias, a.A, static_cast<const __nv_bfloat16 *>(conv ? a.x : a.B),
            static_cast<const __nv_bfloat16 *>(a.C), a.seq_idx, ws, (int)d.L, (int)d.H, (int)d.G, (int)p.nblk,
            a.dt_lo, a.dt_hi, a.conv_w, a.conv_b, (int)a.Cd);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // the kernels after prep may start their prologue while their predecessor
    // finishes; each waits (griddepcontrol.wait) before reading its outputs
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    auto cfg = [&](dim3 grid, unsigned threads, size_t smem) {
        cudaLaunchConfig_t c = {};
        c.gridDim = grid;
        c.blockDim = dim3(threads);
        c.dynamicSmemBytes = smem;
        c.stream = s;
        c.attrs = pdl;
        c.numAttrs = 1;
        return c;
    };
    if (p.U > 1) {
        {
            TraceScope tr(s, kTrTcUnitState);
            const cudaLaunchConfig_t c =
                cfg(dim3((unsigned)d.H, (unsigned)(p.U - 1), (unsigned)d.b), kUsThreads,
                    conv ? UsLayout<true>::kSmem : UsLayout<false>::kSmem);
            if ((e = cudaLaunchKernelEx(&c, conv ? unit_state_kernel<true> : unit_state_kernel<false>, maps, ws,
                                        (int)d.H, (int)d.G, (int)p.nblk, (int)p.U, (int)p.bpu, a.seq_idx ? 1 : 0,
                                        a.conv_w, a.conv_b)) != cudaSuccess)
                return e;
        }
        {
            TraceScope tr(s, kTrTcStatePass);
            const cudaLaunchConfig_t c = cfg(dim3(kNP / 4 / 256, (unsigned)d.H, (unsigned)d.b), 256, 0);
            if ((e = cudaLaunchKernelEx(&c, tc_state_pass_kernel, ws, a.init_state, (int)d.H, (int)p.U)) != cudaSuccess)
                return e;
        }
    }
    {
        TraceScope tr(s, kTrTcChunkOut);
        // C/B prefetch into L2 only pays when the call streams more x and y than
        // L2 holds: otherwise prep's fp16 copies are still there when read.
        const double streamed = (double)d.b * d.L * d.H * d.P * (2.0 + 4.0);
        const int prefetch_cb = streamed > kL2Bytes ? 1 : 0;
        const int fault = tc_test_fault();
        const cudaLaunchConfig_t c = cfg(dim3((unsigned)d.H, (unsigned)p.U, (unsigned)d.b), kCoThreads, kCoSmem);
        // the caller checked that chunk_states come with chunk_size a multiple of kBlk
        const int bpc = (int)(d.Q / kBlk) > 0 ? (int)(d.Q / kBlk) : 1;
        // the combined arrangement takes no packed rows (the caller checked)
        auto kern = conv ? chunk_out_kernel<false, true>
                         : (a.seq_idx ? chunk_out_kernel<true, false> : chunk_out_kernel<false, false>);
        if ((e = cudaLaunchKernelEx(&c, kern, maps, a.D, a.init_state, a.final_state, ws, (int)d.L, (int)d.H,
                                    (int)d.G, (int)p.nblk, (int)p.U, (int)p.bpu, p.U > 1 ? 1 : 0, prefetch_cb,
                                    a.chunk_states, bpc, (int)d.nc, fault ? kTestWaitBudget : kWaitBudget, fault,
                                    a.conv_w, a.conv_b)) != cudaSuccess)
            return e;
    }
    return cudaGetLastError();
}

}  // namespace ssd
