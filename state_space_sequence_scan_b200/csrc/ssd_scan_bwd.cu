// Backward of the chunked SSD scan on CUDA cores in fp32, deterministic.
//
// The pages note that the backward pass of the usual mamba kernels is not
// deterministic (HF transformers issue "mamba2 mixer different outputs",
// reply on the backward pass).  Here every output element has one owning
// thread and every sum runs in a fixed order: no atomics, so two runs on the
// same inputs give the same bits.
//
// The gradients of <dy, y> + <dfinal, final_state> follow the chunked form of
// the forward ("Mamba2" knowledge page: intra-chunk parallel, inter-chunk
// serial).  Within chunk c (local tokens 0..q-1, cum_i the inclusive cumsum
// of dt*A, cl = cum_{q-1}, H_in the entering state, G_c the gradient of the
// state after the chunk):
//   y_i   = sum_{j<=i} (C_i.B_j) e^{cum_i-cum_j} dt_j x_j + e^{cum_i} C_i^T H_in + D x_i
//   H_out = e^{cl} H_in + sum_j e^{cl-cum_j} dt_j B_j x_j^T
// so, with s_ij = dy_i.x_j and L_ij = e^{cum_i-cum_j} (j <= i):
//   G_{c-1} = e^{cl} G_c + sum_i e^{cum_i} C_i dy_i^T          (reverse state pass)
//   dx_j  = dt_j (sum_{i>=j} (C_i.B_j) L_ij dy_i + e^{cl-cum_j} G_c^T B_j) + D dy_j
//   dB_j  = dt_j (sum_{i>=j} L_ij s_ij C_i + e^{cl-cum_j} G_c x_j)
//   dC_i  = sum_{j<=i} L_ij dt_j s_ij B_j + e^{cum_i} H_in dy_i
//   d(dt_j) direct = sum_{i>=j} (C_i.B_j) L_ij s_ij + e^{cl-cum_j} B_j^T G_c x_j
//   d(cum_i): + sum_{j<i} M_ij + e^{cum_i} C_i^T H_in dy_i, - sum_{k>i} M_ki,
//             - E_i, and at i = q-1 also + sum_j E_j + e^{cl} <G_c, H_in>,
//     M_ij = (C_i.B_j) L_ij dt_j s_ij,  E_j = e^{cl-cum_j} dt_j B_j^T G_c x_j;
//   d(dA_k) = sum_{i>=k} d(cum_i),  d(dt_k) += A d(dA_k),  dA += sum_k dt_k d(dA_k);
//   dz_k = d(dt_k) softplus'(z_k) [dt_lo <= softplus(z_k) <= dt_hi] = d(dt_raw_k),
//   d(dt_bias) = sum_k dz_k,  dD = sum_t dy_t.x_t,  d(init_state) = G_{-1}.
// The heads of a group add their dB, dC in head order.
//
// Launches: the forward's state pass (dt, cum, entering states), then
//   1. dstate     per (chunk, head, batch): sum_i e^{cum_i} C_i dy_i^T
//   2. dpass      per (head, batch, state element): the reverse state pass,
//                 G_c in place of 1's output, partial <G_c, H_in> per block
//   3. cols       per (64-token j tile, chunk, head, batch): dx, dB, d(dt) direct,
//                 the column part of d(cum), E_j, dy_j.x_j
//   4. rows       per (64-token i tile, ...): dC and the row part of d(cum)
//   5. finalize   per (chunk, head, batch): d(dA) by a reverse block scan,
//                 d(dt_raw), per-chunk partials of dA, d(dt_bias), dD
//   6. heads      per head: the partials summed over (batch, chunk) in order
//   7. groups     dB, dC: the heads of each group summed in head order
#include "ssd_common.cuh"
#include "ssd_internal.h"
#include "ssd_trace.h"

namespace ssd {
namespace {

constexpr int kThreads = 256;
constexpr int kT = 64;        // tokens per tile in the pair kernels
constexpr int kTK = 32;       // tokens per smem tile in dstate
constexpr int kMaxAcc = 32;   // accumulators per thread in dstate
constexpr int kMaxP = 64, kMaxN = 128;

struct BwdWs {
    SimtWs f;          // forward: dtv, cum, ell, entering states
    float *gst;        // [b, H, nc, N, P]: 1's output, then G_c
    float *ghp;        // [b, H, nc, nblk * 8]: partial <G_c, H_in> per dpass warp
    float *ddt_dir;    // [b, H, L]
    float *dcum_col;   // [b, H, L]
    float *dcum_row;   // [b, H, L]
    float *E;          // [b, H, L]
    float *dyx;        // [b, H, L]: dy_t . x_t
    float *part;       // [b, H, nc, 3]: dA, d(dt_bias), dD per chunk
    float *dBh, *dCh;  // [b, L, H, N] per head (null when G == H)
    float *docc;       // [b, L] packed rows: document starts from the chunk's first token through t
};

int dpass_blocks(const ScanDims &d) { return (int)((d.N * d.P + kThreads - 1) / kThreads); }

size_t bwd_extra_bytes(const ScanDims &d, size_t *offs) {
    const size_t bh = (size_t)d.b * d.H;
    const size_t sizes[7] = {
        bh * d.nc * d.N * d.P * sizeof(float),
        bh * d.nc * dpass_blocks(d) * (kThreads / 32) * sizeof(float),
        bh * d.L * sizeof(float) * 5,
        bh * d.nc * 3 * sizeof(float),
        d.G == d.H ? 0 : (size_t)d.b * d.L * d.H * d.N * sizeof(float),
        d.G == d.H ? 0 : (size_t)d.b * d.L * d.H * d.N * sizeof(float),
        (size_t)d.b * d.L * sizeof(float)};
    size_t off = 0;
    for (int i = 0; i < 7; ++i) {
        if (offs) offs[i] = off;
        off += align256(sizes[i]);
    }
    return off;
}

BwdWs bwd_carve(const ScanDims &d, void *ws) {
    BwdWs w;
    w.f = simt_carve(d, ws);
    size_t offs[7];
    bwd_extra_bytes(d, offs);
    char *p = static_cast<char *>(ws) + simt_workspace_bytes(d);
    const size_t tok = (size_t)d.b * d.H * d.L;
    w.gst = reinterpret_cast<float *>(p + offs[0]);
    w.ghp = reinterpret_cast<float *>(p + offs[1]);
    float *t = reinterpret_cast<float *>(p + offs[2]);
    w.ddt_dir = t;
    w.dcum_col = t + tok;
    w.dcum_row = t + 2 * tok;
    w.E = t + 3 * tok;
    w.dyx = t + 4 * tok;
    w.part = reinterpret_cast<float *>(p + offs[3]);
    w.dBh = d.G == d.H ? nullptr : reinterpret_cast<float *>(p + offs[4]);
    w.dCh = d.G == d.H ? nullptr : reinterpret_cast<float *>(p + offs[5]);
    w.docc = reinterpret_cast<float *>(p + offs[6]);
    return w;
}

// Sum over the block, fixed order; every thread gets the total.
__device__ __forceinline__ float block_sum(float v, float *red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float t = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
    return t;
}

// ---- 0. packed rows: document counters per chunk ---------------------------
__global__ void __launch_bounds__(kThreads)
docs_kernel(const int32_t *__restrict__ seq_idx, float *__restrict__ docc, int L, int Q) {
    __shared__ float wtot[32];
    const int c = blockIdx.x, b = blockIdx.y;
    const int t0 = c * Q, q = min(Q, L - t0);
    float carry = 0.f;
    for (int base = 0; base < q; base += kThreads) {
        const int i = base + threadIdx.x;
        const int t = t0 + i;
        const float f = (i < q && t > 0 && seq_idx[(size_t)b * L + t] != seq_idx[(size_t)b * L + t - 1]) ? 1.f : 0.f;
        float tot;
        const float v = block_inclusive_scan(f, wtot, tot) + carry;
        if (i < q) docc[(size_t)b * L + t] = v;
        carry += tot;
    }
}

// ---- 1. sum_i e^{cum_i} C_i dy_i^T per chunk ------------------------------
template <typename T>
__global__ void __launch_bounds__(kThreads)
dstate_kernel(const T *__restrict__ Cm, const float *__restrict__ dy, BwdWs ws, int L, int H, int P, int N,
              int G, int Q, int nc, int packed) {
    extern __shared__ float sm[];
    float *s_C = sm;                 // kTK * N
    float *s_W = s_C + kTK * N;      // kTK * P
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int g = h / (H / G);
    const int t0 = c * Q, q = min(Q, L - t0);
    const size_t bh = (size_t)b * H + h;
    const int p = threadIdx.x % P, n0 = threadIdx.x / P, RN = kThreads / P;
    const int nacc = (N + RN - 1) / RN;
    float acc[kMaxAcc];
#pragma unroll
    for (int r = 0; r < kMaxAcc; ++r) acc[r] = 0.f;
    for (int k0 = 0; k0 < q; k0 += kTK) {
        const int kk = min(kTK, q - k0);
        __syncthreads();
        for (int e = threadIdx.x; e < kk * N; e += kThreads) {
            const int k = e / N, n = e - k * N;
            s_C[e] = to_f(Cm[(((size_t)b * L + t0 + k0 + k) * G + g) * N + n]);
        }
        for (int e = threadIdx.x; e < kk * P; e += kThreads) {
            const int k = e / P, pp = e - k * P;
            // packed rows: only the chunk's first document reads the entering state
            const bool first = !packed || ws.docc[(size_t)b * L + t0 + k0 + k] == 0.f;
            const float w = first ? expf(fminf(ws.f.cum[bh * L + t0 + k0 + k], 0.f)) : 0.f;
            s_W[e] = w * dy[(((size_t)b * L + t0 + k0 + k) * H + h) * P + pp];
        }
        __syncthreads();
        if (n0 < N) {
            for (int k = 0; k < kk; ++k) {
                const float wv = s_W[k * P + p];
                const float *crow = s_C + k * N + n0;
#pragma unroll
                for (int r = 0; r < kMaxAcc; ++r)
                    if (r < nacc && n0 + r * RN < N) acc[r] = fmaf(crow[r * RN], wv, acc[r]);
            }
        }
    }
    float *out = ws.gst + (bh * nc + c) * (size_t)N * P;
#pragma unroll
    for (int r = 0; r < kMaxAcc; ++r) {
        const int n = n0 + r * RN;
        if (r < nacc && n < N) out[(size_t)n * P + p] = acc[r];
    }
}

// ---- 2. reverse state pass --------------------------------------------------
// Thread = one state element, serial over chunks from the last; the inputs
// of kDpBatch chunks are loaded together before their steps run.  Each
// warp's share of <G_c, H_in> goes to its own slot (a shuffle tree, fixed
// order); finalize adds the slots in index order.
constexpr int kDpBatch = 8;
__global__ void __launch_bounds__(kThreads)
dpass_kernel(BwdWs ws, const float *__restrict__ dfinal, float *__restrict__ dinit, int H, int NP, int nc) {
    const int e = blockIdx.x * kThreads + threadIdx.x;
    const bool live = e < NP;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t bh = (size_t)blockIdx.z * H + blockIdx.y;
    const int nparts = gridDim.x * (kThreads / 32);
    float gcur = (live && dfinal) ? dfinal[bh * NP + e] : 0.f;
    for (int c1 = nc - 1; c1 >= 0; c1 -= kDpBatch) {
        float ds[kDpBatch], hin[kDpBatch], dec[kDpBatch];
#pragma unroll
        for (int k = 0; k < kDpBatch; ++k) {
            const int c = c1 - k;
            ds[k] = hin[k] = dec[k] = 0.f;
            if (c >= 0) {
                dec[k] = expf(fminf(ws.f.ell[bh * nc + c], 0.f));
                if (live) {
                    const size_t off = (bh * nc + c) * (size_t)NP + e;
                    ds[k] = ws.gst[off];
                    hin[k] = ws.f.states[off];
                }
            }
        }
#pragma unroll
        for (int k = 0; k < kDpBatch; ++k) {
            const int c = c1 - k;
            if (c < 0) break;                       // uniform over the block
            if (live) ws.gst[(bh * nc + c) * (size_t)NP + e] = gcur;   // gradient of the state after chunk c
            float v = gcur * hin[k];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0) ws.ghp[(bh * nc + c) * (size_t)nparts + blockIdx.x * (kThreads / 32) + warp] = v;
            gcur = fmaf(dec[k], gcur, ds[k]);
        }
    }
    if (live && dinit) dinit[bh * NP + e] = gcur;
}

// ---- 3/4. pair kernels ------------------------------------------------------
// Tile-map: thread (ig = tid/16, jg = tid%16) owns pair-tile entries
// (ig + 16a, jg + 16b), a, b < 4.  Acc-map: thread (r0 = tid/8, pc = tid%8)
// owns rows r0, r0+32 and columns pc + 8k.  smem rows are padded by one
// float so the column walks hit distinct banks.

// cb[a][b] = C_i . B_j (N long), sx[a][b] = dy_i . x_j (P long) for the thread's 4x4 entries
__device__ __forceinline__ void pair_dots(const float *sC, const float *sB, int ldn, const float *sDY,
                                          const float *sX, int ldp, int N, int P, int ig, int jg,
                                          float cb[4][4], float sx[4][4]) {
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) cb[a][b] = sx[a][b] = 0.f;
    for (int n = 0; n < N; ++n) {
        float cv[4], bv[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) cv[a] = sC[(ig + 16 * a) * ldn + n];
#pragma unroll
        for (int b = 0; b < 4; ++b) bv[b] = sB[(jg + 16 * b) * ldn + n];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) cb[a][b] = fmaf(cv[a], bv[b], cb[a][b]);
    }
    for (int p = 0; p < P; ++p) {
        float dv[4], xv[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) dv[a] = sDY[(ig + 16 * a) * ldp + p];
#pragma unroll
        for (int b = 0; b < 4; ++b) xv[b] = sX[(jg + 16 * b) * ldp + p];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) sx[a][b] = fmaf(dv[a], xv[b], sx[a][b]);
    }
}

size_t cols_smem(const ScanDims &d) {
    const size_t ldn = d.N + 1, ldp = d.P + 1;
    return sizeof(float) * (2 * kT * ldn + 2 * kT * ldp + 2 * kT * (kT + 1) + 2 * 16 * kT + 8 * kT);
}

size_t rows_smem(const ScanDims &d) {
    const size_t ldn = d.N + 1, ldp = d.P + 1;
    return sizeof(float) * (2 * kT * ldn + 2 * kT * ldp + kT * (kT + 1) + 7 * kT);
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
cols_kernel(const T *__restrict__ x, const T *__restrict__ Bm, const T *__restrict__ Cm,
            const float *__restrict__ D, const float *__restrict__ dy, BwdWs ws, float *__restrict__ dx,
            float *__restrict__ dB, int L, int H, int P, int N, int G, int Q, int nc, int packed) {
    extern __shared__ float sm[];
    const int ldn = N + 1, ldp = P + 1;
    float *sB = sm;                        // kT x ldn   (j tile)
    float *sX = sB + kT * ldn;             // kT x ldp   (j tile)
    float *sC = sX + kT * ldp;             // kT x ldn   (i tile); G_c [N x ldp] in the state phase
    float *sDY = sC + kT * ldn;            // kT x ldp   (i tile)
    float *sU = sDY + kT * ldp;            // kT x (kT+1): (C_i.B_j) L_ij, [i][j]
    float *sV = sU + kT * (kT + 1);        // kT x (kT+1): s_ij L_ij
    float *sZ = sV + kT * (kT + 1);        // 16 x kT: column partials of (C.B) L s, all i >= j
    float *sZo = sZ + 16 * kT;             // 16 x kT: the same, i > j
    float *s_cumj = sZo + 16 * kT;
    float *s_dtj = s_cumj + kT;
    float *s_cumi = s_dtj + kT;
    float *s_dst = s_cumi + kT;            // d(dt_j) from the state term
    float *s_E = s_dst + kT;               // E_j
    float *s_dyx = s_E + kT;               // dy_j . x_j
    float *s_docj = s_dyx + kT;            // packed rows: document counters of the j tile
    float *s_doci = s_docj + kT;           // and of the i tile

    const int tiles = (Q + kT - 1) / kT;
    const int c = blockIdx.x / tiles, jt = blockIdx.x - c * tiles;
    const int h = blockIdx.y, b = blockIdx.z;
    const int g = h / (H / G);
    const int t0 = c * Q, q = min(Q, L - t0);
    const int j0 = jt * kT;
    if (j0 >= q) return;                   // uniform over the block
    const int tj = min(kT, q - j0);
    const size_t bh = (size_t)b * H + h;
    const int tid = threadIdx.x;
    const int ig = tid >> 4, jg = tid & 15;
    const int r0 = tid >> 3, pc = tid & 7;
    const int PK = P / 8, NK = N / 8;

    // j tile: B_j, x_j, cum_j, dt_j
    for (int e = tid; e < kT * N; e += kThreads) {
        const int r = e / N, n = e - r * N;
        sB[r * ldn + n] = r < tj ? to_f(Bm[(((size_t)b * L + t0 + j0 + r) * G + g) * N + n]) : 0.f;
    }
    for (int e = tid; e < kT * P; e += kThreads) {
        const int r = e / P, p = e - r * P;
        sX[r * ldp + p] = r < tj ? to_f(x[(((size_t)b * L + t0 + j0 + r) * H + h) * P + p]) : 0.f;
    }
    const float cl = ws.f.cum[bh * L + t0 + q - 1];
    const float dl = packed ? ws.docc[(size_t)b * L + t0 + q - 1] : 0.f;
    for (int r = tid; r < kT; r += kThreads) {
        s_cumj[r] = r < tj ? ws.f.cum[bh * L + t0 + j0 + r] : 0.f;
        s_dtj[r] = r < tj ? ws.f.dtv[bh * L + t0 + j0 + r] : 0.f;
        s_docj[r] = (packed && r < tj) ? ws.docc[(size_t)b * L + t0 + j0 + r] : 0.f;
    }
    // G_c, the gradient of the state after this chunk
    float *sG = sC;
    const float *Gc = ws.gst + (bh * nc + c) * (size_t)N * P;
    for (int e = tid; e < N * P; e += kThreads) {
        const int n = e / P, p = e - n * P;
        sG[n * ldp + p] = Gc[e];
    }
    __syncthreads();

    // state phase: adx = G_c^T B_j, adb = G_c x_j (scaled by e^{cl-cum_j} below)
    float adx[2][kMaxP / 8], adb[2][kMaxN / 8];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
#pragma unroll
        for (int k = 0; k < kMaxP / 8; ++k) adx[r][k] = 0.f;
#pragma unroll
        for (int k = 0; k < kMaxN / 8; ++k) adb[r][k] = 0.f;
    }
    for (int n = 0; n < N; ++n) {
        const float b0 = sB[r0 * ldn + n], b1 = sB[(r0 + 32) * ldn + n];
#pragma unroll
        for (int k = 0; k < kMaxP / 8; ++k)
            if (k < PK) {
                const float gv = sG[n * ldp + pc + 8 * k];
                adx[0][k] = fmaf(b0, gv, adx[0][k]);
                adx[1][k] = fmaf(b1, gv, adx[1][k]);
            }
    }
    for (int p = 0; p < P; ++p) {
        const float x0 = sX[r0 * ldp + p], x1 = sX[(r0 + 32) * ldp + p];
#pragma unroll
        for (int k = 0; k < kMaxN / 8; ++k)
            if (k < NK) {
                const float gv = sG[(pc + 8 * k) * ldp + p];
                adb[0][k] = fmaf(x0, gv, adb[0][k]);
                adb[1][k] = fmaf(x1, gv, adb[1][k]);
            }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int jj = r0 + 32 * r;
        float e1 = 0.f;                    // B_j^T G_c x_j
#pragma unroll
        for (int k = 0; k < kMaxN / 8; ++k)
            if (k < NK) e1 = fmaf(sB[jj * ldn + pc + 8 * k], adb[r][k], e1);
        e1 += __shfl_xor_sync(0xffffffffu, e1, 1);
        e1 += __shfl_xor_sync(0xffffffffu, e1, 2);
        e1 += __shfl_xor_sync(0xffffffffu, e1, 4);
        // packed rows: only the chunk's last document writes into the state it passes on
        const float dec = (jj < tj && s_docj[jj] == dl) ? expf(fminf(cl - s_cumj[jj], 0.f)) : 0.f;
#pragma unroll
        for (int k = 0; k < kMaxP / 8; ++k) adx[r][k] *= dec;
#pragma unroll
        for (int k = 0; k < kMaxN / 8; ++k) adb[r][k] *= dec;
        if (pc == 0) {
            s_dst[jj] = dec * e1;
            s_E[jj] = s_dtj[jj] * dec * e1;
        }
    }

    // intra-chunk part: i tiles from this one to the chunk's end
    float zs = 0.f, zo = 0.f;              // column sums, owned by tid < kT
    for (int i0 = j0; i0 < q; i0 += kT) {
        const int ti = min(kT, q - i0);
        __syncthreads();                   // sG / previous tile no longer read
        for (int e = tid; e < kT * N; e += kThreads) {
            const int r = e / N, n = e - r * N;
            sC[r * ldn + n] = r < ti ? to_f(Cm[(((size_t)b * L + t0 + i0 + r) * G + g) * N + n]) : 0.f;
        }
        for (int e = tid; e < kT * P; e += kThreads) {
            const int r = e / P, p = e - r * P;
            sDY[r * ldp + p] = r < ti ? dy[(((size_t)b * L + t0 + i0 + r) * H + h) * P + p] : 0.f;
        }
        for (int r = tid; r < kT; r += kThreads) {
            s_cumi[r] = r < ti ? ws.f.cum[bh * L + t0 + i0 + r] : 0.f;
            s_doci[r] = (packed && r < ti) ? ws.docc[(size_t)b * L + t0 + i0 + r] : 0.f;
        }
        __syncthreads();
        if (i0 == j0) {                    // the diagonal tile: dy_j . x_j
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int jj = r0 + 32 * r;
                float v = 0.f;
#pragma unroll
                for (int k = 0; k < kMaxP / 8; ++k)
                    if (k < PK) v = fmaf(sX[jj * ldp + pc + 8 * k], sDY[jj * ldp + pc + 8 * k], v);
                v += __shfl_xor_sync(0xffffffffu, v, 1);
                v += __shfl_xor_sync(0xffffffffu, v, 2);
                v += __shfl_xor_sync(0xffffffffu, v, 4);
                if (pc == 0) s_dyx[jj] = v;
            }
        }
        float cb[4][4], sx[4][4];
        pair_dots(sC, sB, ldn, sDY, sX, ldp, N, P, ig, jg, cb, sx);
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) {
            const int jj = jg + 16 * bb;
            float za = 0.f, zb = 0.f;
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int ii = ig + 16 * a;
                const bool ok = ii < ti && jj < tj && i0 + ii >= j0 + jj && s_doci[ii] == s_docj[jj];
                const float lw = ok ? expf(fminf(s_cumi[ii] - s_cumj[jj], 0.f)) : 0.f;
                const float u = cb[a][bb] * lw, v = sx[a][bb] * lw;
                sU[ii * (kT + 1) + jj] = u;
                sV[ii * (kT + 1) + jj] = v;
                const float z = u * sx[a][bb];
                za += z;
                zb += (i0 + ii > j0 + jj) ? z : 0.f;
            }
            sZ[ig * kT + jj] = za;
            sZo[ig * kT + jj] = zb;
        }
        __syncthreads();
        for (int ii = 0; ii < ti; ++ii) {
            const float u0 = sU[ii * (kT + 1) + r0], u1 = sU[ii * (kT + 1) + r0 + 32];
            const float v0 = sV[ii * (kT + 1) + r0], v1 = sV[ii * (kT + 1) + r0 + 32];
#pragma unroll
            for (int k = 0; k < kMaxP / 8; ++k)
                if (k < PK) {
                    const float dv = sDY[ii * ldp + pc + 8 * k];
                    adx[0][k] = fmaf(u0, dv, adx[0][k]);
                    adx[1][k] = fmaf(u1, dv, adx[1][k]);
                }
#pragma unroll
            for (int k = 0; k < kMaxN / 8; ++k)
                if (k < NK) {
                    const float cv = sC[ii * ldn + pc + 8 * k];
                    adb[0][k] = fmaf(v0, cv, adb[0][k]);
                    adb[1][k] = fmaf(v1, cv, adb[1][k]);
                }
        }
        if (tid < kT) {
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                zs += sZ[k * kT + tid];
                zo += sZo[k * kT + tid];
            }
        }
    }
    __syncthreads();

    const float Dh = D[h];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int jj = r0 + 32 * r;
        if (jj < tj) {
            const float dtj = s_dtj[jj];
            const size_t tok = (size_t)b * L + t0 + j0 + jj;
#pragma unroll
            for (int k = 0; k < kMaxP / 8; ++k)
                if (k < PK) {
                    const size_t off = (tok * H + h) * P + pc + 8 * k;
                    dx[off] = fmaf(dtj, adx[r][k], Dh * dy[off]);
                }
#pragma unroll
            for (int k = 0; k < kMaxN / 8; ++k)
                if (k < NK) dB[(tok * H + h) * N + pc + 8 * k] = dtj * adb[r][k];
        }
    }
    if (tid < tj) {
        const size_t o = bh * L + t0 + j0 + tid;
        ws.ddt_dir[o] = s_dst[tid] + zs;
        ws.dcum_col[o] = -(s_dtj[tid] * zo) - s_E[tid];
        ws.E[o] = s_E[tid];
        ws.dyx[o] = s_dyx[tid];
    }
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
rows_kernel(const T *__restrict__ x, const T *__restrict__ Bm, const T *__restrict__ Cm,
            const float *__restrict__ dy, BwdWs ws, float *__restrict__ dC, int L, int H, int P, int N, int G,
            int Q, int nc, int packed) {
    extern __shared__ float sm[];
    const int ldn = N + 1, ldp = P + 1;
    float *sC = sm;                        // kT x ldn   (i tile)
    float *sDY = sC + kT * ldn;            // kT x ldp   (i tile)
    float *sB = sDY + kT * ldp;            // kT x ldn   (j tile); H_in [N x ldp] in the state phase
    float *sX = sB + kT * ldn;             // kT x ldp   (j tile)
    float *sV = sX + kT * ldp;             // kT x (kT+1): L_ij dt_j s_ij, [i][j]
    float *s_cumi = sV + kT * (kT + 1);
    float *s_cumj = s_cumi + kT;
    float *s_dtj = s_cumj + kT;
    float *s_T = s_dtj + kT;               // e^{cum_i} C_i^T H_in dy_i
    float *s_rs = s_T + kT;                // sum_{j<i} M_ij
    float *s_doci = s_rs + kT;             // packed rows: document counters of the i tile
    float *s_docj = s_doci + kT;           // and of the j tile

    const int tiles = (Q + kT - 1) / kT;
    const int c = blockIdx.x / tiles, it = blockIdx.x - c * tiles;
    const int h = blockIdx.y, b = blockIdx.z;
    const int g = h / (H / G);
    const int t0 = c * Q, q = min(Q, L - t0);
    const int i0 = it * kT;
    if (i0 >= q) return;                   // uniform over the block
    const int ti = min(kT, q - i0);
    const size_t bh = (size_t)b * H + h;
    const int tid = threadIdx.x;
    const int ig = tid >> 4, jg = tid & 15;
    const int r0 = tid >> 3, pc = tid & 7;
    const int NK = N / 8;

    for (int e = tid; e < kT * N; e += kThreads) {
        const int r = e / N, n = e - r * N;
        sC[r * ldn + n] = r < ti ? to_f(Cm[(((size_t)b * L + t0 + i0 + r) * G + g) * N + n]) : 0.f;
    }
    for (int e = tid; e < kT * P; e += kThreads) {
        const int r = e / P, p = e - r * P;
        sDY[r * ldp + p] = r < ti ? dy[(((size_t)b * L + t0 + i0 + r) * H + h) * P + p] : 0.f;
    }
    for (int r = tid; r < kT; r += kThreads) {
        s_cumi[r] = r < ti ? ws.f.cum[bh * L + t0 + i0 + r] : 0.f;
        s_doci[r] = (packed && r < ti) ? ws.docc[(size_t)b * L + t0 + i0 + r] : 0.f;
    }
    float *sH = sB;
    const float *Hin = ws.f.states + (bh * nc + c) * (size_t)N * P;
    for (int e = tid; e < N * P; e += kThreads) {
        const int n = e / P, p = e - n * P;
        sH[n * ldp + p] = Hin[e];
    }
    __syncthreads();

    // state phase: adc = H_in dy_i, scaled by e^{cum_i}
    float adc[2][kMaxN / 8];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int k = 0; k < kMaxN / 8; ++k) adc[r][k] = 0.f;
    for (int p = 0; p < P; ++p) {
        const float d0 = sDY[r0 * ldp + p], d1 = sDY[(r0 + 32) * ldp + p];
#pragma unroll
        for (int k = 0; k < kMaxN / 8; ++k)
            if (k < NK) {
                const float hv = sH[(pc + 8 * k) * ldp + p];
                adc[0][k] = fmaf(d0, hv, adc[0][k]);
                adc[1][k] = fmaf(d1, hv, adc[1][k]);
            }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int ii = r0 + 32 * r;
        float tv = 0.f;
#pragma unroll
        for (int k = 0; k < kMaxN / 8; ++k)
            if (k < NK) tv = fmaf(sC[ii * ldn + pc + 8 * k], adc[r][k], tv);
        tv += __shfl_xor_sync(0xffffffffu, tv, 1);
        tv += __shfl_xor_sync(0xffffffffu, tv, 2);
        tv += __shfl_xor_sync(0xffffffffu, tv, 4);
        // packed rows: the entering state reaches only the chunk's first document
        const float dec = (ii < ti && s_doci[ii] == 0.f) ? expf(fminf(s_cumi[ii], 0.f)) : 0.f;
#pragma unroll
        for (int k = 0; k < kMaxN / 8; ++k) adc[r][k] *= dec;
        if (pc == 0) s_T[ii] = dec * tv;
    }

    float rsum[4] = {0.f, 0.f, 0.f, 0.f};  // row sums of M over j < i, owned by jg == 0
    for (int j0 = 0; j0 <= i0; j0 += kT) {
        const int tj = min(kT, q - j0);
        __syncthreads();                   // sH / previous tile no longer read
        for (int e = tid; e < kT * N; e += kThreads) {
            const int r = e / N, n = e - r * N;
            sB[r * ldn + n] = r < tj ? to_f(Bm[(((size_t)b * L + t0 + j0 + r) * G + g) * N + n]) : 0.f;
        }
        for (int e = tid; e < kT * P; e += kThreads) {
            const int r = e / P, p = e - r * P;
            sX[r * ldp + p] = r < tj ? to_f(x[(((size_t)b * L + t0 + j0 + r) * H + h) * P + p]) : 0.f;
        }
        for (int r = tid; r < kT; r += kThreads) {
            s_cumj[r] = r < tj ? ws.f.cum[bh * L + t0 + j0 + r] : 0.f;
            s_dtj[r] = r < tj ? ws.f.dtv[bh * L + t0 + j0 + r] : 0.f;
            s_docj[r] = (packed && r < tj) ? ws.docc[(size_t)b * L + t0 + j0 + r] : 0.f;
        }
        __syncthreads();
        float cb[4][4], sx[4][4];
        pair_dots(sC, sB, ldn, sDY, sX, ldp, N, P, ig, jg, cb, sx);
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const int ii = ig + 16 * a;
            float m = 0.f;
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) {
                const int jj = jg + 16 * bb;
                const bool ok = ii < ti && jj < tj && i0 + ii >= j0 + jj && s_doci[ii] == s_docj[jj];
                const float v = ok ? sx[a][bb] * expf(fminf(s_cumi[ii] - s_cumj[jj], 0.f)) * s_dtj[jj] : 0.f;
                sV[ii * (kT + 1) + jj] = v;
                m += (i0 + ii > j0 + jj) ? cb[a][bb] * v : 0.f;
            }
            m += __shfl_xor_sync(0xffffffffu, m, 1);
            m += __shfl_xor_sync(0xffffffffu, m, 2);
            m += __shfl_xor_sync(0xffffffffu, m, 4);
            m += __shfl_xor_sync(0xffffffffu, m, 8);
            rsum[a] += m;
        }
        __syncthreads();
        for (int jj = 0; jj < tj; ++jj) {
            const float v0 = sV[r0 * (kT + 1) + jj], v1 = sV[(r0 + 32) * (kT + 1) + jj];
#pragma unroll
            for (int k = 0; k < kMaxN / 8; ++k)
                if (k < NK) {
                    const float bv = sB[jj * ldn + pc + 8 * k];
                    adc[0][k] = fmaf(v0, bv, adc[0][k]);
                    adc[1][k] = fmaf(v1, bv, adc[1][k]);
                }
        }
    }
    if (jg == 0) {
#pragma unroll
        for (int a = 0; a < 4; ++a) s_rs[ig + 16 * a] = rsum[a];
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int ii = r0 + 32 * r;
        if (ii < ti) {
            const size_t tok = (size_t)b * L + t0 + i0 + ii;
#pragma unroll
            for (int k = 0; k < kMaxN / 8; ++k)
                if (k < NK) dC[(tok * H + h) * N + pc + 8 * k] = adc[r][k];
        }
    }
    if (tid < ti) ws.dcum_row[bh * L + t0 + i0 + tid] = s_T[tid] + s_rs[tid];
}

// ---- 5. per chunk: d(dA) by a reverse scan, d(dt_raw), partials --------------
__global__ void __launch_bounds__(kThreads)
finalize_kernel(const float *__restrict__ dt_raw, const float *__restrict__ dt_bias, const float *__restrict__ A,
                BwdWs ws, float *__restrict__ ddt_raw, int L, int H, int Q, int nc, int nblk, float lo,
                float hi) {
    __shared__ float red[32], wtot[32];     // block_sum and the scan keep separate scratch
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int t0 = c * Q, q = min(Q, L - t0);
    const size_t bh = (size_t)b * H + h;
    const float Ah = A[h], bias = dt_bias[h];
    // the chunk's last token also carries sum_j E_j + e^{cl} <G_c, H_in>
    float e_part = 0.f;
    for (int i = threadIdx.x; i < q; i += kThreads) e_part += ws.E[bh * L + t0 + i];
    const float etot = block_sum(e_part, red);
    // the reverse pass's per-warp partials of <G_c, H_in>, in a fixed order
    const int nparts = nblk * (kThreads / 32);
    float g_part = 0.f;
    for (int k = threadIdx.x; k < nparts; k += kThreads) g_part += ws.ghp[(bh * nc + c) * (size_t)nparts + k];
    const float gh = block_sum(g_part, red);
    const float extra = etot + expf(fminf(ws.f.ell[bh * nc + c], 0.f)) * gh;

    float carry = 0.f, pa = 0.f, pb = 0.f, pd = 0.f;
    for (int base = 0; base < q; base += kThreads) {
        const int i = q - 1 - (base + (int)threadIdx.x);     // reverse order
        float v = 0.f;
        if (i >= 0) {
            const size_t o = bh * L + t0 + i;
            v = ws.dcum_row[o] + ws.dcum_col[o] + (i == q - 1 ? extra : 0.f);
        }
        float tot;
        const float dda = block_inclusive_scan(v, wtot, tot) + carry;   // sum_{k >= i} d(cum_k)
        carry += tot;
        if (i >= 0) {
            const size_t o = bh * L + t0 + i;
            const float dt = ws.f.dtv[o];
            const float ddt = fmaf(Ah, dda, ws.ddt_dir[o]);
            const float z = dt_raw[((size_t)b * L + t0 + i) * H + h] + bias;
            const float sp = softplus_f(z);
            const float sg = z >= 0.f ? 1.f / (1.f + expf(-z)) : expf(z) / (1.f + expf(z));
            const float dz = (sp >= lo && sp <= hi) ? ddt * sg : 0.f;
            ddt_raw[((size_t)b * L + t0 + i) * H + h] = dz;
            pa = fmaf(dt, dda, pa);
            pb += dz;
            pd += ws.dyx[o];
        }
    }
    pa = block_sum(pa, red);
    pb = block_sum(pb, red);
    pd = block_sum(pd, red);
    if (threadIdx.x == 0) {
        float *o = ws.part + (bh * nc + c) * 3;
        o[0] = pa;
        o[1] = pb;
        o[2] = pd;
    }
}

// ---- 6. per head: partials summed over (batch, chunk) -----------------------
__global__ void __launch_bounds__(kThreads)
heads_kernel(BwdWs ws, float *__restrict__ dA, float *__restrict__ ddt_bias, float *__restrict__ dD, int b,
             int H, int nc) {
    __shared__ float red[32];
    const int h = blockIdx.x;
    float s[3] = {0.f, 0.f, 0.f};
    const int n = b * nc;
    for (int k = threadIdx.x; k < n; k += kThreads) {
        const int bi = k / nc, c = k - bi * nc;
        const float *o = ws.part + (((size_t)bi * H + h) * nc + c) * 3;
        s[0] += o[0];
        s[1] += o[1];
        s[2] += o[2];
    }
    const float a = block_sum(s[0], red), t = block_sum(s[1], red), d = block_sum(s[2], red);
    if (threadIdx.x == 0) {
        dA[h] = a;
        ddt_bias[h] = t;
        dD[h] = d;
    }
}

// ---- 7. dB, dC: the heads of each group in head order -----------------------
__global__ void __launch_bounds__(kThreads)
groups_kernel(const float *__restrict__ dBh, const float *__restrict__ dC_h, float *__restrict__ dB,
              float *__restrict__ dC, int64_t total, int H, int G, int N) {
    // 4 consecutive state elements per thread (N % 8 == 0); the heads of the
    // group are added in head order, the loads of 8 heads issued together
    const int hpg = H / G;
    const int64_t total4 = total / 4;
    for (int64_t e4 = blockIdx.x * (int64_t)kThreads + threadIdx.x; e4 < total4;
         e4 += (int64_t)gridDim.x * kThreads) {
        const int64_t e = 4 * e4;
        const int64_t n = e % N, r = e / N;          // r = (b*L + t)*G + g
        const int64_t g = r % G, tok = r / G;
        const size_t src = ((size_t)tok * H + g * hpg) * N + n;
        float4 sb = make_float4(0.f, 0.f, 0.f, 0.f), sc = sb;
        for (int k0 = 0; k0 < hpg; k0 += 8) {
            float4 vb[8], vc[8];
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (k0 + k < hpg) {
                    vb[k] = *reinterpret_cast<const float4 *>(dBh + src + (size_t)(k0 + k) * N);
                    vc[k] = *reinterpret_cast<const float4 *>(dC_h + src + (size_t)(k0 + k) * N);
                }
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (k0 + k < hpg) {
                    sb.x += vb[k].x; sb.y += vb[k].y; sb.z += vb[k].z; sb.w += vb[k].w;
                    sc.x += vc[k].x; sc.y += vc[k].y; sc.z += vc[k].z; sc.w += vc[k].w;
                }
        }
        *reinterpret_cast<float4 *>(dB + e) = sb;
        *reinterpret_cast<float4 *>(dC + e) = sc;
    }
}

template <typename T>
cudaError_t run(const BwdArgs &a, const ScanDims &d, void *wsp, cudaStream_t s) {
    BwdWs ws = bwd_carve(d, wsp);
    cudaError_t e;
    const size_t smd = sizeof(float) * (size_t)kTK * (d.N + d.P);
    const size_t smc = cols_smem(d), smr = rows_smem(d);
    if ((e = cudaFuncSetAttribute(dstate_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smd)) !=
        cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(cols_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smc)) !=
        cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(rows_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smr)) !=
        cudaSuccess)
        return e;
    const int L = (int)d.L, H = (int)d.H, P = (int)d.P, N = (int)d.N, G = (int)d.G, Q = (int)d.Q;
    const int nc = (int)d.nc, NP = N * P;
    const dim3 gc((unsigned)nc, (unsigned)H, (unsigned)d.b);
    const int packed = a.f.seq_idx ? 1 : 0;
    if (a.tensor) {
        // the chunk states and the per-chunk dy sums on the tensor cores
        // (ssd_scan_bwd_tc.cu), then the forward's state pass
        if (packed) {
            docs_kernel<<<dim3((unsigned)nc, (unsigned)d.b), kThreads, 0, s>>>(a.f.seq_idx, ws.docc, L, Q);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
        BwdStatesArgs sa;
        sa.x = a.f.x; sa.B = a.f.B; sa.C = a.f.C; sa.dt_raw = a.f.dt_raw; sa.dt_bias = a.f.dt_bias; sa.A = a.f.A;
        sa.dy = a.dy; sa.dt_lo = a.f.dt_lo; sa.dt_hi = a.f.dt_hi; sa.dtv = ws.f.dtv; sa.cum = ws.f.cum;
        sa.ell = ws.f.ell; sa.states = ws.f.states; sa.gst = ws.gst; sa.status = ws.f.status;
        sa.docc = packed ? ws.docc : nullptr;
        if ((e = bwd_tc_states(sa, d, s)) != cudaSuccess) return e;
        if ((e = simt_state_pass(a.f, d, wsp, s)) != cudaSuccess) return e;
    } else {
        if ((e = simt_scan_states(a.f, d, wsp, s)) != cudaSuccess) return e;
        if (packed) {
            docs_kernel<<<dim3((unsigned)nc, (unsigned)d.b), kThreads, 0, s>>>(a.f.seq_idx, ws.docc, L, Q);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
        {
            TraceScope tr(s, kTrBwdDstate);
            dstate_kernel<T><<<gc, kThreads, smd, s>>>((const T *)a.f.C, a.dy, ws, L, H, P, N, G, Q, nc, packed);
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    const int nblk = dpass_blocks(d);
    {
        TraceScope tr(s, kTrBwdDpass);
        dpass_kernel<<<dim3((unsigned)nblk, (unsigned)H, (unsigned)d.b), kThreads, 0, s>>>(ws, a.dfinal, a.dinit,
                                                                                         H, NP, nc);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int tiles = (Q + kT - 1) / kT;
    const dim3 gp((unsigned)(nc * tiles), (unsigned)H, (unsigned)d.b);
    float *dBh = ws.dBh ? ws.dBh : a.dB;
    float *dCh = ws.dCh ? ws.dCh : a.dC;
    if (a.tensor) {
        // the pair products on the tensor cores (ssd_scan_bwd_tc.cu)
        BwdPairArgs pa;
        pa.x = a.f.x; pa.B = a.f.B; pa.C = a.f.C; pa.D = a.f.D; pa.dy = a.dy;
        pa.dtv = ws.f.dtv; pa.cum = ws.f.cum; pa.gst = ws.gst; pa.states = ws.f.states;
        pa.ddt_dir = ws.ddt_dir; pa.dcum_col = ws.dcum_col; pa.dcum_row = ws.dcum_row; pa.E = ws.E;
        pa.dyx = ws.dyx; pa.dx = a.dx; pa.dBh = dBh; pa.dCh = dCh; pa.status = ws.f.status;
        pa.docc = packed ? ws.docc : nullptr;
        if ((e = bwd_tc_pairs(pa, d, s)) != cudaSuccess) return e;
    } else {
    {
        TraceScope tr(s, kTrBwdCols);
        cols_kernel<T><<<gp, kThreads, smc, s>>>((const T *)a.f.x, (const T *)a.f.B, (const T *)a.f.C, a.f.D,
                                                 a.dy, ws, a.dx, dBh, L, H, P, N, G, Q, nc, packed);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    {
        TraceScope tr(s, kTrBwdRows);
        rows_kernel<T><<<gp, kThreads, smr, s>>>((const T *)a.f.x, (const T *)a.f.B, (const T *)a.f.C, a.dy, ws,
                                                 dCh, L, H, P, N, G, Q, nc, packed);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        TraceScope tr(s, kTrBwdFinalize);
        finalize_kernel<<<gc, kThreads, 0, s>>>(a.f.dt_raw, a.f.dt_bias, a.f.A, ws, a.ddt_raw, L, H, Q, nc, nblk,
                                                a.f.dt_lo, a.f.dt_hi);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    {
        TraceScope tr(s, kTrBwdReduce);
        heads_kernel<<<(unsigned)H, kThreads, 0, s>>>(ws, a.dA, a.ddt_bias, a.dD, (int)d.b, H, nc);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        if (ws.dBh) {
            const int64_t total = d.b * d.L * d.G * d.N;
            const int64_t blocks = (total / 4 + kThreads - 1) / kThreads;
            groups_kernel<<<(unsigned)(blocks < 148 * 16 ? blocks : 148 * 16), kThreads, 0, s>>>(
                ws.dBh, ws.dCh, a.dB, a.dC, total, H, G, N);
        }
    }
    return cudaGetLastError();
}

}  // namespace

bool bwd_supported(const ScanDims &d) {
    if (!simt_supported(d)) return false;
    if (d.P != 8 && d.P != 16 && d.P != 32 && d.P != 64) return false;
    if (d.N < 8 || d.N > kMaxN || d.N % 8 != 0) return false;
    if (d.nc * ((d.Q + kT - 1) / kT) > 0x7fffffff) return false;
    return cols_smem(d) <= 227 * 1024 && rows_smem(d) <= 227 * 1024;
}

size_t bwd_workspace_bytes(const ScanDims &d) { return simt_workspace_bytes(d) + bwd_extra_bytes(d, nullptr); }

cudaError_t bwd_scan(const BwdArgs &a, const ScanDims &d, void *ws, cudaStream_t s) {
    return a.f.bf16 ? run<__nv_bfloat16>(a, d, ws, s) : run<float>(a, d, ws, s);
}

}  // namespace ssd
