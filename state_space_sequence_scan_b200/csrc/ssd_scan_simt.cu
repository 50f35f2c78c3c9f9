// Chunked SSD forward scan on CUDA cores in fp32: the general path (any
// chunk size >= 1, fp32 or bf16 inputs, head_dim dividing 256,
// state_dim * head_dim <= 8192).
//
// The chunked form ("Mamba2" knowledge page: intra-chunk parallel, inter-chunk
// serial) in three launches:
//   1. chunk_state  per (chunk c, head h, batch b): dt = clamp(softplus(.)),
//      the within-chunk inclusive cumsum cum of dA = dt*A (block scan, fixed
//      order), and the chunk state
//         S_c = sum_j exp(cum_last - cum_j) dt_j B_j x_j^T      [N x P]
//   2. state_pass   per (b, h, state element): serial over chunks,
//         H_{-1} = init (or 0),   H_c = exp(cum_last(c)) H_{c-1} + S_c;
//      the state entering each chunk overwrites S_c, final_state = H_{nc-1}
//      (nnterp guide "Mamba-2", "The state after every token": one cumulative
//      step from the initial state through every chunk boundary).
//   3. chunk_out    per (b, h, chunk, tile of rows i):
//         y_i = sum_{j<=i in chunk} (C_i . B_j) exp(cum_i - cum_j) dt_j x_j
//             + exp(cum_i) C_i^T H_{c-1} + D x_i
// Every exponent is taken on min(cum_i - cum_j, 0) after the j <= i select,
// so no exp() can overflow (the NaN class reported for an SM90 chunk-scan
// kernel on the "Mamba2" knowledge page).
//
// Packed rows (seq_idx given): doc_i counts the document starts (a token
// whose id differs from the previous token's) from the chunk's first token
// through i, a block sum-scan of 0/1 flags.  A pair (j, i) contributes only
// when doc_j == doc_i, the entering state only when doc_i == 0, the chunk
// state only its last document's tokens, and a chunk holding a start passes
// no decayed state on (log decay -inf).
#include "ssd_common.cuh"
#include "ssd_internal.h"
#include "ssd_trace.h"

namespace ssd {
namespace {

constexpr int kThreads = 256;
constexpr int kTK = 32;      // tokens per smem tile in chunk_state
constexpr int kTJ = 32;      // j tokens per tile in chunk_out
constexpr int kTKH = 32;     // state rows per smem tile in chunk_out
constexpr int kMaxAcc = 32;  // accumulators per thread

}  // namespace

SimtWs simt_carve(const ScanDims &d, void *ws) {
    char *p = static_cast<char *>(ws);
    SimtWs w;
    w.status = reinterpret_cast<unsigned *>(p);
    size_t off = kStatusBytes;
    const size_t tok = (size_t)d.b * d.H * d.L * sizeof(float);
    w.dtv = reinterpret_cast<float *>(p + off); off += align256(tok);
    w.cum = reinterpret_cast<float *>(p + off); off += align256(tok);
    w.ell = reinterpret_cast<float *>(p + off); off += align256((size_t)d.b * d.H * d.nc * sizeof(float));
    w.states = reinterpret_cast<float *>(p + off);
    return w;
}

namespace {

// 1 when token t of row b starts a document of a packed row
__device__ __forceinline__ float doc_start(const int32_t *seq_idx, size_t b, int L, int t) {
    return (t > 0 && seq_idx[b * L + t] != seq_idx[b * L + t - 1]) ? 1.f : 0.f;
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
chunk_state_kernel(const T *__restrict__ x, const float *__restrict__ dt_raw,
                   const float *__restrict__ dt_bias, const float *__restrict__ A,
                   const T *__restrict__ Bm, const int32_t *__restrict__ seq_idx, SimtWs ws, int L, int H,
                   int P, int N, int G, int Q, int nc, float lo, float hi) {
    extern __shared__ float sm[];
    float *s_dt = sm;                 // Q
    float *s_cum = s_dt + Q;          // Q
    float *s_doc = s_cum + Q;         // Q (packed rows only)
    float *s_B = s_doc + Q;           // kTK * N
    float *s_X = s_B + kTK * N;       // kTK * P
    __shared__ float wtot[32];

    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int g = h / (H / G);
    const int t0 = c * Q;
    const int q = min(Q, L - t0);
    const float Ah = A[h], bias = dt_bias[h];
    const size_t bh = (size_t)b * H + h;
    if (threadIdx.x == 0 && Ah > 0.f) flag_status(ws.status, kStatusPrecondition);

    float carry = 0.f, dcarry = 0.f;
    for (int base = 0; base < q; base += kThreads) {
        const int i = base + threadIdx.x;
        float d = 0.f, da = 0.f;
        if (i < q) {
            d = dt_of(dt_raw[((size_t)b * L + t0 + i) * H + h], bias, lo, hi);
            da = d * Ah;
        }
        float tot;
        const float s = block_inclusive_scan(da, wtot, tot) + carry;
        if (i < q) {
            s_dt[i] = d;
            s_cum[i] = s;
            ws.dtv[bh * L + t0 + i] = d;
            ws.cum[bh * L + t0 + i] = s;
        }
        carry += tot;
        if (seq_idx) {                                // uniform over the block
            float dtot;
            const float dc = block_inclusive_scan(i < q ? doc_start(seq_idx, b, L, t0 + i) : 0.f, wtot, dtot);
            if (i < q) s_doc[i] = dc + dcarry;
            dcarry += dtot;
        }
    }
    __syncthreads();
    const float clast = s_cum[q - 1];
    const float dlast = seq_idx ? s_doc[q - 1] : 0.f;
    // a chunk that holds a document start passes no decayed state on
    if (threadIdx.x == 0) ws.ell[bh * nc + c] = dlast > 0.f ? -INFINITY : clast;

    // S[n, p] = sum_k w_k B[k, n] x[k, p]; thread owns column p, rows n0 + RN*r.
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
            s_B[k * N + n] = to_f(Bm[(((size_t)b * L + t0 + k0 + k) * G + g) * N + n]);
        }
        for (int e = threadIdx.x; e < kk * P; e += kThreads) {
            const int k = e / P, pp = e - k * P;
            // only the chunk's last document writes into the state it passes on
            const bool live = !seq_idx || s_doc[k0 + k] == dlast;
            const float w = live ? expf(fminf(clast - s_cum[k0 + k], 0.f)) * s_dt[k0 + k] : 0.f;
            s_X[k * P + pp] = w * to_f(x[(((size_t)b * L + t0 + k0 + k) * H + h) * P + pp]);
        }
        __syncthreads();
        if (n0 < N) {
            for (int k = 0; k < kk; ++k) {
                const float xv = s_X[k * P + p];
                const float *brow = s_B + k * N + n0;
#pragma unroll
                for (int r = 0; r < kMaxAcc; ++r)
                    if (r < nacc && n0 + r * RN < N) acc[r] = fmaf(brow[r * RN], xv, acc[r]);
            }
        }
    }
    float *out = ws.states + (bh * nc + c) * (size_t)N * P;
#pragma unroll
    for (int r = 0; r < kMaxAcc; ++r) {
        const int n = n0 + r * RN;
        if (r < nacc && n < N) out[(size_t)n * P + p] = acc[r];
    }
}

__global__ void __launch_bounds__(kThreads)
state_pass_kernel(SimtWs ws, const float *__restrict__ init, float *__restrict__ final_state,
                  float *__restrict__ chunk_states, int H, int NP, int nc) {
    const int e = blockIdx.x * kThreads + threadIdx.x;
    if (e >= NP) return;
    const size_t bh = (size_t)blockIdx.z * H + blockIdx.y;
    // state after chunk c at chunk_states[b, c, h, e]: chunk c's stride is H * NP
    float *out = chunk_states ? chunk_states + ((size_t)blockIdx.z * nc * H + blockIdx.y) * NP + e : nullptr;
    float hs = init ? init[bh * NP + e] : 0.f;
    float *S = ws.states + bh * nc * (size_t)NP + e;
    const float *ell = ws.ell + bh * nc;
    float nxt = S[0];
    for (int c = 0; c < nc; ++c) {
        const float s = nxt;
        if (c + 1 < nc) nxt = S[(size_t)(c + 1) * NP];
        S[(size_t)c * NP] = hs;                         // state entering chunk c
        hs = fmaf(expf(fminf(ell[c], 0.f)), hs, s);
        if (out) out[(size_t)c * H * NP] = hs;          // state after chunk c
    }
    if (final_state) final_state[bh * NP + e] = hs;
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
chunk_out_kernel(const T *__restrict__ x, const T *__restrict__ Bm, const T *__restrict__ Cm,
                 const float *__restrict__ D, const int32_t *__restrict__ seq_idx, SimtWs ws,
                 float *__restrict__ y, int L, int H, int P, int N, int G, int Q, int nc, int TI) {
    extern __shared__ float sm[];
    __shared__ float wtot[32];
    const int NB = N + 1;                       // padded B row
    float *s_doc = sm;                          // Q (packed rows only)
    float *s_C = s_doc + Q;                     // TI * N
    float *s_cumi = s_C + TI * N;               // TI
    float *s_Bj = s_cumi + TI;                  // kTJ * NB
    float *s_xj = s_Bj + kTJ * NB;              // kTJ * P
    float *s_dtj = s_xj + kTJ * P;              // kTJ
    float *s_cumj = s_dtj + kTJ;                // kTJ
    float *s_G = s_cumj + kTJ;                  // TI * (kTJ + 1)
    float *s_H = s_G + TI * (kTJ + 1);          // kTKH * P

    const int tiles = (Q + TI - 1) / TI;
    const int c = blockIdx.x / tiles, it = blockIdx.x - c * tiles;
    const int h = blockIdx.y, b = blockIdx.z;
    const int g = h / (H / G);
    const int t0 = c * Q;
    const int q = min(Q, L - t0);
    const int i0 = it * TI;
    if (i0 >= q) return;                        // uniform over the block
    const int ti = min(TI, q - i0);
    const size_t bh = (size_t)b * H + h;

    const int p = threadIdx.x % P, ib = threadIdx.x / P, RI = kThreads / P;
    const int nacc = (TI + RI - 1) / RI;
    float acc[kMaxAcc];
#pragma unroll
    for (int r = 0; r < kMaxAcc; ++r) acc[r] = 0.f;

    // document counters of the chunk's tokens through the tile's last row
    const int jend = i0 + ti;
    if (seq_idx) {                              // uniform over the block
        float dcarry = 0.f;
        for (int base = 0; base < jend; base += kThreads) {
            const int i = base + threadIdx.x;
            float dtot;
            const float dc = block_inclusive_scan(i < jend ? doc_start(seq_idx, b, L, t0 + i) : 0.f, wtot, dtot);
            if (i < jend) s_doc[i] = dc + dcarry;
            dcarry += dtot;
        }
        __syncthreads();
    }

    for (int e = threadIdx.x; e < TI * N; e += kThreads) {
        const int ii = e / N, n = e - ii * N;
        s_C[e] = ii < ti ? to_f(Cm[(((size_t)b * L + t0 + i0 + ii) * G + g) * N + n]) : 0.f;
    }
    for (int ii = threadIdx.x; ii < TI; ii += kThreads)
        s_cumi[ii] = ii < ti ? ws.cum[bh * L + t0 + i0 + ii] : 0.f;

    // state entering the chunk: acc_i = C_i^T H_{c-1}
    const float *Hin = ws.states + (bh * nc + c) * (size_t)N * P;
    for (int k0 = 0; k0 < N; k0 += kTKH) {
        const int kk = min(kTKH, N - k0);
        __syncthreads();
        for (int e = threadIdx.x; e < kk * P; e += kThreads) s_H[e] = Hin[(size_t)k0 * P + e];
        __syncthreads();
        if (ib < TI) {
            for (int k = 0; k < kk; ++k) {
                const float hv = s_H[k * P + p];
#pragma unroll
                for (int r = 0; r < kMaxAcc; ++r)
                    if (r < nacc) acc[r] = fmaf(s_C[(ib + r * RI) * N + k0 + k], hv, acc[r]);
            }
        }
    }
    // the entering state reaches row i only if no document starts in the chunk up to i
#pragma unroll
    for (int r = 0; r < kMaxAcc; ++r) {
        const int ii = ib + r * RI;
        if (r < nacc && ii < TI)
            acc[r] *= (!seq_idx || ii >= ti || s_doc[i0 + ii] == 0.f) ? expf(fminf(s_cumi[ii], 0.f)) : 0.f;
    }

    // intra-chunk part: j from the chunk start through the tile's last row
    for (int j0 = 0; j0 < jend; j0 += kTJ) {
        const int tj = min(kTJ, jend - j0);
        __syncthreads();
        for (int e = threadIdx.x; e < tj * N; e += kThreads) {
            const int jj = e / N, n = e - jj * N;
            s_Bj[jj * NB + n] = to_f(Bm[(((size_t)b * L + t0 + j0 + jj) * G + g) * N + n]);
        }
        for (int e = threadIdx.x; e < tj * P; e += kThreads) {
            const int jj = e / P, pp = e - jj * P;
            s_xj[jj * P + pp] = to_f(x[(((size_t)b * L + t0 + j0 + jj) * H + h) * P + pp]);
        }
        for (int jj = threadIdx.x; jj < tj; jj += kThreads) {
            s_dtj[jj] = ws.dtv[bh * L + t0 + j0 + jj];
            s_cumj[jj] = ws.cum[bh * L + t0 + j0 + jj];
        }
        __syncthreads();
        for (int e = threadIdx.x; e < TI * kTJ; e += kThreads) {
            const int ii = e / kTJ, jj = e - ii * kTJ;
            const int gi = i0 + ii, gj = j0 + jj;
            float v = 0.f;
            // causal select (and, on packed rows, same document) before any exp()
            if (ii < ti && jj < tj && gj <= gi && (!seq_idx || s_doc[gj] == s_doc[gi])) {
                const float *cr = s_C + ii * N;
                const float *br = s_Bj + jj * NB;
                float dot = 0.f;
                for (int n = 0; n < N; ++n) dot = fmaf(cr[n], br[n], dot);
                v = dot * expf(fminf(s_cumi[ii] - s_cumj[jj], 0.f)) * s_dtj[jj];
            }
            s_G[ii * (kTJ + 1) + jj] = v;
        }
        __syncthreads();
        if (ib < TI) {
            for (int jj = 0; jj < tj; ++jj) {
                const float xv = s_xj[jj * P + p];
#pragma unroll
                for (int r = 0; r < kMaxAcc; ++r)
                    if (r < nacc) acc[r] = fmaf(s_G[(ib + r * RI) * (kTJ + 1) + jj], xv, acc[r]);
            }
        }
    }

    const float Dh = D[h];
#pragma unroll
    for (int r = 0; r < kMaxAcc; ++r) {
        const int ii = ib + r * RI;
        if (r < nacc && ii < ti) {
            const size_t off = (((size_t)b * L + t0 + i0 + ii) * H + h) * P + p;
            y[off] = fmaf(Dh, to_f(x[off]), acc[r]);
        }
    }
}

int pick_ti(const ScanDims &d) {
    const int RI = kThreads / (int)d.P;
    int ti = 64;
    while (ti > 1 && (ti + RI - 1) / RI > kMaxAcc) ti >>= 1;
    return ti;
}

size_t state_smem(const ScanDims &d) {
    return sizeof(float) * (3 * (size_t)d.Q + (size_t)kTK * d.N + (size_t)kTK * d.P);
}

size_t out_smem(const ScanDims &d, int TI) {
    return sizeof(float) * ((size_t)d.Q + (size_t)TI * d.N + TI + (size_t)kTJ * (d.N + 1) + (size_t)kTJ * d.P +
                            2 * kTJ + (size_t)TI * (kTJ + 1) + (size_t)kTKH * d.P);
}

// Launches 1 and 2: dt, cum, the chunk log decays and the state entering
// every chunk (ws.states), plus final_state / chunk_states when asked for.
template <typename T>
cudaError_t run_states(const ScanArgs &a, const ScanDims &d, const SimtWs &ws, cudaStream_t s) {
    const size_t sm1 = state_smem(d);
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(chunk_state_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)sm1)) != cudaSuccess)
        return e;
    const dim3 g1((unsigned)d.nc, (unsigned)d.H, (unsigned)d.b);
    {
        TraceScope tr(s, kTrSimtChunkState);
        chunk_state_kernel<T><<<g1, kThreads, sm1, s>>>(
            (const T *)a.x, a.dt_raw, a.dt_bias, a.A, (const T *)a.B, a.seq_idx, ws, (int)d.L, (int)d.H,
            (int)d.P, (int)d.N, (int)d.G, (int)d.Q, (int)d.nc, a.dt_lo, a.dt_hi);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int NP = (int)(d.N * d.P);
    const dim3 g2((unsigned)((NP + kThreads - 1) / kThreads), (unsigned)d.H, (unsigned)d.b);
    {
        TraceScope tr(s, kTrSimtStatePass);
        state_pass_kernel<<<g2, kThreads, 0, s>>>(ws, a.init_state, a.final_state, a.chunk_states, (int)d.H, NP,
                                                  (int)d.nc);
    }
    return cudaGetLastError();
}

template <typename T>
cudaError_t run(const ScanArgs &a, const ScanDims &d, void *wsp, cudaStream_t s) {
    SimtWs ws = simt_carve(d, wsp);
    const int TI = pick_ti(d);
    const size_t sm3 = out_smem(d, TI);
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(chunk_out_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)sm3)) != cudaSuccess)
        return e;
    if ((e = run_states<T>(a, d, ws, s)) != cudaSuccess) return e;
    const int tiles = (int)((d.Q + TI - 1) / TI);
    const dim3 g3((unsigned)(d.nc * tiles), (unsigned)d.H, (unsigned)d.b);
    {
        TraceScope tr(s, kTrSimtChunkOut);
        chunk_out_kernel<T><<<g3, kThreads, sm3, s>>>(
            (const T *)a.x, (const T *)a.B, (const T *)a.C, a.D, a.seq_idx, ws, a.y, (int)d.L, (int)d.H,
            (int)d.P, (int)d.N, (int)d.G, (int)d.Q, (int)d.nc, TI);
    }
    return cudaGetLastError();
}

}  // namespace

bool simt_supported(const ScanDims &d) {
    if (d.P < 1 || d.P > kThreads || kThreads % d.P != 0) return false;
    if (d.N < 1 || d.N * d.P > (int64_t)kThreads * kMaxAcc) return false;
    if (d.Q < 1 || d.Q > 8192) return false;
    if (d.nc > 0x7fffffff / 64 || d.H > 65535 || d.b > 65535) return false;
    return state_smem(d) <= 200 * 1024 && out_smem(d, pick_ti(d)) <= 200 * 1024;
}

size_t simt_workspace_bytes(const ScanDims &d) {
    const size_t tok = (size_t)d.b * d.H * d.L * sizeof(float);
    return kStatusBytes + 2 * align256(tok) + align256((size_t)d.b * d.H * d.nc * sizeof(float)) +
           align256((size_t)d.b * d.H * d.nc * d.N * d.P * sizeof(float));
}

cudaError_t simt_scan(const ScanArgs &a, const ScanDims &d, void *ws, cudaStream_t s) {
    return a.bf16 ? run<__nv_bfloat16>(a, d, ws, s) : run<float>(a, d, ws, s);
}

cudaError_t simt_state_pass(const ScanArgs &a, const ScanDims &d, void *wsp, cudaStream_t s) {
    const SimtWs ws = simt_carve(d, wsp);
    const int NP = (int)(d.N * d.P);
    const dim3 g2((unsigned)((NP + kThreads - 1) / kThreads), (unsigned)d.H, (unsigned)d.b);
    {
        TraceScope tr(s, kTrSimtStatePass);
        state_pass_kernel<<<g2, kThreads, 0, s>>>(ws, a.init_state, a.final_state, a.chunk_states, (int)d.H, NP,
                                                  (int)d.nc);
    }
    return cudaGetLastError();
}

cudaError_t simt_scan_states(const ScanArgs &a, const ScanDims &d, void *ws, cudaStream_t s) {
    const SimtWs w = simt_carve(d, ws);
    return a.bf16 ? run_states<__nv_bfloat16>(a, d, w, s) : run_states<float>(a, d, w, s);
}

}  // namespace ssd
