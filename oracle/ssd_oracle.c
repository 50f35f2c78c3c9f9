/*
 * ssd_oracle.c -- plain, slow fp64 CPU evaluation of the Mamba-2 SSD
 * selective-state-space recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or helper with the CUDA path in state_space_sequence_scan_b200/
 * and the CUDA path never calls it.
 *
 * What it computes (nnterp guide "Mamba-2", opening paragraph and the table
 * in "The values"):
 *   per head h, with state S an N x P matrix (state_dim rows, head_dim cols,
 *   "key side first"), for every token t in order:
 *     dt  = clamp(softplus(dt_raw[t,h] + dt_bias[h]), dt_lo, dt_hi)
 *     a   = exp(dt * A[h])                       (A*dt is the log decay)
 *     S   = a * S + dt * B[t,g] (outer) x[t,h]   (B is the key, x the value)
 *     y[t,h] = S^T C[t,g] + D[h] * x[t,h]        (C reads the state)
 *   where g = h / (H / G) is the group whose B and C head h uses ("one per
 *   group of heads"), S starts from init_state (zeros when absent, as for a
 *   fresh prompt) and final_state is S after the last token.
 * The decode step (nnterp guide "Mamba-2", section "The state between
 * steps") is the same loop body for one token with the state updated in
 * place.
 * Packed sequences (the "Mamba2" knowledge page notes sample packing for
 * Mamba2): with seq_idx [b, L] given, a token whose seq_idx differs from the
 * previous token's starts a new document, and the state is set to zero
 * before its update; the first document of a row starts from init_state.
 * The chunk-boundary states (same guide, "The state after every token"):
 *   states[b, c, h] = S after token min((c+1) Q, L) - 1, for c < ceil(L / Q),
 *   so the last one is final_state and Q = 1 gives the state after every
 *   token.
 *
 * Readings where the pages are silent: softplus in its exact stable form;
 * the clamp is applied after the softplus; groups are contiguous blocks of
 * heads; D is one scalar per head.
 *
 * Inputs are float32 arrays holding exactly the values given to the GPU
 * (bf16 inputs widened to float32, which is exact); all arithmetic is double.
 * Layouts (row-major, contiguous):
 *   x [b,L,H,P]  dt_raw [b,L,H]  dt_bias [H]  A [H]  B,C [b,L,G,N]  D [H]
 *   init_state [b,H,N,P] (may be NULL)   y [b,L,H,P]  final_state [b,H,N,P]
 *   chunk_states [b, ceil(L/Q), H, N, P] (may be NULL)
 *
 * Parity: pinned by tests/test_oracle.py (closed form, invariants, special
 * cases, hand-computed golden example).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

static double sp_exact(double z)
{
    /* softplus(z) = log(1 + e^z), written so neither branch overflows */
    return (z > 0.0 ? z : 0.0) + log1p(exp(-fabs(z)));
}

static double clamp_dt(double v, double lo, double hi)
{
    if (v < lo) v = lo;
    if (v > hi) v = hi;
    return v;
}

double ssd_oracle_softplus(double z) { return sp_exact(z); }

typedef struct {
    const float *x, *dt_raw, *dt_bias, *A, *B, *C, *D, *init_state;
    double *y, *final_state;
    double *chunk_states;     /* [b, nc, H, N, P] or NULL */
    const int32_t *seq_idx;   /* [b, L] or NULL: document ids of packed rows */
    int64_t b, L, H, P, N, G;
    int64_t Q, nc;            /* chunk size and count for chunk_states */
    double dt_lo, dt_hi;
    int64_t next;             /* next chain to claim */
    pthread_mutex_t lock;
    int status;
} scan_job;

static int64_t claim(scan_job *J)
{
    int64_t c;
    pthread_mutex_lock(&J->lock);
    c = J->next++;
    pthread_mutex_unlock(&J->lock);
    return c;
}

/* One (batch, head) chain of the recurrence, token by token. */
static int run_chain(scan_job *J, int64_t bi, int64_t h, double *S, double *yacc)
{
    const int64_t L = J->L, H = J->H, P = J->P, N = J->N, G = J->G;
    const int64_t g = h / (H / G);
    const double A = J->A[h], Dh = J->D[h], bias = J->dt_bias[h];
    int64_t n, p, t;

    if (J->init_state) {
        const float *s0 = J->init_state + (bi * H + h) * N * P;
        for (n = 0; n < N * P; ++n) S[n] = (double)s0[n];
    } else {
        memset(S, 0, sizeof(double) * (size_t)(N * P));
    }

    for (t = 0; t < L; ++t) {
        const double z = (double)J->dt_raw[(bi * L + t) * H + h] + bias;
        if (J->seq_idx && t > 0 && J->seq_idx[bi * L + t] != J->seq_idx[bi * L + t - 1])
            memset(S, 0, sizeof(double) * (size_t)(N * P));      /* a new document */
        const double dt = clamp_dt(sp_exact(z), J->dt_lo, J->dt_hi);
        const double a = exp(dt * A);
        const float *xr = J->x + ((bi * L + t) * H + h) * P;
        const float *Br = J->B + ((bi * L + t) * G + g) * N;
        const float *Cr = J->C + ((bi * L + t) * G + g) * N;
        double *yr = J->y + ((bi * L + t) * H + h) * P;

        /* S <- a S + dt B x^T */
        for (n = 0; n < N; ++n) {
            const double w = dt * (double)Br[n];
            double *Sn = S + n * P;
            for (p = 0; p < P; ++p) Sn[p] = a * Sn[p] + w * (double)xr[p];
        }
        /* y <- S^T C + D x */
        for (p = 0; p < P; ++p) yacc[p] = 0.0;
        for (n = 0; n < N; ++n) {
            const double c = (double)Cr[n];
            const double *Sn = S + n * P;
            for (p = 0; p < P; ++p) yacc[p] += c * Sn[p];
        }
        for (p = 0; p < P; ++p) yr[p] = yacc[p] + Dh * (double)xr[p];

        /* the state after the last token of a chunk */
        if (J->chunk_states && ((t + 1) % J->Q == 0 || t == L - 1)) {
            double *sc = J->chunk_states + ((bi * J->nc + t / J->Q) * H + h) * N * P;
            memcpy(sc, S, sizeof(double) * (size_t)(N * P));
        }
    }

    if (J->final_state) {
        double *sf = J->final_state + (bi * H + h) * N * P;
        memcpy(sf, S, sizeof(double) * (size_t)(N * P));
    }
    return 0;
}

static void *scan_worker(void *arg)
{
    scan_job *J = (scan_job *)arg;
    double *S = (double *)malloc(sizeof(double) * (size_t)(J->N * J->P));
    double *yacc = (double *)malloc(sizeof(double) * (size_t)J->P);
    int64_t c;
    if (!S || !yacc) {
        J->status = -2;
        free(S);
        free(yacc);
        return NULL;
    }
    while ((c = claim(J)) < J->b * J->H) run_chain(J, c / J->H, c % J->H, S, yacc);
    free(S);
    free(yacc);
    return NULL;
}

static int pick_threads(int nthreads, int64_t chains)
{
    if (nthreads <= 0) {
        long nc = sysconf(_SC_NPROCESSORS_ONLN);
        nthreads = nc > 0 ? (int)nc : 1;
    }
    if (nthreads > chains) nthreads = (int)chains;
    if (nthreads < 1) nthreads = 1;
    return nthreads;
}

static int run_threads(void *(*fn)(void *), void *job, int nthreads)
{
    pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    int i, started = 0;
    if (!tid) {
        fn(job);               /* run on the calling thread alone */
        return 0;
    }
    for (i = 0; i < nthreads - 1; ++i)
        if (pthread_create(&tid[started], NULL, fn, job) == 0) ++started;
    fn(job);
    for (i = 0; i < started; ++i) pthread_join(tid[i], NULL);
    free(tid);
    return 0;
}

/* Whole-sequence recurrence, also recording the state after every chunk of Q
 * tokens into chunk_states when that is not NULL.  Returns 0, or -1 on bad
 * dimensions, -2 when out of memory.  nthreads <= 0 uses every online core. */
int ssd_oracle_scan_varlen(const float *x, const float *dt_raw, const float *dt_bias,
                           const float *A, const float *B, const float *C, const float *D,
                           const float *init_state, const int32_t *seq_idx, double *y,
                           double *final_state, double *chunk_states, int64_t b, int64_t L, int64_t H,
                           int64_t P, int64_t N, int64_t G, int64_t Q, double dt_lo, double dt_hi,
                           int nthreads)
{
    scan_job J;
    if (b < 0 || L < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || H % G != 0) return -1;
    if (chunk_states && Q < 1) return -1;
    if (b == 0) return 0;
    memset(&J, 0, sizeof J);
    J.x = x; J.dt_raw = dt_raw; J.dt_bias = dt_bias; J.A = A; J.B = B; J.C = C; J.D = D;
    J.init_state = init_state; J.y = y; J.final_state = final_state;
    J.chunk_states = chunk_states;
    J.seq_idx = seq_idx;
    J.Q = Q > 0 ? Q : 1;
    J.nc = (L + J.Q - 1) / J.Q;
    J.b = b; J.L = L; J.H = H; J.P = P; J.N = N; J.G = G;
    J.dt_lo = dt_lo; J.dt_hi = dt_hi;
    pthread_mutex_init(&J.lock, NULL);
    run_threads(scan_worker, &J, pick_threads(nthreads, b * H));
    pthread_mutex_destroy(&J.lock);
    return J.status;
}

/* Whole-sequence recurrence with the chunk-boundary states, no packing. */
int ssd_oracle_scan_states(const float *x, const float *dt_raw, const float *dt_bias,
                           const float *A, const float *B, const float *C, const float *D,
                           const float *init_state, double *y, double *final_state,
                           double *chunk_states, int64_t b, int64_t L, int64_t H, int64_t P,
                           int64_t N, int64_t G, int64_t Q, double dt_lo, double dt_hi, int nthreads)
{
    return ssd_oracle_scan_varlen(x, dt_raw, dt_bias, A, B, C, D, init_state, NULL, y, final_state,
                                  chunk_states, b, L, H, P, N, G, Q, dt_lo, dt_hi, nthreads);
}

/* Whole-sequence recurrence: y and final_state only. */
int ssd_oracle_scan(const float *x, const float *dt_raw, const float *dt_bias,
                    const float *A, const float *B, const float *C, const float *D,
                    const float *init_state, double *y, double *final_state,
                    int64_t b, int64_t L, int64_t H, int64_t P, int64_t N, int64_t G,
                    double dt_lo, double dt_hi, int nthreads)
{
    return ssd_oracle_scan_states(x, dt_raw, dt_bias, A, B, C, D, init_state, y, final_state, NULL,
                                  b, L, H, P, N, G, 1, dt_lo, dt_hi, nthreads);
}

typedef struct {
    const float *x, *dt_raw, *dt_bias, *A, *B, *C, *D;
    double *state, *y;
    int64_t b, H, P, N, G;
    double dt_lo, dt_hi;
    int64_t next;
    pthread_mutex_t lock;
} step_job;

static void *step_worker(void *arg)
{
    step_job *J = (step_job *)arg;
    const int64_t H = J->H, P = J->P, N = J->N, G = J->G;
    int64_t c, n, p;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        c = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (c >= J->b * H) break;
        {
            const int64_t bi = c / H, h = c % H, g = h / (H / G);
            const double z = (double)J->dt_raw[bi * H + h] + (double)J->dt_bias[h];
            const double dt = clamp_dt(sp_exact(z), J->dt_lo, J->dt_hi);
            const double a = exp(dt * (double)J->A[h]);
            const float *xr = J->x + (bi * H + h) * P;
            const float *Br = J->B + (bi * G + g) * N;
            const float *Cr = J->C + (bi * G + g) * N;
            double *S = J->state + (bi * H + h) * N * P;
            double *yr = J->y + (bi * H + h) * P;
            for (n = 0; n < N; ++n) {
                const double w = dt * (double)Br[n];
                for (p = 0; p < P; ++p) S[n * P + p] = a * S[n * P + p] + w * (double)xr[p];
            }
            for (p = 0; p < P; ++p) yr[p] = 0.0;
            for (n = 0; n < N; ++n) {
                const double cn = (double)Cr[n];
                for (p = 0; p < P; ++p) yr[p] += cn * S[n * P + p];
            }
            for (p = 0; p < P; ++p) yr[p] += (double)J->D[h] * (double)xr[p];
        }
    }
    return NULL;
}

/* One decode token: state [b,H,N,P] (double) updated in place, y [b,H,P].
 * x [b,H,P], dt_raw [b,H], B,C [b,G,N]. */
int ssd_oracle_step(const float *x, const float *dt_raw, const float *dt_bias,
                    const float *A, const float *B, const float *C, const float *D,
                    double *state, double *y,
                    int64_t b, int64_t H, int64_t P, int64_t N, int64_t G,
                    double dt_lo, double dt_hi, int nthreads)
{
    step_job J;
    if (b < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || H % G != 0) return -1;
    if (b == 0) return 0;
    memset(&J, 0, sizeof J);
    J.x = x; J.dt_raw = dt_raw; J.dt_bias = dt_bias; J.A = A; J.B = B; J.C = C; J.D = D;
    J.state = state; J.y = y;
    J.b = b; J.H = H; J.P = P; J.N = N; J.G = G;
    J.dt_lo = dt_lo; J.dt_hi = dt_hi;
    pthread_mutex_init(&J.lock, NULL);
    run_threads(step_worker, &J, pick_threads(nthreads, b * H));
    pthread_mutex_destroy(&J.lock);
    return 0;
}

/* ---------------------------------------------------------------------------
 * The steps either side of the scan in a Mamba-2 layer (the nnterp guide's y
 * is taken "before the gated norm and out_proj"; the state-spaces/mamba
 * issue names causal_conv1d_fn applied before the chunk scan).  Readings
 * where the pages give no numbers: the conv is causal and depthwise over the
 * channels that become x, B and C, width K, with a bias and SiLU, starting
 * from zeros; the gate is y * silu(z) and the norm an RMS norm over groups of
 * `group` channels, times a per-channel weight.
 *
 * conv1d_silu:  in [b, L, Cd] (Cd channels), w [Cd, K], bias [Cd] ->
 *   out[b,t,c] = silu(bias[c] + sum_{k<K} w[c,k] in[b, t-(K-1)+k, c]),
 *   in[b, t<0, c] = 0.
 * gated_rmsnorm: y, z [T, D], weight [D], groups of `group` channels ->
 *   v = y * silu(z);  out = v / sqrt(mean_group(v^2) + eps) * weight.
 * silu(u) = u / (1 + exp(-u)).
 */
static double silu_d(double u) { return u / (1.0 + exp(-u)); }

int ssd_oracle_conv1d_silu(const float *in, const float *w, const float *bias, double *out,
                           int64_t b, int64_t L, int64_t Cd, int64_t K)
{
    int64_t bi, t, c, k;
    if (b < 0 || L < 0 || Cd <= 0 || K <= 0) return -1;
    for (bi = 0; bi < b; ++bi)
        for (t = 0; t < L; ++t)
            for (c = 0; c < Cd; ++c) {
                double acc = (double)bias[c];
                for (k = 0; k < K; ++k) {
                    const int64_t s = t - (K - 1) + k;
                    if (s >= 0) acc += (double)w[c * K + k] * (double)in[(bi * L + s) * Cd + c];
                }
                out[(bi * L + t) * Cd + c] = silu_d(acc);
            }
    return 0;
}

int ssd_oracle_gated_rmsnorm(const float *y, const float *z, const float *weight, double *out,
                             int64_t T, int64_t D, int64_t group, double eps)
{
    int64_t t, g0, j;
    if (T < 0 || D <= 0 || group <= 0 || D % group != 0 || eps < 0) return -1;
    for (t = 0; t < T; ++t)
        for (g0 = 0; g0 < D; g0 += group) {
            double ss = 0.0, r;
            for (j = g0; j < g0 + group; ++j) {
                const double v = (double)y[t * D + j] * silu_d((double)z[t * D + j]);
                ss += v * v;
            }
            r = 1.0 / sqrt(ss / (double)group + eps);
            for (j = g0; j < g0 + group; ++j) {
                const double v = (double)y[t * D + j] * silu_d((double)z[t * D + j]);
                out[t * D + j] = v * r * (double)weight[j];
            }
        }
    return 0;
}

/* ---------------------------------------------------------------------------
 * Backward of the scan: reverse mode of the token-by-token recurrence.  The
 * pages say only that the backward pass of the usual mamba kernels is not
 * deterministic (HF transformers issue "mamba2 mixer different outputs",
 * reply on the backward pass); the gradients themselves are the plain
 * derivatives of the recurrence above.  For an upstream gradient dy of y and
 * dfinal of final_state, with G = dLoss/dS_t running backwards from
 * G = dfinal (zeros when NULL):
 *   G      += C_t dy_t^T                        (y_t reads S_t)
 *   dC_t    = S_t dy_t
 *   dx_t    = dt_t G^T B_t + D dy_t
 *   dB_t    = dt_t G x_t
 *   ddt_t   = B_t^T G x_t + A a_t <G, S_{t-1}>  (a_t = exp(dt_t A))
 *   dA     += dt_t a_t <G, S_{t-1}>,   dD += dy_t . x_t
 *   dz_t    = ddt_t softplus'(z_t) [dt_lo <= softplus(z_t) <= dt_hi]
 *   G       = a_t G                             (S_t = a_t S_{t-1} + ...)
 * and dinit = G after token 0.  dz_t is the gradient of dt_raw[t] and, summed
 * over tokens, of dt_bias.  Packed rows (seq_idx given): at a document start
 * the state is zeroed before the update, so S_{t-1} reads as zero there (no
 * decay term) and no gradient passes to earlier tokens (G = 0 after it).  Per head: dB_h/dC_h [b,L,H,N] (the caller sums the
 * heads of each group), dA_h/ddt_bias_h/dD_h [b,H] (the caller sums over b).
 * The states S_t are recomputed forward from checkpoints every kSeg tokens,
 * which changes no arithmetic (the same products in the same order).
 */
#define kSeg 64

typedef struct {
    const float *x, *dt_raw, *dt_bias, *A, *B, *C, *D, *init_state, *dy, *dfinal;
    const int32_t *seq_idx;   /* [b, L] or NULL */
    double *dx, *ddt_raw, *dB_h, *dC_h, *dA_h, *ddt_bias_h, *dD_h, *dinit;
    int64_t b, L, H, P, N, G;
    double dt_lo, dt_hi;
    int64_t next;
    pthread_mutex_t lock;
    int status;
} bwd_job;

static double sigmoid_exact(double z)
{
    /* d softplus / dz, in a form that never overflows */
    return z >= 0.0 ? 1.0 / (1.0 + exp(-z)) : exp(z) / (1.0 + exp(z));
}

/* 1 when token t of row bi starts a document of a packed row */
static int doc_start(const bwd_job *J, int64_t bi, int64_t t)
{
    return J->seq_idx && t > 0 && J->seq_idx[bi * J->L + t] != J->seq_idx[bi * J->L + t - 1];
}

/* forward update of S by token t of chain (bi, h) */
static void fwd_token(const bwd_job *J, int64_t bi, int64_t h, int64_t t, double *S, double *dt_out,
                      double *a_out)
{
    const int64_t L = J->L, H = J->H, P = J->P, N = J->N, G = J->G, g = h / (H / G);
    const double z = (double)J->dt_raw[(bi * L + t) * H + h] + (double)J->dt_bias[h];
    const double dt = clamp_dt(sp_exact(z), J->dt_lo, J->dt_hi);
    const double a = exp(dt * (double)J->A[h]);
    const float *xr = J->x + ((bi * L + t) * H + h) * P;
    const float *Br = J->B + ((bi * L + t) * G + g) * N;
    int64_t n, p;
    if (doc_start(J, bi, t)) memset(S, 0, sizeof(double) * (size_t)(N * P));    /* a new document */
    for (n = 0; n < N; ++n) {
        const double w = dt * (double)Br[n];
        for (p = 0; p < P; ++p) S[n * P + p] = a * S[n * P + p] + w * (double)xr[p];
    }
    *dt_out = dt;
    *a_out = a;
}

static void bwd_chain(bwd_job *J, int64_t bi, int64_t h, double *ck, double *seg, double *Gm)
{
    const int64_t L = J->L, H = J->H, P = J->P, N = J->N, G = J->G, g = h / (H / G);
    const int64_t NP = N * P, nseg = (L + kSeg - 1) / kSeg;
    const double A = J->A[h], Dh = J->D[h];
    double dA = 0.0, dbias = 0.0, dD = 0.0, dt, a;
    int64_t s, t, n, p, i;

    /* checkpoints: ck[s] = the state before token s*kSeg */
    if (J->init_state) {
        for (i = 0; i < NP; ++i) ck[i] = (double)J->init_state[(bi * H + h) * NP + i];
    } else {
        memset(ck, 0, sizeof(double) * (size_t)NP);
    }
    for (s = 0; s + 1 < nseg; ++s) {
        memcpy(ck + (s + 1) * NP, ck + s * NP, sizeof(double) * (size_t)NP);
        for (t = s * kSeg; t < (s + 1) * kSeg; ++t) fwd_token(J, bi, h, t, ck + (s + 1) * NP, &dt, &a);
    }

    if (J->dfinal) {
        for (i = 0; i < NP; ++i) Gm[i] = (double)J->dfinal[(bi * H + h) * NP + i];
    } else {
        memset(Gm, 0, sizeof(double) * (size_t)NP);
    }
    for (s = nseg - 1; s >= 0; --s) {
        const int64_t t0 = s * kSeg, t1 = (t0 + kSeg < L) ? t0 + kSeg : L;
        /* seg[k] = S after token t0 + k - 1 (seg[0] = the checkpoint) */
        double dts[kSeg], as[kSeg];
        memcpy(seg, ck + s * NP, sizeof(double) * (size_t)NP);
        for (t = t0; t < t1; ++t) {
            memcpy(seg + (t - t0 + 1) * NP, seg + (t - t0) * NP, sizeof(double) * (size_t)NP);
            fwd_token(J, bi, h, t, seg + (t - t0 + 1) * NP, &dts[t - t0], &as[t - t0]);
        }
        for (t = t1 - 1; t >= t0; --t) {
            const double *Scur = seg + (t - t0 + 1) * NP, *Sprev = seg + (t - t0) * NP;
            const int start = doc_start(J, bi, t);
            const double dtt = dts[t - t0], at = as[t - t0];
            const float *xr = J->x + ((bi * L + t) * H + h) * P;
            const float *Br = J->B + ((bi * L + t) * G + g) * N;
            const float *Cr = J->C + ((bi * L + t) * G + g) * N;
            const float *dyr = J->dy + ((bi * L + t) * H + h) * P;
            double *dxr = J->dx + ((bi * L + t) * H + h) * P;
            double *dBr = J->dB_h + ((bi * L + t) * H + h) * N;
            double *dCr = J->dC_h + ((bi * L + t) * H + h) * N;
            const double z = (double)J->dt_raw[(bi * L + t) * H + h] + (double)J->dt_bias[h];
            const double sp = sp_exact(z);
            double bgx = 0.0, gs = 0.0, dz;

            for (n = 0; n < N; ++n)
                for (p = 0; p < P; ++p) Gm[n * P + p] += (double)Cr[n] * (double)dyr[p];
            for (n = 0; n < N; ++n) {
                double acc = 0.0;
                for (p = 0; p < P; ++p) acc += Scur[n * P + p] * (double)dyr[p];
                dCr[n] = acc;
            }
            for (p = 0; p < P; ++p) {
                double acc = 0.0;
                for (n = 0; n < N; ++n) acc += Gm[n * P + p] * (double)Br[n];
                dxr[p] = dtt * acc + Dh * (double)dyr[p];
            }
            for (n = 0; n < N; ++n) {
                double acc = 0.0;
                for (p = 0; p < P; ++p) acc += Gm[n * P + p] * (double)xr[p];
                dBr[n] = dtt * acc;
                bgx += (double)Br[n] * acc;
            }
            if (!start)
                for (i = 0; i < NP; ++i) gs += Gm[i] * Sprev[i];
            for (p = 0; p < P; ++p) dD += (double)dyr[p] * (double)xr[p];
            dA += dtt * at * gs;
            dz = (bgx + A * at * gs) * ((sp >= J->dt_lo && sp <= J->dt_hi) ? sigmoid_exact(z) : 0.0);
            J->ddt_raw[(bi * L + t) * H + h] = dz;
            dbias += dz;
            for (i = 0; i < NP; ++i) Gm[i] = start ? 0.0 : Gm[i] * at;
        }
    }
    memcpy(J->dinit + (bi * H + h) * NP, Gm, sizeof(double) * (size_t)NP);
    J->dA_h[bi * H + h] = dA;
    J->ddt_bias_h[bi * H + h] = dbias;
    J->dD_h[bi * H + h] = dD;
}

static void *bwd_worker(void *arg)
{
    bwd_job *J = (bwd_job *)arg;
    const int64_t NP = J->N * J->P, nseg = (J->L + kSeg - 1) / kSeg;
    double *ck = (double *)malloc(sizeof(double) * (size_t)(NP * (nseg > 0 ? nseg : 1)));
    double *seg = (double *)malloc(sizeof(double) * (size_t)(NP * (kSeg + 1)));
    double *Gm = (double *)malloc(sizeof(double) * (size_t)NP);
    int64_t c;
    if (!ck || !seg || !Gm) {
        J->status = -2;
    } else {
        for (;;) {
            pthread_mutex_lock(&J->lock);
            c = J->next++;
            pthread_mutex_unlock(&J->lock);
            if (c >= J->b * J->H) break;
            bwd_chain(J, c / J->H, c % J->H, ck, seg, Gm);
        }
    }
    free(ck);
    free(seg);
    free(Gm);
    return NULL;
}

/* Gradients of <dy, y> + <dfinal, final_state> for the whole-sequence scan,
 * over packed rows when seq_idx [b, L] (document ids) is not NULL.  dy [b,L,H,P] and dfinal [b,H,N,P] (may be NULL) are float32
 * as given to the GPU; outputs are double: dx [b,L,H,P], ddt_raw [b,L,H],
 * dB_h, dC_h [b,L,H,N] (per head), dA_h, ddt_bias_h, dD_h [b,H] (per chain),
 * dinit [b,H,N,P].  Returns 0, -1 on bad dimensions, -2 when out of memory. */
int ssd_oracle_scan_bwd_varlen(const float *x, const float *dt_raw, const float *dt_bias, const float *A,
                               const float *B, const float *C, const float *D, const float *init_state,
                               const int32_t *seq_idx, const float *dy, const float *dfinal, double *dx,
                               double *ddt_raw, double *dB_h, double *dC_h, double *dA_h, double *ddt_bias_h,
                               double *dD_h, double *dinit, int64_t b, int64_t L, int64_t H, int64_t P, int64_t N,
                               int64_t G, double dt_lo, double dt_hi, int nthreads)
{
    bwd_job J;
    if (b < 0 || L < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || H % G != 0) return -1;
    if (b == 0) return 0;
    memset(&J, 0, sizeof J);
    J.x = x; J.dt_raw = dt_raw; J.dt_bias = dt_bias; J.A = A; J.B = B; J.C = C; J.D = D;
    J.init_state = init_state; J.dy = dy; J.dfinal = dfinal; J.seq_idx = seq_idx;
    J.dx = dx; J.ddt_raw = ddt_raw; J.dB_h = dB_h; J.dC_h = dC_h;
    J.dA_h = dA_h; J.ddt_bias_h = ddt_bias_h; J.dD_h = dD_h; J.dinit = dinit;
    J.b = b; J.L = L; J.H = H; J.P = P; J.N = N; J.G = G;
    J.dt_lo = dt_lo; J.dt_hi = dt_hi;
    pthread_mutex_init(&J.lock, NULL);
    run_threads(bwd_worker, &J, pick_threads(nthreads, b * H));
    pthread_mutex_destroy(&J.lock);
    return J.status;
}

/* ssd_oracle_scan_bwd_varlen without packing. */
int ssd_oracle_scan_bwd(const float *x, const float *dt_raw, const float *dt_bias, const float *A,
                        const float *B, const float *C, const float *D, const float *init_state,
                        const float *dy, const float *dfinal, double *dx, double *ddt_raw, double *dB_h,
                        double *dC_h, double *dA_h, double *ddt_bias_h, double *dD_h, double *dinit,
                        int64_t b, int64_t L, int64_t H, int64_t P, int64_t N, int64_t G, double dt_lo,
                        double dt_hi, int nthreads)
{
    return ssd_oracle_scan_bwd_varlen(x, dt_raw, dt_bias, A, B, C, D, init_state, NULL, dy, dfinal, dx, ddt_raw,
                                      dB_h, dC_h, dA_h, ddt_bias_h, dD_h, dinit, b, L, H, P, N, G, dt_lo, dt_hi,
                                      nthreads);
}
