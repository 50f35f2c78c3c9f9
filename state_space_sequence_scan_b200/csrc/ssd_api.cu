// C ABI of libssd.so: argument checks, path selection, workspace carve-up and
// launches.  Declared in include/ssd.h, which documents every argument.
#include <math.h>
#include <stdint.h>

#include "../../include/ssd.h"
#include "ssd_common.cuh"
#include "ssd_internal.h"

namespace {

thread_local int g_last_cuda_error = 0;

ssd_status cuda_fail(cudaError_t e) {
    g_last_cuda_error = (int)e;
    return SSD_ERR_CUDA;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool dtype_ok(int t) { return t == SSD_F32 || t == SSD_BF16; }

bool limits_ok(float lo, float hi) {
    return !isnan(lo) && !isnan(hi) && lo >= 0.0f && hi >= lo;
}

ssd_status check_scan_dims(int64_t b, int64_t L, int64_t H, int64_t P, int64_t N, int64_t G,
                           int64_t Q, int in_dtype, int path) {
    if (b < 0 || L < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || Q <= 0) return SSD_ERR_INVALID_ARG;
    if (H % G != 0) return SSD_ERR_INVALID_ARG;
    if (!dtype_ok(in_dtype)) return SSD_ERR_UNSUPPORTED;
    if (path != SSD_PATH_AUTO && path != SSD_PATH_SIMT && path != SSD_PATH_TENSOR)
        return SSD_ERR_INVALID_ARG;
    // every flat index fits comfortably in 63 bits; per-launch grid limits are
    // checked by the path's own support test
    if (b > (1ll << 20) || L > (1ll << 31) || H > 65535 || P > 65535 || N > 65535) return SSD_ERR_UNSUPPORTED;
    return SSD_OK;
}

// SSD_PATH_AUTO picks the tensor-core path when this is set and the shape fits.
constexpr bool kAutoTensor = true;

// Resolves `path` for these sizes; SSD_ERR_UNSUPPORTED when nothing fits.
ssd_status resolve_path(const ssd::ScanDims &d, int in_dtype, int path, int *chosen) {
    const bool tc = ssd::tc_supported(d, in_dtype == SSD_BF16);
    const bool simt = ssd::simt_supported(d);
    if (path == SSD_PATH_TENSOR) {
        if (!tc) return SSD_ERR_UNSUPPORTED;
        *chosen = SSD_PATH_TENSOR;
    } else if (path == SSD_PATH_SIMT) {
        if (!simt) return SSD_ERR_UNSUPPORTED;
        *chosen = SSD_PATH_SIMT;
    } else if (tc && kAutoTensor) {
        *chosen = SSD_PATH_TENSOR;
    } else if (simt) {
        *chosen = SSD_PATH_SIMT;
    } else {
        return SSD_ERR_UNSUPPORTED;
    }
    return SSD_OK;
}

ssd::ScanDims make_dims(int64_t b, int64_t L, int64_t H, int64_t P, int64_t N, int64_t G, int64_t Q) {
    ssd::ScanDims d;
    d.b = b; d.L = L; d.H = H; d.P = P; d.N = N; d.G = G; d.Q = Q;
    d.nc = (L + Q - 1) / Q;
    return d;
}

}  // namespace

namespace ssd {
int record_cuda_error(cudaError_t e) { return (int)cuda_fail(e); }
}  // namespace ssd

namespace {

size_t path_ws(const ssd::ScanDims &d, int chosen) {
    return chosen == SSD_PATH_TENSOR ? ssd::tc_workspace_bytes(d) : ssd::simt_workspace_bytes(d);
}

}  // namespace

extern "C" {

int ssd_version(void) { return (1 << 16) | 3; }

ssd_status ssd_set_test_fault(int kind) {
    if (kind != 0 && kind != 1) return SSD_ERR_INVALID_ARG;
    ssd::tc_set_test_fault(kind);
    return SSD_OK;
}

int ssd_last_cuda_error(void) { return g_last_cuda_error; }

const char *ssd_status_string(int s) {
    switch (s) {
        case SSD_OK: return "ok";
        case SSD_ERR_INVALID_ARG: return "invalid argument";
        case SSD_ERR_UNSUPPORTED: return "unsupported dtype, path or size";
        case SSD_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
        case SSD_ERR_WORKSPACE: return "workspace missing or too small";
        case SSD_ERR_CUDA: return "CUDA error";
        case SSD_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
        case SSD_ERR_PRECONDITION:
            return "precondition violated on device (A > 0, or a tensor-path operand outside the fp16 range)";
        default: return "unknown status";
    }
}

ssd_status ssd_chunk_scan_workspace_size(int64_t batch, int64_t seqlen, int64_t nheads,
                                         int64_t head_dim, int64_t state_dim, int64_t ngroups,
                                         int64_t chunk_size, int in_dtype, int path, size_t *bytes) {
    if (!bytes) return SSD_ERR_INVALID_ARG;
    ssd_status st = check_scan_dims(batch, seqlen, nheads, head_dim, state_dim, ngroups, chunk_size,
                                    in_dtype, path);
    if (st != SSD_OK) return st;
    const ssd::ScanDims d = make_dims(batch, seqlen, nheads, head_dim, state_dim, ngroups, chunk_size);
    int chosen = 0;
    if ((st = resolve_path(d, in_dtype, path, &chosen)) != SSD_OK) return st;
    *bytes = path_ws(d, chosen);
    return SSD_OK;
}

namespace {

// The forward scan, with or without the chunk-boundary states and packed rows.
ssd_status scan_fwd(const void *x, const float *dt_raw, const float *dt_bias, const float *A, const void *B,
                    const void *C, const float *D, const float *init_state, const int32_t *seq_idx, float *y,
                    float *final_state, float *chunk_states, int64_t batch, int64_t seqlen, int64_t nheads,
                    int64_t head_dim, int64_t state_dim, int64_t ngroups, int64_t chunk_size, float dt_lo,
                    float dt_hi, int in_dtype, int path, void *workspace, size_t workspace_bytes, void *stream,
                    const float *conv_w = nullptr, const float *conv_b = nullptr) {
    ssd_status st = check_scan_dims(batch, seqlen, nheads, head_dim, state_dim, ngroups, chunk_size,
                                    in_dtype, path);
    if (st != SSD_OK) return st;
    if (!limits_ok(dt_lo, dt_hi)) return SSD_ERR_INVALID_ARG;
    if (!dt_bias || !A || !D) return SSD_ERR_INVALID_ARG;
    const bool has_tokens = batch > 0 && seqlen > 0;
    // the combined arrangement: x is xbc, B and C are inside it
    const bool conv = conv_w != nullptr;
    if (conv && (!conv_b || !aligned16(conv_w) || !aligned16(conv_b)))
        return !conv_b ? SSD_ERR_INVALID_ARG : SSD_ERR_ALIGNMENT;
    if (has_tokens && (!x || !dt_raw || (!conv && (!B || !C)) || !y)) return SSD_ERR_INVALID_ARG;
    if ((x && !aligned16(x)) || (B && !aligned16(B)) || (C && !aligned16(C)) || (y && !aligned16(y)) ||
        (init_state && !aligned16(init_state)) || (final_state && !aligned16(final_state)) ||
        (chunk_states && !aligned16(chunk_states)))
        return SSD_ERR_ALIGNMENT;
    const ssd::ScanDims d = make_dims(batch, seqlen, nheads, head_dim, state_dim, ngroups, chunk_size);
    if (seq_idx && (reinterpret_cast<uintptr_t>(seq_idx) & 3u)) return SSD_ERR_ALIGNMENT;
    int chosen = 0;
    if ((st = resolve_path(d, in_dtype, path, &chosen)) != SSD_OK) return st;
    // the tensor path has the state at its 128-token block ends only
    if (chunk_states && chosen == SSD_PATH_TENSOR && chunk_size % 128 != 0) return SSD_ERR_UNSUPPORTED;
    if (!workspace || workspace_bytes < path_ws(d, chosen)) return SSD_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SSD_ERR_ALIGNMENT;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(workspace, 0, ssd::kStatusBytes, s);
    if (e != cudaSuccess) return cuda_fail(e);
    if (batch == 0) return SSD_OK;
    const size_t state_bytes = (size_t)batch * nheads * state_dim * head_dim * sizeof(float);
    if (seqlen == 0) {
        // no tokens: the state leaves as it came in
        if (final_state) {
            e = init_state ? cudaMemcpyAsync(final_state, init_state, state_bytes, cudaMemcpyDeviceToDevice, s)
                           : cudaMemsetAsync(final_state, 0, state_bytes, s);
            if (e != cudaSuccess) return cuda_fail(e);
        }
        return SSD_OK;
    }

    ssd::ScanArgs a;
    a.x = x; a.dt_raw = dt_raw; a.dt_bias = dt_bias; a.A = A; a.B = B; a.C = C; a.D = D;
    a.init_state = init_state; a.y = y; a.final_state = final_state; a.chunk_states = chunk_states;
    a.seq_idx = seq_idx;
    a.dt_lo = dt_lo; a.dt_hi = dt_hi; a.bf16 = in_dtype == SSD_BF16;
    if (conv) {
        a.conv_w = conv_w;
        a.conv_b = conv_b;
        a.Cd = nheads * head_dim + 2 * ngroups * state_dim;
    }
    e = chosen == SSD_PATH_TENSOR ? ssd::tc_scan(a, d, workspace, s) : ssd::simt_scan(a, d, workspace, s);
    if (e != cudaSuccess) return cuda_fail(e);
    return SSD_OK;
}

}  // namespace

ssd_status ssd_chunk_scan_fwd(const void *x, const float *dt_raw, const float *dt_bias,
                              const float *A, const void *B, const void *C, const float *D,
                              const float *init_state, float *y, float *final_state,
                              int64_t batch, int64_t seqlen, int64_t nheads, int64_t head_dim,
                              int64_t state_dim, int64_t ngroups, int64_t chunk_size,
                              float dt_lo, float dt_hi, int in_dtype, int path,
                              void *workspace, size_t workspace_bytes, void *stream) {
    return scan_fwd(x, dt_raw, dt_bias, A, B, C, D, init_state, nullptr, y, final_state, nullptr, batch, seqlen,
                    nheads, head_dim, state_dim, ngroups, chunk_size, dt_lo, dt_hi, in_dtype, path, workspace,
                    workspace_bytes, stream);
}

ssd_status ssd_chunk_scan_fwd_states(const void *x, const float *dt_raw, const float *dt_bias,
                                     const float *A, const void *B, const void *C, const float *D,
                                     const float *init_state, float *y, float *final_state,
                                     float *chunk_states, int64_t batch, int64_t seqlen, int64_t nheads,
                                     int64_t head_dim, int64_t state_dim, int64_t ngroups,
                                     int64_t chunk_size, float dt_lo, float dt_hi, int in_dtype, int path,
                                     void *workspace, size_t workspace_bytes, void *stream) {
    return scan_fwd(x, dt_raw, dt_bias, A, B, C, D, init_state, nullptr, y, final_state, chunk_states, batch,
                    seqlen, nheads, head_dim, state_dim, ngroups, chunk_size, dt_lo, dt_hi, in_dtype, path, workspace,
                    workspace_bytes, stream);
}

ssd_status ssd_chunk_scan_fwd_varlen(const void *x, const float *dt_raw, const float *dt_bias,
                                     const float *A, const void *B, const void *C, const float *D,
                                     const float *init_state, const int32_t *seq_idx, float *y,
                                     float *final_state, float *chunk_states, int64_t batch, int64_t seqlen,
                                     int64_t nheads, int64_t head_dim, int64_t state_dim, int64_t ngroups,
                                     int64_t chunk_size, float dt_lo, float dt_hi, int in_dtype, int path,
                                     void *workspace, size_t workspace_bytes, void *stream) {
    return scan_fwd(x, dt_raw, dt_bias, A, B, C, D, init_state, seq_idx, y, final_state, chunk_states, batch,
                    seqlen, nheads, head_dim, state_dim, ngroups, chunk_size, dt_lo, dt_hi, in_dtype, path, workspace,
                    workspace_bytes, stream);
}

ssd_status ssd_conv_scan_fwd(const void *xbc, const float *conv_w, const float *conv_b, int64_t kernel_width,
                             const float *dt_raw, const float *dt_bias, const float *A, const float *D,
                             const float *init_state, float *y, float *final_state, int64_t batch, int64_t seqlen,
                             int64_t nheads, int64_t head_dim, int64_t state_dim, int64_t ngroups,
                             int64_t chunk_size, float dt_lo, float dt_hi, int in_dtype, void *workspace,
                             size_t workspace_bytes, void *stream) {
    if (!conv_w) return SSD_ERR_INVALID_ARG;
    // the tensor path's shapes, bf16, width 4 (the conv runs inside its kernels)
    if (kernel_width != 4 || in_dtype != SSD_BF16) return SSD_ERR_UNSUPPORTED;
    return scan_fwd(xbc, dt_raw, dt_bias, A, nullptr, nullptr, D, init_state, nullptr, y, final_state, nullptr, batch,
                    seqlen, nheads, head_dim, state_dim, ngroups, chunk_size, dt_lo, dt_hi, in_dtype, SSD_PATH_TENSOR,
                    workspace, workspace_bytes, stream, conv_w, conv_b);
}

ssd_status ssd_chunk_scan_bwd_workspace_size(int64_t batch, int64_t seqlen, int64_t nheads, int64_t head_dim,
                                             int64_t state_dim, int64_t ngroups, int64_t chunk_size, int in_dtype,
                                             size_t *bytes) {
    if (!bytes) return SSD_ERR_INVALID_ARG;
    ssd_status st = check_scan_dims(batch, seqlen, nheads, head_dim, state_dim, ngroups, chunk_size, in_dtype,
                                    SSD_PATH_SIMT);
    if (st != SSD_OK) return st;
    const ssd::ScanDims d = make_dims(batch, seqlen, nheads, head_dim, state_dim, ngroups, chunk_size);
    if (!ssd::bwd_supported(d)) return SSD_ERR_UNSUPPORTED;
    *bytes = ssd::bwd_workspace_bytes(d);
    return SSD_OK;
}

ssd_status ssd_chunk_scan_bwd_varlen(const void *x, const float *dt_raw, const float *dt_bias, const float *A,
                                     const void *B, const void *C, const float *D, const float *init_state,
                                     const int32_t *seq_idx, const float *dy, const float *dfinal_state,
                                     float *dx, float *ddt_raw, float *ddt_bias, float *dA, float *dB, float *dC,
                                     float *dD, float *dinit_state, int64_t batch, int64_t seqlen, int64_t nheads,
                                     int64_t head_dim, int64_t state_dim, int64_t ngroups, int64_t chunk_size,
                                     float dt_lo, float dt_hi, int in_dtype, int path, void *workspace,
                                     size_t workspace_bytes, void *stream) {
    ssd_status st = check_scan_dims(batch, seqlen, nheads, head_dim, state_dim, ngroups, chunk_size, in_dtype,
                                    path);
    if (st != SSD_OK) return st;
    if (!limits_ok(dt_lo, dt_hi)) return SSD_ERR_INVALID_ARG;
    if (!dt_bias || !A || !D || !ddt_bias || !dA || !dD) return SSD_ERR_INVALID_ARG;
    const bool has_tokens = batch > 0 && seqlen > 0;
    if (has_tokens && (!x || !dt_raw || !B || !C || !dy || !dx || !ddt_raw || !dB || !dC))
        return SSD_ERR_INVALID_ARG;
    const void *al[] = {x, B, C, init_state, dy, dfinal_state, dx, dB, dC, dinit_state};
    for (const void *p : al)
        if (p && !aligned16(p)) return SSD_ERR_ALIGNMENT;
    if ((reinterpret_cast<uintptr_t>(dt_raw) | reinterpret_cast<uintptr_t>(ddt_raw) |
         reinterpret_cast<uintptr_t>(seq_idx)) & 3u)
        return SSD_ERR_ALIGNMENT;
    const ssd::ScanDims d = make_dims(batch, seqlen, nheads, head_dim, state_dim, ngroups, chunk_size);
    if (!ssd::bwd_supported(d)) return SSD_ERR_UNSUPPORTED;
    const bool tc = ssd::bwd_tc_supported(d, in_dtype == SSD_BF16, seq_idx != nullptr);
    if (path == SSD_PATH_TENSOR && !tc) return SSD_ERR_UNSUPPORTED;
    const bool use_tc = tc && path != SSD_PATH_SIMT;
    if (!workspace || workspace_bytes < ssd::bwd_workspace_bytes(d)) return SSD_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SSD_ERR_ALIGNMENT;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(workspace, 0, ssd::kStatusBytes, s);
    if (e != cudaSuccess) return cuda_fail(e);
    if (!has_tokens) {
        // no tokens: the per-head sums are zero and the seed passes to the initial state as it is
        const size_t hb = (size_t)nheads * sizeof(float);
        if ((e = cudaMemsetAsync(dA, 0, hb, s)) != cudaSuccess || (e = cudaMemsetAsync(dD, 0, hb, s)) != cudaSuccess ||
            (e = cudaMemsetAsync(ddt_bias, 0, hb, s)) != cudaSuccess)
            return cuda_fail(e);
        if (dinit_state && batch > 0) {
            const size_t sb = (size_t)batch * nheads * state_dim * head_dim * sizeof(float);
            e = dfinal_state ? cudaMemcpyAsync(dinit_state, dfinal_state, sb, cudaMemcpyDeviceToDevice, s)
                             : cudaMemsetAsync(dinit_state, 0, sb, s);
            if (e != cudaSuccess) return cuda_fail(e);
        }
        return SSD_OK;
    }
    ssd::BwdArgs a;
    a.f.x = x; a.f.dt_raw = dt_raw; a.f.dt_bias = dt_bias; a.f.A = A; a.f.B = B; a.f.C = C; a.f.D = D;
    a.f.init_state = init_state; a.f.y = nullptr; a.f.final_state = nullptr;
    a.f.seq_idx = seq_idx;
    a.f.dt_lo = dt_lo; a.f.dt_hi = dt_hi; a.f.bf16 = in_dtype == SSD_BF16;
    a.tensor = use_tc ? 1 : 0;
    a.dy = dy; a.dfinal = dfinal_state;
    a.dx = dx; a.ddt_raw = ddt_raw; a.ddt_bias = ddt_bias; a.dA = dA; a.dB = dB; a.dC = dC; a.dD = dD;
    a.dinit = dinit_state;
    e = ssd::bwd_scan(a, d, workspace, s);
    if (e != cudaSuccess) return cuda_fail(e);
    return SSD_OK;
}

ssd_status ssd_chunk_scan_bwd(const void *x, const float *dt_raw, const float *dt_bias, const float *A,
                              const void *B, const void *C, const float *D, const float *init_state,
                              const float *dy, const float *dfinal_state, float *dx, float *ddt_raw,
                              float *ddt_bias, float *dA, float *dB, float *dC, float *dD, float *dinit_state,
                              int64_t batch, int64_t seqlen, int64_t nheads, int64_t head_dim, int64_t state_dim,
                              int64_t ngroups, int64_t chunk_size, float dt_lo, float dt_hi, int in_dtype,
                              void *workspace, size_t workspace_bytes, void *stream) {
    return ssd_chunk_scan_bwd_varlen(x, dt_raw, dt_bias, A, B, C, D, init_state, nullptr, dy, dfinal_state, dx,
                                     ddt_raw, ddt_bias, dA, dB, dC, dD, dinit_state, batch, seqlen, nheads, head_dim,
                                     state_dim, ngroups, chunk_size, dt_lo, dt_hi, in_dtype, SSD_PATH_SIMT,
                                     workspace, workspace_bytes, stream);
}

ssd_status ssd_step(const void *x, const float *dt_raw, const float *dt_bias, const float *A,
                    const void *B, const void *C, const float *D, float *state, float *y,
                    int64_t batch, int64_t nheads, int64_t head_dim, int64_t state_dim,
                    int64_t ngroups, float dt_lo, float dt_hi, int in_dtype, void *stream) {
    if (batch < 0 || nheads <= 0 || head_dim <= 0 || state_dim <= 0 || ngroups <= 0) return SSD_ERR_INVALID_ARG;
    if (nheads % ngroups != 0 || !limits_ok(dt_lo, dt_hi)) return SSD_ERR_INVALID_ARG;
    if (!dtype_ok(in_dtype)) return SSD_ERR_UNSUPPORTED;
    if (!ssd::step_supported(head_dim, state_dim) || batch * nheads > 0x7fffffffll) return SSD_ERR_UNSUPPORTED;
    if (batch == 0) return SSD_OK;
    if (!x || !dt_raw || !dt_bias || !A || !B || !C || !D || !state || !y) return SSD_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(B) || !aligned16(C) || !aligned16(state) || !aligned16(y))
        return SSD_ERR_ALIGNMENT;
    ssd::StepArgs a;
    a.x = x; a.dt_raw = dt_raw; a.dt_bias = dt_bias; a.A = A; a.B = B; a.C = C; a.D = D;
    a.state = state; a.y = y;
    a.b = batch; a.H = nheads; a.P = head_dim; a.N = state_dim; a.G = ngroups;
    a.dt_lo = dt_lo; a.dt_hi = dt_hi; a.bf16 = in_dtype == SSD_BF16;
    cudaError_t e = ssd::step_launch(a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e);
    return SSD_OK;
}

ssd_status ssd_read_device_status(const void *workspace, void *stream) {
    unsigned word = 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (!workspace) {
        e = ssd::front_status_read(s, &word);
    } else {
        e = cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    }
    if (e != cudaSuccess) return cuda_fail(e);
    if (word & ssd::kStatusTimeout) return SSD_ERR_DEVICE_TIMEOUT;
    if (word & (ssd::kStatusPrecondition | ssd::kStatusRange)) return SSD_ERR_PRECONDITION;
    return SSD_OK;
}

}  // extern "C"
