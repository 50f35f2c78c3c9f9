// Internal launcher interface between the C ABI (ssd_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace ssd {

struct ScanDims {
    int64_t b, L, H, P, N, G, Q;   // batch, seqlen, heads, head_dim, state_dim, groups, chunk
    int64_t nc;                    // ceil(L / Q)
};

struct ScanArgs {
    const void *x;
    const float *dt_raw, *dt_bias, *A;
    const void *B, *C;
    const float *D, *init_state;
    float *y, *final_state;
    float *chunk_states = nullptr;  // [b, nc, H, N, P] or null: the state after every chunk
    const int32_t *seq_idx = nullptr;  // [b, L] document ids of packed rows, or null (SIMT path)
    float dt_lo, dt_hi;
    int bf16;                      // 1: x/B/C are bfloat16, 0: float32
    // the combined arrangement (tensor path): x points at xbc [b, L, Cd] (the
    // conv's input, channels x | B | C), B and C are unused, and x, B, C are
    // conv1d + SiLU of xbc computed inside the scan's kernels (width 4)
    const float *conv_w = nullptr;  // [Cd, 4]
    const float *conv_b = nullptr;  // [Cd]
    int64_t Cd = 0;
};

struct StepArgs {
    const void *x;
    const float *dt_raw, *dt_bias, *A;
    const void *B, *C;
    const float *D;
    float *state, *y;
    int64_t b, H, P, N, G;
    float dt_lo, dt_hi;
    int bf16;
};

// Records `e` as the last CUDA error of this host thread; returns SSD_ERR_CUDA (5).
int record_cuda_error(cudaError_t e);

// Workspace carve-up: [status | per-path regions], every region 256-byte aligned.
inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// ---- SIMT fp32 path (any chunk size) --------------------------------------
// Its workspace after the status region (every region 256-byte aligned).
struct SimtWs {
    unsigned *status;
    float *dtv;     // [b, H, L]  dt
    float *cum;     // [b, H, L]  within-chunk inclusive cumsum of dt * A
    float *ell;     // [b, H, nc] chunk log decay (cum at the chunk's last token)
    float *states;  // [b, H, nc, N, P]  after the state pass: the state entering each chunk
};
SimtWs simt_carve(const ScanDims &d, void *workspace);
bool simt_supported(const ScanDims &d);
size_t simt_workspace_bytes(const ScanDims &d);
cudaError_t simt_scan(const ScanArgs &a, const ScanDims &d, void *workspace, cudaStream_t s);
// The first two launches of simt_scan alone (no y): fills dtv, cum, ell and
// the entering states; writes final_state / chunk_states when not null.
cudaError_t simt_scan_states(const ScanArgs &a, const ScanDims &d, void *workspace, cudaStream_t s);
// Launch 2 of simt_scan alone: the chunk states already in the workspace
// (with dtv, cum, ell) become the states entering each chunk.
cudaError_t simt_state_pass(const ScanArgs &a, const ScanDims &d, void *workspace, cudaStream_t s);

// ---- backward of the scan (SIMT fp32, deterministic) -----------------------
struct BwdArgs {
    ScanArgs f;                    // the forward's inputs (y, final_state, chunk_states unused)
    const float *dy, *dfinal;      // [b,L,H,P], [b,H,N,P] or null
    float *dx, *ddt_raw, *ddt_bias, *dA, *dB, *dC, *dD, *dinit;
    int tensor = 0;                // 1: the tensor-core pair kernels (bwd_tc_supported)
};
bool bwd_supported(const ScanDims &d);

// The tensor-core pair kernels of the backward (ssd_scan_bwd_tc.cu): the
// same outputs as the CUDA-core `cols` and `rows` kernels, from the same
// workspace (the forward recompute's dt, cum and entering states, the
// reverse pass's G_c).  bf16 inputs, P 64, N 128, Q a multiple of 128.
struct BwdPairArgs {
    const void *x, *B, *C;         // bf16 inputs
    const float *D, *dy;
    const float *dtv, *cum;        // [b, H, L]
    const float *gst, *states;     // [b, H, nc, N, P]: G_c, H_in
    float *ddt_dir, *dcum_col, *dcum_row, *E, *dyx;  // [b, H, L]
    float *dx;                     // [b, L, H, P]
    float *dBh, *dCh;              // [b, L, H, N] per head
    unsigned *status;
    const float *docc = nullptr;   // [b, L] packed rows: document starts from the chunk's first token
                                   // through each token (null: one document per row)
};
bool bwd_tc_supported(const ScanDims &d, int bf16, int packed);
cudaError_t bwd_tc_pairs(const BwdPairArgs &a, const ScanDims &d, cudaStream_t s);
// The forward recompute's first launch and the backward's per-chunk sums on
// the tensor cores, for the same shapes: dt, cum and the chunk log decay
// (ell), the chunk state S_c = sum_j e^{cl-cum_j} dt_j B_j x_j^T into
// `states`, and sum_i e^{cum_i} C_i dy_i^T into `gst`, per (chunk, head,
// batch).  The state passes run after it as before.
struct BwdStatesArgs {
    const void *x, *B, *C;          // bf16
    const float *dt_raw, *dt_bias, *A, *dy;
    float dt_lo, dt_hi;
    float *dtv, *cum, *ell;         // [b, H, L], [b, H, L], [b, H, nc]
    float *states, *gst;            // [b, H, nc, N, P]
    unsigned *status;
    const float *docc = nullptr;    // as in BwdPairArgs
};
cudaError_t bwd_tc_states(const BwdStatesArgs &a, const ScanDims &d, cudaStream_t s);
size_t bwd_workspace_bytes(const ScanDims &d);
cudaError_t bwd_scan(const BwdArgs &a, const ScanDims &d, void *workspace, cudaStream_t s);

// ---- tcgen05 tensor-core path -----------------------------------------------
bool tc_supported(const ScanDims &d, int bf16);
size_t tc_workspace_bytes(const ScanDims &d);
cudaError_t tc_scan(const ScanArgs &a, const ScanDims &d, void *workspace, cudaStream_t s);
// Test hook for the device-side timeout path (ssd_set_test_fault): 0 = off;
// 1 = the tensor-path chunk-output kernel never requests its first C and B
// tiles and its waits give up after about a millisecond.
void tc_set_test_fault(int kind);
int tc_test_fault();

// ---- decode step ------------------------------------------------------------
bool step_supported(int64_t P, int64_t N);
cudaError_t step_launch(const StepArgs &a, cudaStream_t s);

// Reads and clears the status word of the kernels that take no workspace
// (conv1d); waits for `s`.
cudaError_t front_status_read(cudaStream_t s, unsigned *word);

}  // namespace ssd
