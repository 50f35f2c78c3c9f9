/*
 * ssd.h -- C ABI of libssd.so, the B200 (sm_100a) Mamba-2 SSD scan.
 *
 * The operation (nnterp guide "Mamba-2", opening paragraph and the table in
 * "The values"): per head h, with state S an N x P matrix stored state_dim
 * first ("key side first"), for every token t
 *     dt  = clamp(softplus(dt_raw[t,h] + dt_bias[h]), dt_lo, dt_hi)
 *     S   = exp(dt * A[h]) * S + dt * B[t,g] (outer) x[t,h]
 *     y   = S^T C[t,g] + D[h] * x[t,h]
 * where head h reads the B and C of group g = h / (H / G) (B and C are "one
 * per group of heads").  A * dt is the log decay and must be <= 0.
 *
 * Conventions shared by every entry point
 *   - Pointers are DEVICE pointers unless stated; the caller allocates and
 *     owns every buffer, workspace included.  The library never allocates,
 *     frees or synchronises on the compute calls; work is enqueued on
 *     `stream` (a cudaStream_t; NULL is the legacy default stream) and the
 *     call returns before it finishes.
 *   - Layouts are contiguous, row-major, with these shapes:
 *       x            [batch, seqlen, nheads, head_dim]     in_dtype
 *       dt_raw       [batch, seqlen, nheads]               float32
 *       dt_bias, A, D [nheads]                             float32
 *       B, C         [batch, seqlen, ngroups, state_dim]   in_dtype
 *       init_state, final_state, state
 *                    [batch, nheads, state_dim, head_dim]  float32
 *       y            [batch, seqlen, nheads, head_dim]     float32
 *     (the decode step drops the seqlen axis).
 *   - x, B, C, y and every state pointer must be 16-byte aligned.
 *   - Errors come back as an ssd_status; nothing is thrown across the ABI.
 *     Argument errors are detected on the host before anything is enqueued.
 *     Conditions only the GPU can see (a positive A in the chunked scan) are
 *     recorded in a status word at the start of the workspace and read back
 *     with ssd_read_device_status().
 */
#ifndef SSD_H_
#define SSD_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SSD_API __attribute__((visibility("default")))
#else
#define SSD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum ssd_status {
    SSD_OK = 0,
    SSD_ERR_INVALID_ARG = 1,    /* null pointer, size <= 0, H % G != 0, bad dt limits */
    SSD_ERR_UNSUPPORTED = 2,    /* dtype, path or size outside what is implemented */
    SSD_ERR_ALIGNMENT = 3,      /* a pointer is not 16-byte aligned */
    SSD_ERR_WORKSPACE = 4,      /* workspace null or smaller than ssd_chunk_scan_workspace_size() */
    SSD_ERR_CUDA = 5,           /* a CUDA call failed; see ssd_last_cuda_error() */
    SSD_ERR_DEVICE_TIMEOUT = 6, /* a bounded device-side wait gave up */
    SSD_ERR_PRECONDITION = 7    /* the GPU saw A > 0 (the log decay must be non-positive), or on the
                                   tensor path an operand outside the fp16 range (|v| > 65504).  The
                                   tensor path detects the latter as a non-finite y or final state
                                   (an fp16 overflow always reaches one of them), so non-finite
                                   inputs report it too */
} ssd_status;

typedef enum ssd_dtype {
    SSD_F32 = 0,   /* float32 x, B, C */
    SSD_BF16 = 1   /* bfloat16 x, B, C */
} ssd_dtype;

typedef enum ssd_path {
    SSD_PATH_AUTO = 0,    /* tensor-core path when the shape allows it, else SIMT */
    SSD_PATH_SIMT = 1,    /* fp32 CUDA-core kernels: any chunk size, fp32 or bf16 inputs */
    SSD_PATH_TENSOR = 2   /* tcgen05 kernels: bf16 inputs, state_dim 128, head_dim 64,
                             chunk size 64, 128 or 256; fp16 operands, fp32 accumulate */
} ssd_path;

/* Bytes of device workspace ssd_chunk_scan_fwd needs for these sizes and
 * this path (SSD_PATH_AUTO resolves as the forward call would).  Host only;
 * enqueues nothing.  Returns SSD_ERR_INVALID_ARG / SSD_ERR_UNSUPPORTED for
 * sizes the forward call would reject. */
SSD_API ssd_status ssd_chunk_scan_workspace_size(int64_t batch, int64_t seqlen, int64_t nheads,
                                         int64_t head_dim, int64_t state_dim, int64_t ngroups,
                                         int64_t chunk_size, int in_dtype, int path,
                                         size_t *bytes);

/* Chunked forward scan over whole sequences (the prompt path: nnterp guide
 * "Mamba-2", sections "The values" and "The state after every token";
 * chunked two-stage evaluation as on the "Mamba2" knowledge page).
 *
 * Evaluates the recurrence above for every (batch, head) from init_state
 * (NULL means zeros, a fresh prompt) and writes y for every token and
 * final_state, the state after the last token (final_state may be NULL when
 * not wanted).  The work is split into chunks of chunk_size tokens: within a
 * chunk a masked, decay-weighted C.B^T contraction; between chunks a serial
 * pass of the chunk states.  The result equals the token-by-token recurrence
 * up to rounding, whatever the chunk size.
 *   dt_lo, dt_hi  the time-step limit applied after the softplus
 *                 (0 and +INFINITY for no limit); 0 <= dt_lo <= dt_hi.
 *   in_dtype      ssd_dtype of x, B and C.
 *   path          ssd_path.
 *   workspace     device scratch of at least ssd_chunk_scan_workspace_size()
 *                 bytes, 256-byte aligned; its first 256 bytes hold the
 *                 device status word.  It is overwritten by every call, so
 *                 two calls in flight at once need two workspaces.
 * Inputs are never modified.  y, final_state and the workspace must not
 * overlap the inputs. */
SSD_API ssd_status ssd_chunk_scan_fwd(const void *x, const float *dt_raw, const float *dt_bias,
                              const float *A, const void *B, const void *C, const float *D,
                              const float *init_state, float *y, float *final_state,
                              int64_t batch, int64_t seqlen, int64_t nheads, int64_t head_dim,
                              int64_t state_dim, int64_t ngroups, int64_t chunk_size,
                              float dt_lo, float dt_hi, int in_dtype, int path,
                              void *workspace, size_t workspace_bytes, void *stream);

/* ssd_chunk_scan_fwd that also writes the chunk-boundary states (nnterp
 * guide "Mamba-2", section "The state after every token": the chunk scan
 * holds the state at every chunk boundary, and with chunk_size 1 every token
 * is one).
 *   chunk_states  [batch, nchunks, nheads, state_dim, head_dim] float32 out,
 *                 nchunks = ceil(seqlen / chunk_size).  Chunk c holds the
 *                 state after token min((c+1) chunk_size, seqlen) - 1, so the
 *                 last one equals final_state.  16-byte aligned; must not
 *                 overlap the inputs, y, final_state or the workspace.  NULL
 *                 makes the call ssd_chunk_scan_fwd.
 * Every other argument is as for ssd_chunk_scan_fwd, the workspace sized by
 * ssd_chunk_scan_workspace_size for the same path.  The tensor-core path
 * holds the state only at the ends of its 128-token blocks: when the call
 * resolves to it (SSD_PATH_TENSOR, or SSD_PATH_AUTO on a shape it takes), a
 * chunk_size that is not a multiple of 128 returns SSD_ERR_UNSUPPORTED before
 * anything is enqueued.  SSD_PATH_SIMT takes any chunk size. */
SSD_API ssd_status ssd_chunk_scan_fwd_states(const void *x, const float *dt_raw, const float *dt_bias,
                                     const float *A, const void *B, const void *C, const float *D,
                                     const float *init_state, float *y, float *final_state,
                                     float *chunk_states, int64_t batch, int64_t seqlen, int64_t nheads,
                                     int64_t head_dim, int64_t state_dim, int64_t ngroups,
                                     int64_t chunk_size, float dt_lo, float dt_hi, int in_dtype, int path,
                                     void *workspace, size_t workspace_bytes, void *stream);

/* One decode token (nnterp guide "Mamba-2", section "The state between
 * steps": the update writes the new state into the cache and returns only y;
 * there is no sequence axis).
 *   x [batch, nheads, head_dim], dt_raw [batch, nheads],
 *   B, C [batch, ngroups, state_dim], state [batch, nheads, state_dim, head_dim]
 *   float32, updated IN PLACE; y [batch, nheads, head_dim] float32 out.
 *   dt_lo, dt_hi  as for the scan; pass 0 and +INFINITY for the pages'
 *                 decode semantics (no clamp).
 * head_dim must be a multiple of 4 with head_dim / 4 dividing 256.  A > 0 is
 * evaluated as written (nothing in the step depends on its sign). */
SSD_API ssd_status ssd_step(const void *x, const float *dt_raw, const float *dt_bias, const float *A,
                    const void *B, const void *C, const float *D, float *state, float *y,
                    int64_t batch, int64_t nheads, int64_t head_dim, int64_t state_dim,
                    int64_t ngroups, float dt_lo, float dt_hi, int in_dtype, void *stream);

/* ssd_chunk_scan_fwd without a caller-provided workspace.  The pages have no
 * counterpart: this entry point exists for callers that cannot allocate
 * device memory -- code that runs where cudaMalloc is forbidden or unsafe
 * (inside a host callback, a plug-in of another runtime that owns every
 * allocation, a memory-capped sandbox) or that is handed only its input and
 * output buffers.  The scratch it needs lives in a fixed 32 MiB device array
 * inside libssd.so, which every GPU that loads the library holds until the
 * process exits.  Arguments are those of ssd_chunk_scan_fwd minus the
 * workspace; inputs and outputs are still the caller's.
 *   - Sizes whose workspace (ssd_chunk_scan_workspace_size) exceeds 32 MiB
 *     are rejected with SSD_ERR_UNSUPPORTED before anything is enqueued.
 *   - It never calls cudaMalloc, cudaFree or any allocating routine.
 *   - The first call on each device looks the array's device address up
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture.  The address is kept per device index and
 *     holds for the device's primary context, the one the CUDA runtime and
 *     PyTorch use: after cudaDeviceReset, or from a context made current
 *     through the driver API, it no longer names the array.
 *   - Every call shares the one array and it keeps the last call's contents
 *     (each call clears the part that must start at zero).  Calls whose work
 *     overlaps on the GPU -- two streams, or two host threads -- race on it;
 *     serialise them.
 *   - The device status word sits in that array and is not read back here:
 *     host-side errors come back as usual, device-side conditions
 *     (SSD_ERR_PRECONDITION) are only visible through ssd_chunk_scan_fwd. */
SSD_API ssd_status ssd_chunk_scan_fwd_noalloc(const void *x, const float *dt_raw, const float *dt_bias,
                                      const float *A, const void *B, const void *C, const float *D,
                                      const float *init_state, float *y, float *final_state,
                                      int64_t batch, int64_t seqlen, int64_t nheads, int64_t head_dim,
                                      int64_t state_dim, int64_t ngroups, int64_t chunk_size,
                                      float dt_lo, float dt_hi, int in_dtype, int path, void *stream);

/* ssd_chunk_scan_fwd_states over packed rows (the "Mamba2" knowledge page:
 * sample packing for Mamba2).
 *   seq_idx  [batch, seqlen] int32, 4-byte aligned: a document id per token.
 *            A token whose id differs from the previous token's starts a new
 *            document: the state is zero before its update, so no token
 *            reads across a document start.  The first document of a row
 *            starts from init_state (NULL: zeros).  final_state is the state
 *            after the row's last token (its last document's) and
 *            chunk_states (may be NULL) as for ssd_chunk_scan_fwd_states.
 *            NULL makes the call ssd_chunk_scan_fwd_states.
 * Both paths take packed rows and resolve as for ssd_chunk_scan_fwd (the
 * workspace is sized the same way).  Every other argument as for
 * ssd_chunk_scan_fwd_states. */
SSD_API ssd_status ssd_chunk_scan_fwd_varlen(const void *x, const float *dt_raw, const float *dt_bias,
                                     const float *A, const void *B, const void *C, const float *D,
                                     const float *init_state, const int32_t *seq_idx, float *y,
                                     float *final_state, float *chunk_states, int64_t batch, int64_t seqlen,
                                     int64_t nheads, int64_t head_dim, int64_t state_dim, int64_t ngroups,
                                     int64_t chunk_size, float dt_lo, float dt_hi, int in_dtype, int path,
                                     void *workspace, size_t workspace_bytes, void *stream);

/* The causal depthwise conv1d that runs before the scan in a Mamba-2 layer
 * (state-spaces/mamba issue on the training and inference paths:
 * causal_conv1d_fn, then the chunk scan), in the split arrangement: it
 * writes the scan's x, B and C directly.  For every channel c of
 *   xbc [batch, seqlen, Cd],  Cd = nheads*head_dim + 2*ngroups*state_dim
 *   (channels in the order x | B | C, the same dtype as the outputs),
 *   out[t, c] = silu(bias[c] + sum_{k<K} weight[c, k] * xbc[t - (K-1) + k, c]),
 *   xbc[t < 0] = 0 (a fresh sequence),  silu(u) = u / (1 + exp(-u)),
 * and out is split into x [batch, seqlen, nheads, head_dim] and
 * B, C [batch, seqlen, ngroups, state_dim].
 *   weight [Cd, K] and bias [Cd] float32; K = kernel_width, 1..4.
 *   in_dtype  ssd_dtype of xbc, x, B, C.
 * nheads*head_dim and ngroups*state_dim must be multiples of 8; xbc, x, B
 * and C 16-byte aligned and not overlapping; seqlen below 2^31 - 128 and
 * seqlen*Cd*4 below 2^40 (SSD_ERR_UNSUPPORTED otherwise).  Queued on
 * `stream`.  Its waits on its own copies are bounded: one that gives up
 * (about 2 s) leaves SSD_ERR_DEVICE_TIMEOUT for ssd_read_device_status(NULL,
 * stream), and the outputs undefined. */
SSD_API ssd_status ssd_conv1d_silu_split(const void *xbc, const float *weight, const float *bias, void *x,
                                 void *B, void *C, int64_t batch, int64_t seqlen, int64_t nheads,
                                 int64_t head_dim, int64_t ngroups, int64_t state_dim,
                                 int64_t kernel_width, int in_dtype, void *stream);

/* The conv1d and the scan in the combined arrangement (the HF transformers
 * issue "mamba2 mixer different outputs" contrasts a fused
 * mamba_split_conv1d_scan_combined with causal_conv1d_fn followed by
 * mamba_chunk_scan_combined): y and final_state of ssd_chunk_scan_fwd on the
 * x, B and C that ssd_conv1d_silu_split would write from xbc, without writing
 * them.  The scan's kernels read xbc itself: each 128-token block's x tile
 * arrives with the 3 rows before it and is convolved in shared memory, and
 * the fp16 copies of B and C are convolved where they are made.  The
 * arithmetic is the split conv's (each value rounded to bf16 as that conv
 * stores it), so the two arrangements give the same bits.
 *   xbc      [batch, seqlen, Cd] bf16, Cd = nheads*head_dim + 2*ngroups*state_dim
 *            (channels x | B | C), 16-byte aligned
 *   conv_w   [Cd, 4] float32, conv_b [Cd] float32, both 16-byte aligned
 *            (SSD_ERR_ALIGNMENT) and neither NULL (SSD_ERR_INVALID_ARG)
 *   kernel_width  4 (else SSD_ERR_UNSUPPORTED)
 *   the rest as for ssd_chunk_scan_fwd on the tensor-core path: in_dtype
 *   SSD_BF16, head_dim 64, state_dim 128, chunk_size 64, 128 or 256 (else
 *   SSD_ERR_UNSUPPORTED); workspace of ssd_chunk_scan_workspace_size(...,
 *   SSD_PATH_TENSOR) bytes; status word as for ssd_chunk_scan_fwd.
 * No packed rows and no chunk states here (use the split arrangement).
 * Queued on `stream`. */
SSD_API ssd_status ssd_conv_scan_fwd(const void *xbc, const float *conv_w, const float *conv_b,
                                     int64_t kernel_width, const float *dt_raw, const float *dt_bias,
                                     const float *A, const float *D, const float *init_state, float *y,
                                     float *final_state, int64_t batch, int64_t seqlen, int64_t nheads,
                                     int64_t head_dim, int64_t state_dim, int64_t ngroups, int64_t chunk_size,
                                     float dt_lo, float dt_hi, int in_dtype, void *workspace,
                                     size_t workspace_bytes, void *stream);

/* The gated RMS norm that takes y after the scan (nnterp guide "Mamba-2",
 * table "The values": y is taken before the gated norm and out_proj):
 *   v = y * silu(z),  out = v / sqrt(mean_{group}(v^2) + eps) * weight
 * over each group of group_size consecutive channels of a token.
 *   y [tokens, dim] float32 (the scan's y viewed as [b*L, H*P]),
 *   z [tokens, dim] of z_dtype, weight [dim] float32, out [tokens, dim]
 *   float32.  dim a multiple of group_size, group_size a multiple of 4;
 *   y, weight and out 16-byte aligned, z 8-byte aligned; eps >= 0.
 * Queued on `stream`. */
SSD_API ssd_status ssd_gated_rmsnorm(const float *y, const void *z, const float *weight, float *out,
                             int64_t tokens, int64_t dim, int64_t group_size, float eps, int z_dtype,
                             void *stream);

/* Bytes of device workspace ssd_chunk_scan_bwd needs for these sizes.  Host
 * only.  SSD_ERR_UNSUPPORTED for sizes the backward does not take. */
SSD_API ssd_status ssd_chunk_scan_bwd_workspace_size(int64_t batch, int64_t seqlen, int64_t nheads,
                                             int64_t head_dim, int64_t state_dim, int64_t ngroups,
                                             int64_t chunk_size, int in_dtype, size_t *bytes);

/* Backward of the chunked scan, deterministic (the HF transformers issue
 * "mamba2 mixer different outputs" notes that the backward pass of the usual
 * mamba kernels is not; this one has no atomics and sums in a fixed order, so
 * repeated calls on the same inputs give the same bits).
 *
 * Given the forward's inputs (as for ssd_chunk_scan_fwd; packed rows through
 * ssd_chunk_scan_bwd_varlen) and
 * the gradients dy of y and dfinal_state of final_state, writes the gradient
 * of <dy, y> + <dfinal_state, final_state> with respect to every input:
 *   dy           [batch, seqlen, nheads, head_dim] float32 in
 *   dfinal_state [batch, nheads, state_dim, head_dim] float32 in, NULL = zeros
 *   dx           [batch, seqlen, nheads, head_dim] float32 out
 *   ddt_raw      [batch, seqlen, nheads] float32 out (4-byte aligned), zero
 *                where the time-step limit clamps softplus(dt_raw + dt_bias)
 *                strictly outside [dt_lo, dt_hi]
 *   ddt_bias, dA, dD  [nheads] float32 out
 *   dB, dC       [batch, seqlen, ngroups, state_dim] float32 out (the heads of
 *                a group summed)
 *   dinit_state  [batch, nheads, state_dim, head_dim] float32 out, or NULL
 *                when not wanted (written also when init_state is NULL)
 * Gradients are float32 whatever in_dtype is.  The states the gradients need
 * are recomputed from the inputs inside the call; nothing from a forward call
 * is reused.  The work runs on CUDA cores in fp32 in chunks of chunk_size
 * tokens (any chunk_size >= 1); head_dim must be 8, 16, 32 or 64 and
 * state_dim a multiple of 8 up to 128, else SSD_ERR_UNSUPPORTED.  16-byte
 * alignment as for the forward; outputs must not overlap the inputs or each
 * other; the workspace is at least ssd_chunk_scan_bwd_workspace_size() bytes,
 * 256-byte aligned, its status word read by ssd_read_device_status()
 * (SSD_ERR_PRECONDITION for A > 0). */
SSD_API ssd_status ssd_chunk_scan_bwd(const void *x, const float *dt_raw, const float *dt_bias, const float *A,
                              const void *B, const void *C, const float *D, const float *init_state,
                              const float *dy, const float *dfinal_state, float *dx, float *ddt_raw,
                              float *ddt_bias, float *dA, float *dB, float *dC, float *dD, float *dinit_state,
                              int64_t batch, int64_t seqlen, int64_t nheads, int64_t head_dim,
                              int64_t state_dim, int64_t ngroups, int64_t chunk_size, float dt_lo, float dt_hi,
                              int in_dtype, void *workspace, size_t workspace_bytes, void *stream);

/* ssd_chunk_scan_bwd over packed rows: the gradients of the forward of
 * ssd_chunk_scan_fwd_varlen with the same seq_idx ([batch, seqlen] int32,
 * 4-byte aligned; a token whose id differs from the previous token's starts a
 * document and the state is zero before its update).  No gradient crosses a
 * document start; dinit_state reaches only each row's first document.  NULL
 * seq_idx makes the call ssd_chunk_scan_bwd (on the path chosen below).
 * path (ssd_path):
 *   SSD_PATH_SIMT    the fp32 CUDA-core kernels, as ssd_chunk_scan_bwd;
 *   SSD_PATH_TENSOR  the products of two 128-token blocks (C.B^T, dy.x^T and
 *                    the accumulations into dx, dB, dC) on the tcgen05
 *                    tensor cores with fp16 operands and fp32 accumulation:
 *                    bf16 inputs, head_dim 64, state_dim 128, chunk_size a
 *                    multiple of 128 up to 1024 (else SSD_ERR_UNSUPPORTED);
 *                    packed rows included.  The gradients carry the forward
 *                    tensor path's precision (about 1e-3 of their RMS), and
 *                    a value outside fp16's range shows as
 *                    SSD_ERR_PRECONDITION in the status word;
 *   SSD_PATH_AUTO    the tensor path where it applies, else SIMT.
 * Same workspace size and determinism, and the other arguments as
 * ssd_chunk_scan_bwd. */
SSD_API ssd_status ssd_chunk_scan_bwd_varlen(const void *x, const float *dt_raw, const float *dt_bias,
                                     const float *A, const void *B, const void *C, const float *D,
                                     const float *init_state, const int32_t *seq_idx, const float *dy,
                                     const float *dfinal_state, float *dx, float *ddt_raw, float *ddt_bias,
                                     float *dA, float *dB, float *dC, float *dD, float *dinit_state,
                                     int64_t batch, int64_t seqlen, int64_t nheads, int64_t head_dim,
                                     int64_t state_dim, int64_t ngroups, int64_t chunk_size, float dt_lo,
                                     float dt_hi, int in_dtype, int path, void *workspace,
                                     size_t workspace_bytes, void *stream);

/* Waits for `stream`, then reads the device status word that the last
 * ssd_chunk_scan_fwd on this workspace left: SSD_OK, SSD_ERR_PRECONDITION or
 * SSD_ERR_DEVICE_TIMEOUT.  `workspace` is a device pointer.  With workspace
 * NULL it reads, and then clears, the current device's status word of the
 * kernels that take no workspace (ssd_conv1d_silu_split): SSD_OK or
 * SSD_ERR_DEVICE_TIMEOUT since the last such read. */
SSD_API ssd_status ssd_read_device_status(const void *workspace, void *stream);

/* Text for a status code (static storage; never NULL). */
SSD_API const char *ssd_status_string(int status);

/* The cudaError_t behind the last SSD_ERR_CUDA returned on this host thread. */
SSD_API int ssd_last_cuda_error(void);

/* Kernel tracing, off by default.  ssd_trace_enable(n) creates 2n CUDA
 * events once (n <= 8192), clears earlier records and from then on brackets
 * each kernel the library launches with an event pair recorded on the
 * launching stream, for the first n launches; ssd_trace_enable(0) stops
 * recording (records are kept).  ssd_trace_read() waits for the recorded
 * events of kernel id `kernel` (0 <= kernel < ssd_trace_kernel_count()) and
 * returns how many launches were recorded and their summed device time in
 * milliseconds.  ssd_trace_kernel_name() names a kernel id.  Not
 * thread-safe against concurrent compute calls from other host threads. */
SSD_API ssd_status ssd_trace_enable(int max_launches);
SSD_API ssd_status ssd_trace_read(int kernel, int *launches, double *total_ms);
SSD_API const char *ssd_trace_kernel_name(int kernel);
SSD_API int ssd_trace_kernel_count(void);

/* TEST ONLY: makes the device-side timeout path run, without any fault.
 * kind 1: from the next tensor-path scan call on, the chunk-output kernel
 * never requests its first C and B tiles, and every bounded
 * wait gives up after about 2^21 clock cycles instead of 2^32.  The call
 * then completes, the CTAs drain the copies and MMAs they issued, release
 * their tensor memory and return, and ssd_read_device_status() reports
 * SSD_ERR_DEVICE_TIMEOUT; the outputs are undefined.  kind 0 restores
 * normal operation.  Not for production use; affects every host thread. */
SSD_API ssd_status ssd_set_test_fault(int kind);

/* ABI version: (major << 16) | minor.  1.1 added the chunk-state, packed-row,
 * conv/norm and backward entry points to the 1.0 scan and step; 1.2 the test
 * hook ssd_set_test_fault and ssd_chunk_scan_bwd_varlen; 1.3
 * ssd_conv_scan_fwd, the workspace-free status read and the `path` argument
 * of ssd_chunk_scan_bwd_varlen (the tensor-core backward). */
SSD_API int ssd_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SSD_H_ */
