/* libjmix -- the Mamba-1 mixer core of Jamba v0.1 on B200 (sm_100a).
 *
 * The mixer core runs from the in_proj output (x, z) to the gated output y
 * (TransformerLens "Jamba" adapter page: the Jamba Mamba mixer is Mamba-1 with
 * in_proj / conv1d / x_proj / dt_proj / out_proj plus Jamba's own
 * dt_layernorm / b_layernorm / c_layernorm on the selective parameters):
 *
 *   u      = SiLU(causal depthwise conv1d(x) + conv_b)         width d_conv
 *   [dt|B|C] = u . xproj_w^T                                   x_proj, d_inner -> R + 2N
 *   dt_n, B_n, C_n = RMSNorm(dt) w_dt, RMSNorm(B) w_B, RMSNorm(C) w_C
 *   delta  = softplus(dt_n . dtproj_w^T + dt_bias)              dt_proj, R -> d_inner
 *   h_t    = exp(delta_t A) * h_{t-1} + delta_t B_t u_t,  A = -exp(A_log)
 *   y_t    = (C_t . h_t + D u_t) * SiLU(z_t)
 *
 * (discretisation exp(delta A), B-bar ~ delta B and the recurrence: aifetchly
 * "Jamba Guide", section "Inside the Mamba State-Space Layers"; A_log and
 * softplus(dt_proj(.)): the same guide, "Hands-On Implementation"; sizes
 * d_inner 8192, d_state 16, d_conv 4, dt_rank 256: llm-architectures-explained
 * "Jamba v0.1", "Every architecture field"; the cached conv and recurrent
 * states that decoding threads through: TransformerLens "Jamba" adapter page.)
 *
 * Conventions for every entry point
 * ---------------------------------
 * Layouts are row-major, last index contiguous:
 *   x, z, y          [batch, seqlen, d_inner]          io dtype
 *   conv_w           [d_inner, d_conv]                 io dtype; tap d_conv-1 multiplies the current token
 *   conv_b           [d_inner]                         io dtype
 *   xproj_w          [dt_rank + 2*d_state, d_inner]    io dtype; rows are dt, then B, then C
 *   dt_norm_w        [dt_rank]; b_norm_w, c_norm_w [d_state]   io dtype
 *   dtproj_w         [d_inner, dt_rank]                io dtype
 *   dt_bias, D       [d_inner]                         float32
 *   A_log            [d_inner, d_state]                float32
 *   conv states      [batch, d_inner, d_conv-1]        io dtype, oldest tap first
 *   SSM states       [batch, d_inner, d_state]         float32
 * All pointers given to the compute entry points are DEVICE pointers (the
 * _host variant below is the one exception), owned by the caller.  libjmix
 * never allocates, frees or synchronises, except jm_poll_error (which
 * synchronises the given stream).  Calls are asynchronous on `stream`.  A
 * call's kernels follow one another (and the kernel before the call) with
 * programmatic dependent launch: a kernel may be scheduled while the one before
 * it finishes, but none reads what earlier work on the stream writes before
 * that work has completed; to the caller, stream order holds.
 *
 * Errors: host-side validation runs before any launch and returns
 * JM_ERR_INVALID_ARG (NULL required pointer, negative size, pointer not
 * 16-byte aligned, d_inner or dt_rank not a multiple of 8, y overlapping x or
 * z, workspace too small -> JM_ERR_WORKSPACE) or JM_ERR_UNSUPPORTED
 * (d_state != 16, d_conv != 4, dt_rank > 256).  A failed launch returns
 * JM_ERR_CUDA.  Nothing is launched when validation fails.  There is no
 * fallback path.  jm_last_error() gives a message for the calling thread.
 */
#ifndef JMIX_H
#define JMIX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* jm_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  JM_OK = 0,
  JM_ERR_INVALID_ARG = 1,
  JM_ERR_UNSUPPORTED = 2,
  JM_ERR_CUDA = 3,
  JM_ERR_TIMEOUT = 4,  /* a bounded device-side wait ran out (reported by jm_poll_error) */
  JM_ERR_WORKSPACE = 5
} jm_status;

typedef enum { JM_F32 = 0, JM_BF16 = 1 } jm_dtype;

typedef struct {
  int64_t batch;    /* sequences, >= 0 */
  int64_t seqlen;   /* tokens per sequence, >= 0 (jm_mixer_step: must be 1) */
  int64_t d_inner;  /* channels, > 0, multiple of 8 */
  int64_t d_state;  /* N, must be 16 */
  int64_t d_conv;   /* conv width, must be 4 */
  int64_t dt_rank;  /* R, 8..256, multiple of 8 */
  float eps;        /* RMSNorm epsilon, inside the square root, >= 0 */
  jm_dtype io;      /* dtype of x, z, y, conv states and the io-dtype weights */
  int32_t discretization; /* JM_DISC_EULER (0): Bbar = delta B;
                             JM_DISC_ZOH (1): Bbar = (exp(delta A) - 1) / A B */
  int32_t reserved;       /* must be 0 */
} jm_dims;

/* How B is discretised.  Abar = exp(delta A) in both; Euler takes delta B (the
 * Jamba guide's "Bbar ~ delta B"), zero-order hold the exact one-step solution
 * of dh/dt = A h + B u for u held over the step. */
enum { JM_DISC_EULER = 0, JM_DISC_ZOH = 1 };

/* Bytes of device workspace jm_mixer_fwd needs for these dims (0 if the dims
 * are invalid; see jm_last_error).  The workspace must be 256-byte aligned.
 * Its first 256 bytes hold device-side error flags that jm_poll_error reads. */
size_t jm_mixer_fwd_workspace_size(const jm_dims* dims);

/* Same for jm_mixer_step (dims->seqlen must be 1). */
size_t jm_mixer_step_workspace_size(const jm_dims* dims);

/* Mixer forward over whole sequences: the formulas above for t = 0..seqlen-1.
 *   x, z            in:  [B, L, d]
 *   y               out: [B, L, d]; must not overlap x or z
 *   final_state     out: [B, d, N] float32, h after the last token (required)
 *   init_conv_state in:  [B, d, d_conv-1] conv history before token 0, or NULL = zeros
 *   init_ssm_state  in:  [B, d, N] h before token 0, or NULL = zeros
 *   final_conv_state out: [B, d, d_conv-1] the last d_conv-1 conv inputs, or NULL = skip;
 *                   may equal init_conv_state (updated in place)
 *   workspace       scratch of at least jm_mixer_fwd_workspace_size(dims) bytes
 * With seqlen == 0 the final states are the initial ones (or zeros). */
jm_status jm_mixer_fwd(const jm_dims* dims, const void* x, const void* z, const void* conv_w,
                       const void* conv_b, const void* xproj_w, const void* dt_norm_w,
                       const void* b_norm_w, const void* c_norm_w, const void* dtproj_w,
                       const float* dt_bias, const float* A_log, const float* D, void* y,
                       float* final_state, const void* init_conv_state,
                       const float* init_ssm_state, void* final_conv_state, void* workspace,
                       size_t ws_bytes, jm_stream_t stream);

/* One decode step for every sequence (dims->seqlen must be 1): the forward
 * with the cached states as history, then, in place,
 *   conv_state[b, c, :] <- [conv_state[b, c, 1:], x_t[b, c]]  and  ssm_state <- h.
 *   x_t, z_t   in:  [B, d];   y_t out: [B, d] (must not overlap x_t, z_t)
 *   conv_state in/out [B, d, d_conv-1];  ssm_state in/out [B, d, N] float32 */
jm_status jm_mixer_step(const jm_dims* dims, const void* x_t, const void* z_t, void* conv_state,
                        float* ssm_state, const void* conv_w, const void* conv_b,
                        const void* xproj_w, const void* dt_norm_w, const void* b_norm_w,
                        const void* c_norm_w, const void* dtproj_w, const float* dt_bias,
                        const float* A_log, const float* D, void* y_t, void* workspace,
                        size_t ws_bytes, jm_stream_t stream);

/* Bytes of the fp16 weight copies jm_prepare_weights writes (0 for invalid
 * dims or float32 io). */
size_t jm_prepared_weights_size(const jm_dims* dims);

/* Converts xproj_w [R + 2N, d] and dtproj_w [d, R] (bf16, device) once into the
 * fp16 operands the tensor-core path feeds its two contractions (exact for
 * |w| >= 2^-14; fp16 subnormals below), into `prepared` (device, 256-byte
 * aligned, at least jm_prepared_weights_size bytes, owned by the caller).  A
 * decode loop passes it to jm_mixer_step_indexed so that no step re-converts
 * the weights; it stays valid until the weights change.  bf16 io only
 * (JM_ERR_UNSUPPORTED otherwise).  Asynchronous on `stream`. */
jm_status jm_prepare_weights(const jm_dims* dims, const void* xproj_w, const void* dtproj_w,
                             void* prepared, size_t bytes, jm_stream_t stream);

/* One decode step for a batch of rows whose states live in slots of a state
 * pool, as a continuously batching server keeps them: the set of active
 * sequences changes from step to step, their cached states stay in place.
 * (TransformerLens "Jamba" adapter page: generation threads the cache of conv
 * and recurrent states through the mixer.)
 *   dims->batch  B rows this step; dims->seqlen must be 1; bf16 io only
 *   state_idx    DEVICE int32 [B]: row b of x_t, z_t, y_t uses slot state_idx[b];
 *                the B slots must be distinct (duplicates leave those slots and
 *                rows unspecified; no access leaves the buffers)
 *   n_slots      slots S in the pools, B <= S < 2^31
 *   conv_pool    in/out [S, d, d_conv-1] bf16;  ssm_pool in/out [S, d, N] float32
 *   prepared     fp16 weights from jm_prepare_weights, or NULL (then the step
 *                converts xproj_w and dtproj_w itself, as jm_mixer_step does)
 * Slot state_idx[b] is updated in place exactly as jm_mixer_step updates row b;
 * no other slot is read or written.  A slot outside [0, S) is checked on the
 * device: that row's y_t is left unwritten, its slot untouched, and
 * jm_poll_error returns JM_ERR_INVALID_ARG.  Workspace: at least
 * jm_mixer_step_workspace_size(dims) bytes.  Other arguments, errors and
 * ownership as jm_mixer_step. */
jm_status jm_mixer_step_indexed(const jm_dims* dims, const int32_t* state_idx, int64_t n_slots,
                                const void* x_t, const void* z_t, void* conv_pool,
                                float* ssm_pool, const void* conv_w, const void* conv_b,
                                const void* xproj_w, const void* dt_norm_w,
                                const void* b_norm_w, const void* c_norm_w,
                                const void* dtproj_w, const float* dt_bias, const float* A_log,
                                const float* D, const void* prepared, void* y_t,
                                void* workspace, size_t ws_bytes, jm_stream_t stream);

/* jm_mixer_step without a caller workspace, for callers that cannot allocate
 * device memory: serving engines that hand all device memory to their own
 * caches and give plug-ins no allocator, or host code that must stay off the
 * allocator.  The paper has no counterpart to this entry point.
 *
 * Arguments and results are those of jm_mixer_step without workspace and
 * ws_bytes.  The scratch is a static 32 MiB device array inside libjmix, held
 * by every GPU that loads the library until the process exits; a step at
 * Jamba v0.1 mixer shapes (d_inner 8192, dt_rank 256) needs about 14 MiB for
 * 256 sequences.  A step that needs more returns JM_ERR_UNSUPPORTED with a
 * message and launches nothing.  The function itself allocates nothing.
 *
 * The first call on a device looks up the array's device address (once per
 * device, with that device current).  All calls share the one array, and each call clears what it needs
 * cleared, so the previous call's contents never leak into a result; but two
 * calls whose kernels overlap on the GPU (different streams, or different
 * host threads on one device) race on the array and must be serialised by the
 * caller.  Launch errors are returned as JM_ERR_CUDA; device-side flags (a
 * bounded wait that ran out) are read with jm_noalloc_poll_error, since
 * jm_poll_error needs a caller workspace. */
jm_status jm_mixer_step_noalloc(const jm_dims* dims, const void* x_t, const void* z_t,
                                void* conv_state, float* ssm_state, const void* conv_w,
                                const void* conv_b, const void* xproj_w, const void* dt_norm_w,
                                const void* b_norm_w, const void* c_norm_w,
                                const void* dtproj_w, const float* dt_bias, const float* A_log,
                                const float* D, void* y_t, jm_stream_t stream);

/* jm_poll_error for jm_mixer_step_noalloc: synchronises `stream`, then reads
 * the error flags that the steps write into the header of the static array on
 * the current device.  JM_ERR_TIMEOUT if a bounded device-side wait ran out
 * since the last jm_mixer_step_noalloc on this device (each step clears the
 * flags), JM_ERR_CUDA if the stream reports an error, JM_OK otherwise.
 * Allocates nothing. */
jm_status jm_noalloc_poll_error(jm_stream_t stream);

/* The failure-detection self-test (see jm_selftest_timeout) aimed at the static
 * array's error header: a following jm_noalloc_poll_error returns
 * JM_ERR_TIMEOUT.  The same sharing rules as jm_mixer_step_noalloc apply. */
jm_status jm_noalloc_selftest_timeout(jm_stream_t stream);

/* End-to-end forward from HOST buffers: copies x_host and z_host (pinned host
 * memory, [B, L, d] io dtype) into the caller's device buffers x_dev / z_dev,
 * runs the forward, and copies y and the final SSM state back into y_host and
 * final_state_host.  The batch runs in up to 8 groups of whole sequences so
 * that copies in both directions overlap the compute: each group's inputs go
 * up on an internal stream, its forward runs on `stream`, its outputs come down
 * on a second internal stream (both created once per host thread; no device
 * memory is allocated).  The call returns without waiting, and `stream` covers
 * every copy: synchronise it before reading y_host.  A group uses the same
 * arithmetic as jm_mixer_fwd on its sequences (the x_proj split and the scan
 * schedule follow the group's size, so bits may differ from one jm_mixer_fwd
 * call over the whole batch, within the same tolerances).  If a group would
 * need more than ws_bytes, the batch runs as one group.  Weights are device
 * pointers as in jm_mixer_fwd; the states start from zero. */
jm_status jm_mixer_fwd_host(const jm_dims* dims, const void* x_host, const void* z_host,
                            void* y_host, float* final_state_host, void* x_dev, void* z_dev,
                            void* y_dev, float* final_state_dev, const void* conv_w,
                            const void* conv_b, const void* xproj_w, const void* dt_norm_w,
                            const void* b_norm_w, const void* c_norm_w, const void* dtproj_w,
                            const float* dt_bias, const float* A_log, const float* D,
                            void* workspace, size_t ws_bytes, jm_stream_t stream);

/* Synchronises `stream`, then reads the error flags in `workspace`'s first
 * 256 bytes: JM_ERR_TIMEOUT if a bounded device-side wait ran out since the
 * last call that cleared them (every jm_mixer_fwd / jm_mixer_step clears
 * them), JM_ERR_INVALID_ARG if a device-side input check failed (the
 * cu_seqlens of jm_mixer_fwd_varlen, the state_idx of jm_mixer_step_indexed),
 * JM_ERR_CUDA if the stream reports an error, JM_OK otherwise. */
jm_status jm_poll_error(void* workspace, jm_stream_t stream);

/* The full Mamba layer around the mixer core (bf16 io only):
 *   [x | z] = hidden . in_proj_w^T,  y = mixer core (as jm_mixer_fwd),
 *   out = y . out_proj_w^T.
 * hidden: [B, L, d_model]; in_proj_w: [2 d_inner, d_model] (rows 0 .. d_inner-1
 * give x, the rest z); out_proj_w: [d_model, d_inner]; out: [B, L, d_model]; all
 * bf16 device memory, 16-byte aligned; d_model a positive multiple of 8.  The
 * mixer arguments, states, errors and ownership are those of jm_mixer_fwd.  The
 * projections run on libjmix's tcgen05 GEMM (fp32 accumulation, bf16 x, z, y
 * and out; in_proj writes x and z straight into the mixer's layout) with the
 * caller's workspace as scratch: jm_layer_fwd_workspace_size(dims, d_model)
 * bytes, 256-byte aligned; its first 256 bytes are the error header that
 * jm_poll_error reads (the projections' flags and the mixer's).  JM_ERR_UNSUPPORTED
 * for float32 io. */
size_t jm_layer_fwd_workspace_size(const jm_dims* dims, int64_t d_model);
jm_status jm_layer_fwd(const jm_dims* dims, int64_t d_model, const void* hidden,
                       const void* in_proj_w, const void* conv_w, const void* conv_b,
                       const void* xproj_w, const void* dt_norm_w, const void* b_norm_w,
                       const void* c_norm_w, const void* dtproj_w, const float* dt_bias,
                       const float* A_log, const float* D, const void* out_proj_w, void* out,
                       float* final_state, const void* init_conv_state,
                       const float* init_ssm_state, void* final_conv_state, void* workspace,
                       size_t ws_bytes, jm_stream_t stream);

/* Backward of the selective-scan core (training), float32 throughout, Euler B.
 * Forward: h_t = exp(delta_t A) h_{t-1} + delta_t B_t u_t, A = -exp(A_log),
 * y_t = C_t . h_t + D u_t (per sequence and channel; the Jamba guide, "Inside
 * the Mamba State-Space Layers").  Given gy = dLoss/dy it writes every input
 * gradient: g_delta, g_u [B, L, d]; g_B, g_C [B, L, 16] (summed over channels);
 * g_A_log [d, 16], g_D [d] (summed over sequences and tokens); g_h0 [B, d, 16]
 * (may be NULL).  Inputs: delta, u, gy [B, L, d]; B, C [B, L, 16]; A_log [d, 16];
 * D [d]; h0 [B, d, 16] or NULL (zero).  dims: batch, seqlen, d_inner, d_state
 * (must be 16) and discretization (JM_DISC_EULER only) are read.  Results are
 * deterministic (fixed summation order).  Workspace:
 * jm_scan_bwd_workspace_size(dims) bytes, 256-byte aligned (state checkpoints
 * every 4 tokens and per-warp partial sums; its first 256 bytes are the error
 * header jm_poll_error reads).  Asynchronous on `stream`. */
size_t jm_scan_bwd_workspace_size(const jm_dims* dims);
jm_status jm_scan_bwd(const jm_dims* dims, const float* delta, const float* u, const float* B,
                      const float* C, const float* A_log, const float* D, const float* h0,
                      const float* gy, float* g_delta, float* g_u, float* g_B, float* g_C,
                      float* g_A_log, float* g_D, float* g_h0, void* workspace, size_t ws_bytes,
                      jm_stream_t stream);

/* How jm_scan_bwd will cut each sequence into time parts for these dims:
 * *n_parts parts (1..16) of whole 4-token chunks, at least 2 chunks each, that
 * run side by side; each part folds the others' results in through exp(A S), S
 * the part's sum of delta (both the state recurrence and its adjoint are linear
 * with the same decays).  One part when the (128-channel tile, sequence) CTAs
 * already fill at least 90% of their waves on a B200.  Depends only on the
 * dims, like the workspace size.  Returns JM_ERR_INVALID_ARG for invalid dims or
 * a NULL output, JM_ERR_UNSUPPORTED as jm_scan_bwd does. */
jm_status jm_scan_bwd_schedule(const jm_dims* dims, int* n_parts);

/* Failure-detection self-test: launches one thread that waits, through the
 * same bounded wait the pipelines use, on a barrier that nothing completes.
 * The wait gives up after its limit (2 s), records site 99 in workspace's
 * error header and returns, so a following jm_poll_error(workspace) returns
 * JM_ERR_TIMEOUT and the CUDA context stays usable.  workspace: device, at
 * least 256 bytes (its first 256 bytes are overwritten).  Asynchronous on
 * `stream`.  JM_ERR_WORKSPACE if workspace is NULL or too small. */
jm_status jm_selftest_timeout(void* workspace, size_t ws_bytes, jm_stream_t stream);

/* Message of the last failed call on this thread ("" if none). */
const char* jm_last_error(void);

/* Number of kernel launches the last successful jm_mixer_fwd / jm_mixer_step /
 * jm_mixer_fwd_host on this thread issued (for launch accounting). */
int jm_last_launch_count(void);

/* Name of the index-th kernel the last successful compute call on this thread
 * launched ("" when out of range).  The string is static. */
const char* jm_last_kernel_name(int index);

/* Forward over a packed batch of variable-length sequences (serving prefill).
 * dims->batch = number of sequences B, dims->seqlen = total tokens T.
 * x, z, y: [T, d_inner], the sequences one after another.  cu_seqlens: DEVICE
 * int32 [B + 1] token offsets, cu_seqlens[0] = 0, nondecreasing,
 * cu_seqlens[B] = T; sequence b is tokens cu_seqlens[b] .. cu_seqlens[b+1]-1
 * (a sequence may be empty).  final_state, init_ssm_state: [B, d_inner, 16];
 * init_conv_state, final_conv_state: [B, d_inner, 3], per sequence exactly as
 * in jm_mixer_fwd (each sequence starts from its own initial states).  bf16 io
 * only: JM_ERR_UNSUPPORTED for JM_F32.  The offsets live on the device, so
 * they are checked there: a cu_seqlens that breaks the rules above leaves
 * y and the states unspecified (no access leaves the buffers) and makes
 * jm_poll_error return JM_ERR_INVALID_ARG.  Workspace:
 * jm_mixer_fwd_varlen_workspace_size(dims).  Other arguments, errors and
 * ownership as jm_mixer_fwd. */
size_t jm_mixer_fwd_varlen_workspace_size(const jm_dims* dims);
jm_status jm_mixer_fwd_varlen(const jm_dims* dims, const int32_t* cu_seqlens, const void* x,
                              const void* z, const void* conv_w, const void* conv_b,
                              const void* xproj_w, const void* dt_norm_w, const void* b_norm_w,
                              const void* c_norm_w, const void* dtproj_w, const float* dt_bias,
                              const float* A_log, const float* D, void* y, float* final_state,
                              const void* init_conv_state, const float* init_ssm_state,
                              void* final_conv_state, void* workspace, size_t ws_bytes,
                              jm_stream_t stream);

/* How jm_mixer_fwd will schedule the scan of this problem (bf16 I/O; float32
 * problems run one part per sequence).  Each sequence is cut into *n_parts time
 * parts of whole 32-token chunks.  *two_pass = 0: the parts of a sequence run
 * one after another, each starting from the state the previous one handed over
 * (used when the (sequence, 128-channel tile) pairs fill the GPU).  *two_pass = 1:
 * a state pass records each part's end state from a zero start and its sum of
 * delta, then every part computes its outputs from the fold of the earlier
 * parts' results (used for few sequences).  Depends only on the dims.  Returns
 * JM_ERR_INVALID_ARG for invalid dims or NULL outputs. */
jm_status jm_mixer_fwd_schedule(const jm_dims* dims, int* n_parts, int* two_pass);

/* Per-kernel timing hook for benchmarks.  `events` is an array of n_events
 * cudaEvent_t handles created by the caller.  While set (for calls on this
 * thread), each compute call records events[0] on its stream before its
 * first kernel and events[i] right after its i-th kernel, for i < n_events;
 * the caller reads the kernel durations with cudaEventElapsedTime.  Pass
 * (NULL, 0) to stop.  Returns JM_ERR_INVALID_ARG for a NULL array with
 * n_events > 0. */
jm_status jm_set_kernel_events(void* const* events, int n_events);

#ifdef __cplusplus
}
#endif

#endif /* JMIX_H */
