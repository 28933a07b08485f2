/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention forward library.
 *
 * The operation (KDA notes, "KDA 递归核心", §逐步公式 steps 1-4; KDA ledger DER1):
 * every (sequence b, value head hv) keeps a key-major state S in R^{K x V};
 * for each token t
 *     S_dec = exp(g_t) (.) S_{t-1}          decay, one factor per KEY channel (row of S)
 *     r_t   = v_t - k_t . S_dec             delta-rule residual
 *     S_t   = S_dec + (beta_t k_t) (x) r_t  rank-1 write
 *     o_t   = scale * q_t . S_t             read-out, scale = 1/sqrt(K) by default
 * Grouped value attention (KDA notes, "KDA 递归核心", input-tensor table:
 * q, k are repeat_interleave'd to HV heads): value head hv reads q/k head
 * hv / (HV/H).  The gate (KDA notes, "Gate 激活", table "两种 Gate"):
 *     input = g_raw + dt_bias[hv, :],  rate = exp(A_log[hv])
 *     SAFE      g = lower_bound * sigmoid(rate * input)     in [lower_bound, 0]
 *     STANDARD  g = -rate * softplus(input)                 in (-inf, 0]
 *
 * Conventions shared by every entry point
 *   - All tensors are dense, contiguous, row-major DEVICE buffers with the
 *     shapes given per argument; the caller owns and allocates all of them.
 *     The library never allocates, never frees and keeps no pointer after
 *     the call returns.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL means
 *     the legacy default stream).  No entry point synchronises the device,
 *     except kda_read_status, which exists to do so.
 *   - Arguments are validated on the host before anything is launched.  On an
 *     invalid argument nothing is launched and KDA_ERR_INVALID_ARG or
 *     KDA_ERR_UNSUPPORTED is returned; a launch failure returns KDA_ERR_CUDA.
 *     kda_last_error() then describes the failure (thread-local string).
 *   - No C++ exception crosses this interface.
 *   - Per-token tensors (q, k, v, g, beta, o) share one dtype (`dtype`);
 *     A_log, dt_bias and the state are always float32.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Binary-compatible with cudaStream_t. */
typedef struct CUstream_st* kda_stream_t;

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1, /* null pointer, bad shape or bad value; nothing launched     */
    KDA_ERR_UNSUPPORTED = 2, /* valid but outside the built kernels (K, V, chunk, dtype)  */
    KDA_ERR_CUDA = 3,        /* a CUDA call failed; kda_last_error() names it             */
    KDA_ERR_TIMEOUT = 4      /* a bounded on-device wait gave up (see kda_read_status)   */
} kda_status;

typedef enum { KDA_F32 = 0, KDA_BF16 = 1 } kda_dtype;

/* Mirrors the op's `use_gate_in_kernel` / `safe_gate` switches (KDA notes, "Gate 激活",
 * §Gate 在 API 中的位置): NONE means `g` already holds the log-space decay. */
typedef enum { KDA_GATE_NONE = 0, KDA_GATE_SAFE = 1, KDA_GATE_STANDARD = 2 } kda_gate_mode;

/* Input options of kda_chunk_fwd_ex and kda_recurrent_step_ex (bit flags).  By default the op takes
 * q, k as given and beta as the write strength itself (KDA notes, "KDA 递归核心": beta is an input
 * write strength; DeltaNet-family digest: keys are assumed L2-normalised).  These options move the
 * two input-side steps into the kernels' load stage, so that a caller holding raw projections does
 * not pay a separate pass over HBM for them:
 *   KDA_INPUT_L2NORM_QK   q and k are divided by their L2 norm over the K channels, per token and
 *                         q/k head, in float32: x / max(||x||, 1e-6).
 *   KDA_INPUT_BETA_LOGITS beta holds logits; the kernels use sigmoid(beta) = 1 / (1 + exp(-beta)). */
typedef enum { KDA_INPUT_RAW = 0, KDA_INPUT_L2NORM_QK = 1, KDA_INPUT_BETA_LOGITS = 2 } kda_input_flags;

/* Thread-local description of the last failure on the calling thread ("" if none). */
const char* kda_last_error(void);

/* Library version string. */
const char* kda_version(void);

/*
 * kda_gate -- the gate activation alone (KDA notes, "Gate 激活", code box
 * kda_gate_reference and table "两种 Gate").
 *   g_raw    [B, T, HV, K]  dtype           raw gate projection
 *   A_log    [HV]           float32         head-wise log rate
 *   dt_bias  [HV, K]        float32 or NULL (NULL: no bias)
 *   mode     KDA_GATE_SAFE or KDA_GATE_STANDARD (NONE is INVALID_ARG)
 *   lower_bound  SAFE only: finite and < 0, else INVALID_ARG
 *   g_out    [B, T, HV, K]  float32         log-space decay, written
 * B, T, HV, K >= 1 (B*T*HV*K < 2^31).
 */
kda_status kda_gate(const void* g_raw, kda_dtype dtype, const float* A_log, const float* dt_bias,
                    int B, int T, int HV, int K, kda_gate_mode mode, float lower_bound,
                    float* g_out, kda_stream_t stream);

/*
 * kda_chunk_fwd_workspace_size -- bytes of device workspace with which kda_chunk_fwd
 * runs its fastest schedule for these sizes.  Always >= 256: the first 256 bytes hold
 * the on-device status word read by kda_read_status.  For K = V = 128, chunk 64 and at
 * most 96 (sequence, value head) pairs (B * HV) it adds the per-chunk records of the
 * two-pass schedule (146 KiB per chunk of 64 tokens per pair), as long as there are fewer
 * than 2^30 chunks in all and T * HV * 256 < 2^40; where that schedule splits its state pass
 * along the sequence (long sequences, few pairs), 128 KiB per segment per pair more for the
 * segments' chunk maps.  Returns 0 for sizes kda_chunk_fwd rejects.
 */
size_t kda_chunk_fwd_workspace_size(int B, int T, int H, int HV, int K, int V, int chunk);

/*
 * kda_chunk_fwd -- chunked prefill (DeltaNet-family digest, sections "Chunkwise
 * KDA" and "Chunkwise Triton pipeline"): the same result as running the
 * recurrence above token by token, computed C tokens at a time with the
 * in-chunk cumulative log-decay, the triangular solve for the in-chunk delta
 * errors and one state update per chunk.
 * Schedules (bf16 inputs, K = V = 128, chunk 64): for at most 96 (sequence, value head)
 * pairs and a workspace of at least kda_chunk_fwd_workspace_size bytes, two passes --
 * every chunk's local work in parallel, then the state recurrence over chunks; otherwise
 * one pass with one CTA per pair.  Both compute the same quantities to the same
 * tolerance.  Other shapes and float32 inputs use one pass on the CUDA cores.
 *   q, k     [B, T, H, K]   dtype
 *   v        [B, T, HV, V]  dtype
 *   g        [B, T, HV, K]  dtype   g_raw when gate_mode != NONE, else the log decay (<= 0)
 *   beta     [B, T, HV]     dtype   write strength (the op applies no sigmoid)
 *   A_log    [HV] float32, dt_bias [HV, K] float32 or NULL -- used when gate_mode != NONE
 *            (A_log may be NULL only when gate_mode == NONE)
 *   S0       [B, HV, K, V]  float32 initial state, or NULL for zeros
 *   chunk    16 or 64 (the pages' default is 64)
 *   scale    read-out scale; <= 0 selects 1/sqrt(K)
 *   o        [B, T, HV, V]  dtype, written; must not alias any input
 *   S_T      [B, HV, K, V]  float32 final state, written; or NULL.  May alias S0
 *            (in-place state update).
 *   workspace, workspace_bytes  >= 256 bytes of caller-owned device memory,
 *            256-byte aligned (kda_chunk_fwd_workspace_size(...) bytes select the
 *            fastest schedule); contents need no initialisation and are scratch
 *            after the call.
 * Constraints: HV % H == 0; K, V in {16, 32, 64, 128}; T >= 1 (a last partial
 * chunk is handled); every pointer 16-byte aligned.
 * Calls that share one workspace must be ordered on one stream.
 */
kda_status kda_chunk_fwd(const void* q, const void* k, const void* v, const void* g,
                         const void* beta, const float* A_log, const float* dt_bias,
                         const float* S0, int B, int T, int H, int HV, int K, int V, int chunk,
                         kda_gate_mode gate_mode, float lower_bound, float scale, kda_dtype dtype,
                         void* o, float* S_T, void* workspace, size_t workspace_bytes,
                         kda_stream_t stream);

/*
 * kda_chunk_fwd_ex -- kda_chunk_fwd with input options: `input_flags` is a bitwise OR of
 * kda_input_flags values (0 gives exactly kda_chunk_fwd).  Every other argument, layout, schedule
 * and error is that of kda_chunk_fwd; unknown flag bits return KDA_ERR_INVALID_ARG.
 */
kda_status kda_chunk_fwd_ex(const void* q, const void* k, const void* v, const void* g, const void* beta,
                            const float* A_log, const float* dt_bias, const float* S0, int B, int T, int H,
                            int HV, int K, int V, int chunk, kda_gate_mode gate_mode, float lower_bound,
                            float scale, kda_dtype dtype, unsigned int input_flags, void* o, float* S_T,
                            void* workspace, size_t workspace_bytes, kda_stream_t stream);

/* Schedules of kda_chunk_fwd. */
typedef enum {
    KDA_SCHEDULE_CUDA_CORE = 0,     /* one kernel on the CUDA cores (float32 inputs, other shapes)     */
    KDA_SCHEDULE_TC_SINGLE_PASS = 1, /* one tensor-core kernel, one CTA per (sequence, value head)      */
    KDA_SCHEDULE_TC_TWO_PASS = 2,    /* two tensor-core kernels: all chunks' local work, then the state */
    KDA_SCHEDULE_TC_TWO_PASS_SCAN = 3 /* the two passes with the state pass split along the sequence:
                                        segments' chunk maps, the segment chain, then the outputs (four
                                        kernels); taken for long sequences with few (sequence, head) pairs */
} kda_schedule;

/*
 * kda_chunk_fwd_schedule -- the schedule kda_chunk_fwd runs for these sizes, input dtype and
 * workspace size (a kda_schedule value), or -1 for arguments it rejects.  No launch, no device
 * access.
 */
int kda_chunk_fwd_schedule(int B, int T, int H, int HV, int K, int V, int chunk, kda_dtype dtype,
                           size_t workspace_bytes);

/*
 * kda_read_status -- synchronises `stream`, then reads the status word a
 * kda_chunk_fwd call left in `workspace` and clears it.  Returns KDA_OK, or
 * KDA_ERR_TIMEOUT if a bounded on-device wait of that call gave up (its
 * outputs are then undefined), or KDA_ERR_CUDA.
 */
kda_status kda_read_status(const void* workspace, kda_stream_t stream);

/* Size, in bytes, of the built-in workspace behind kda_chunk_fwd_noalloc. */
#define KDA_NOALLOC_SCRATCH_BYTES 4096

/*
 * kda_chunk_fwd_noalloc -- kda_chunk_fwd for callers that cannot allocate device memory.
 * The pages have no counterpart to this call; it is an interface convenience of this library.
 * Who needs it: code that only ever holds pointers to buffers owned by someone else -- e.g. a
 * host application or plugin handed its tensors by an outer runtime that keeps a fixed
 * device-memory budget and exposes no allocator, or a latency-critical serving loop in which
 * allocating on the call path is not allowed -- and so has no workspace to pass.
 * Arguments, layouts, results and errors are those of kda_chunk_fwd without the workspace: the
 * library supplies it from a fixed array of KDA_NOALLOC_SCRATCH_BYTES bytes of device memory that
 * is part of the library (every GPU that loads the library holds it until the process exits).
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library routine is called.
 *   - Every call resolves the array's address in the current device's context
 *     (cudaGetSymbolAddress), so a context that was reset or replaced since an earlier call is
 *     handled.  The first call on a device may also load the library's device code there; make
 *     that first call before any stream capture.
 *   - The array is smaller than the two-pass schedule's per-chunk records, so these calls
 *     run the single-pass schedule (see kda_chunk_fwd), which needs only the 256-byte status
 *     block: every size kda_chunk_fwd accepts fits.  A size that needed more workspace than
 *     KDA_NOALLOC_SCRATCH_BYTES would return KDA_ERR_UNSUPPORTED with a message, nothing launched.
 *   - Every call uses the same array and leaves its contents behind; each call clears the part
 *     that must start at zero (the status word).  Calls whose work overlaps on the GPU (for
 *     example on two streams at once) race on the array: order them on one stream.
 */
kda_status kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const void* g,
                                 const void* beta, const float* A_log, const float* dt_bias,
                                 const float* S0, int B, int T, int H, int HV, int K, int V, int chunk,
                                 kda_gate_mode gate_mode, float lower_bound, float scale,
                                 kda_dtype dtype, void* o, float* S_T, kda_stream_t stream);

/*
 * kda_chunk_fwd_noalloc_read_status -- kda_read_status for the built-in workspace of
 * kda_chunk_fwd_noalloc on the current device: synchronises `stream`, then reads and clears the
 * status word the last kda_chunk_fwd_noalloc call left there.  Returns KDA_OK, KDA_ERR_TIMEOUT if a
 * bounded on-device wait of that call gave up (its outputs are then undefined), or KDA_ERR_CUDA.
 * Call it before the next kda_chunk_fwd_noalloc call on that device, which clears the word again.
 * The pages have no counterpart to this call.
 */
kda_status kda_chunk_fwd_noalloc_read_status(kda_stream_t stream);

/*
 * kda_recurrent_step -- one decode step for a batch of sequences, fused
 * (DeltaNet-family digest, "decode के लिए fused recurrent Triton kernel": the
 * recurrent schedule for decode and stateful serving).  S is read once and
 * written once, in place.
 *   q, k     [B, H, K]      dtype   (one token per sequence, i.e. [B, 1, H, K])
 *   v        [B, HV, V]     dtype
 *   g        [B, HV, K]     dtype   g_raw when gate_mode != NONE, else the log decay
 *   beta     [B, HV]        dtype
 *   A_log, dt_bias          as for kda_chunk_fwd
 *   S        [B, HV, K, V]  float32, read and overwritten with S_t
 *   o        [B, HV, V]     dtype, written; must not alias any input
 * Constraints: HV % H == 0; K, V in {16, 32, 64, 128}; every pointer 16-byte aligned.
 */
kda_status kda_recurrent_step(const void* q, const void* k, const void* v, const void* g,
                              const void* beta, const float* A_log, const float* dt_bias,
                              int B, int H, int HV, int K, int V, kda_gate_mode gate_mode,
                              float lower_bound, float scale, kda_dtype dtype, float* S, void* o,
                              kda_stream_t stream);

/*
 * kda_recurrent_step_ex -- kda_recurrent_step with input options (see kda_chunk_fwd_ex):
 * `input_flags` is a bitwise OR of kda_input_flags values; 0 gives exactly kda_recurrent_step.
 */
kda_status kda_recurrent_step_ex(const void* q, const void* k, const void* v, const void* g, const void* beta,
                                 const float* A_log, const float* dt_bias, int B, int H, int HV, int K, int V,
                                 kda_gate_mode gate_mode, float lower_bound, float scale, kda_dtype dtype,
                                 unsigned int input_flags, float* S, void* o, kda_stream_t stream);

/*
 * kda_backward_workspace_size -- bytes of device workspace kda_backward needs for these sizes (the
 * state saved every 8 tokens, B * HV * ceil(T / 8) * K * V * 4 bytes, the fp32 decays exp(gate)
 * of every token, B * T * HV * K * 4 bytes, and the fp32 residuals of every token, B * T * HV * V * 4
 * bytes), or 0 for sizes it rejects.
 */
size_t kda_backward_workspace_size(int B, int T, int H, int HV, int K, int V);

/*
 * kda_backward -- reverse mode of kda_chunk_fwd: the gradients of a scalar loss L given
 * dO = dL/do and dS_T = dL/dS_T, with respect to every input.  The pages define the forward pass
 * only; the adjoint is derived from its four steps (KDA notes, "KDA 递归核心", §逐步公式) taken in
 * reverse order, and from the gate formulas (KDA notes, "Gate 激活", table "两种 Gate").
 *   q, k, v, g, beta, A_log, dt_bias, S0, B..V, gate_mode, lower_bound, scale, dtype
 *            exactly as given to kda_chunk_fwd (the forward pass is recomputed)
 *   dO       [B, T, HV, V]  dtype   gradient with respect to o (required)
 *   dS_T     [B, HV, K, V]  float32 gradient with respect to the final state, or NULL for zeros
 *   dq, dk   [B, T, H, K]   float32, written (summed over the value heads that read each q/k head)
 *   dv       [B, T, HV, V]  float32, written
 *   dg       [B, T, HV, K]  float32, written: the gradient with respect to the `g` argument -- the
 *            log decay when gate_mode == KDA_GATE_NONE, else g_raw
 *   dbeta    [B, T, HV]     float32, written
 *   dS0      [B, HV, K, V]  float32 gradient with respect to S0, written; or NULL
 *   dA_log   [HV] float32, ddt_bias [HV, K] float32: written when a gate ran (each may be NULL);
 *            ignored for KDA_GATE_NONE
 *   workspace, workspace_bytes  >= kda_backward_workspace_size(...) bytes, 16-byte aligned, scratch
 * Constraints as kda_chunk_fwd's (no chunk argument: the gradients do not depend on it).  All work
 * runs on the CUDA cores in float32 on `stream`; outputs summed from several CTAs use atomic adds, so
 * their last bits may differ from run to run.  Outputs must not alias inputs or each other.
 */
kda_status kda_backward(const void* q, const void* k, const void* v, const void* g, const void* beta,
                        const float* A_log, const float* dt_bias, const float* S0, const void* dO,
                        const float* dS_T, int B, int T, int H, int HV, int K, int V, kda_gate_mode gate_mode,
                        float lower_bound, float scale, kda_dtype dtype, float* dq, float* dk, float* dv,
                        float* dg, float* dbeta, float* dS0, float* dA_log, float* ddt_bias, void* workspace,
                        size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_mla_decode_workspace_size -- bytes of device workspace kda_mla_decode needs (q_abs and the
 * per-split partial results), or 0 for sizes it rejects.
 */
size_t kda_mla_decode_workspace_size(int B, int T, int H, int d_q, int d_v, int r);

/*
 * kda_mla_decode -- absorbed MLA decode step: one query token per sequence attends, with softmax, to the
 * sequence's cached latent vectors, without decompressing keys or values (KDA ledger, derivation DER2,
 * claim C4: q_abs = q W_UK; score = q_abs c^T; o_lat = softmax(scale score) c; o = o_lat W_UV^T).  The
 * MLA layer of the K3 architecture uses no positional encoding ("NoPE"), so none is applied.
 *   q        [B, H, d_q]   bf16     the new token's queries
 *   W_UK     [H, d_q, r]   bf16     key up-projection, absorbed into q
 *   W_UV     [H, d_v, r]   bf16     value up-projection, applied to the attended latent
 *   c        [B, T, r]     bf16     latent cache (shared by every head)
 *   lengths  [B] int32 in [1, T], or NULL: positions of each sequence that take part (the rest of its
 *            rows of c are not read)
 *   scale    softmax scale on the scores; <= 0 selects 1 / sqrt(d_q)
 *   dtype    KDA_BF16 (the only one built)
 *   o        [B, H, d_v]   bf16, written
 *   workspace, workspace_bytes  >= kda_mla_decode_workspace_size(...) bytes, 16-byte aligned, scratch
 * Constraints: d_q, d_v in {64, 128}; r in {128, 256, 512}; H >= 1; T >= 1.  Scores and the weighted sum
 * run on the tensor cores with float32 accumulation (q_abs enters them as two bf16 terms); the softmax
 * and both projections in float32.
 */
kda_status kda_mla_decode(const void* q, const void* W_UK, const void* W_UV, const void* c, const int* lengths,
                          int B, int T, int H, int d_q, int d_v, int r, float scale, kda_dtype dtype, void* o,
                          void* workspace, size_t workspace_bytes, kda_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
