/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention operator library
 * (libkda.so).
 *
 * The operator is the per-head recurrence of Kimi Delta Attention (page
 * "Kimi Linear" on docsaid.org, section "KDA : une decroissance propre a
 * chaque canal", the KDA update equation; course page "Attention lineaire et
 * recurrence", section "Kimi Delta Attention = les trois remedes combines"):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t
 *
 * with a per-key-channel forget gate alpha_t = exp(log_alpha_t) in (0, 1]^{d_k}
 * and a scalar write strength beta_t in [0, 1] per token and head.  The state
 * S is d_k x d_v per (sequence, head) and is kept in fp32.  The read-out uses
 * the updated state S_t; no 1/sqrt(d_k) scale is applied (fold it into q).
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *     allocates no device memory and keeps no state between calls except
 *     launch settings cached per device under a lock (each kernel's shared-
 *     memory limit, the SM count), so several host threads and several GPUs
 *     may share one process.
 *   - Tensors are dense, row-major, token-major:
 *       q, k, log_alpha : [T_total, H, d_k]
 *       v, o            : [T_total, H, d_v]
 *       beta            : [T_total, H]
 *       states          : [N, H, d_k, d_v] fp32, d_v fastest
 *     For decode, T_total is the batch size (one token per sequence).
 *   - Alignment: fp32 state pointers, and q, k, v, log_alpha and o of
 *     kda_prefill, must be 16-byte aligned; beta, cu_seqlens and every input
 *     of kda_decode_step other than the state need only their element's
 *     natural alignment.  The workspace is 256-byte aligned.
 *   - Calls are asynchronous on `stream` (0 = legacy default stream) and never
 *     synchronise, except kda_check_workspace_error.
 *   - Arguments are validated on the host; a failed check returns a status
 *     and launches nothing.  Launch failures return KDA_ERR_CUDA.  No C++
 *     exception crosses this boundary and no kernel traps or asserts.
 *   - Data preconditions that are documented but not checked: log_alpha <= 0
 *     (alpha in (0, 1]; -inf is allowed and means alpha = 0), beta in [0, 1],
 *     finite values, and, for the fast path's accuracy bound, L2-normalised
 *     q and k (the pages normalise q and k before the operator).
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The stream type of the CUDA runtime, declared opaquely so that this header
 * does not need cuda_runtime.h. */
typedef struct CUstream_st *kda_stream_t;

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned pointer   */
    KDA_ERR_UNSUPPORTED = 2,  /* shape or dtype without a kernel               */
    KDA_ERR_WORKSPACE = 3,    /* workspace missing or too small                */
    KDA_ERR_CUDA = 4          /* a CUDA runtime call or launch failed          */
} kda_status;

/* Element type of q, k, v, log_alpha, beta and o.  States are always fp32. */
typedef enum {
    KDA_BF16 = 0,
    KDA_FP32 = 1
} kda_dtype;

/* Human-readable name of a status code (static string, never NULL). */
const char *kda_status_string(kda_status s);

/* Library version as major*10000 + minor*100 + patch. */
int kda_version(void);

/*
 * Workspace bytes for kda_prefill's fastest path on this problem (a multiple
 * of 256).  For d_k = d_v = 128 this includes one 73 KB record per (chunk of
 * 64 tokens, head) for the two-kernel tensor-core path, i.e. about
 * 1.2 KB per (token, head): 4.9 GB for 131072 tokens x 32 heads.  Pure host
 * arithmetic, no CUDA call.  Returns 0 for arguments kda_prefill would reject.
 */
size_t kda_prefill_workspace_size(int32_t num_seqs, int64_t total_tokens,
                                  int32_t H, int32_t d_k, int32_t d_v);

/*
 * Chunkwise prefill over a packed batch of sequences.
 *
 * Computes o_t for every token and, per sequence, the state after its last
 * token.  The sequence is cut into chunks of 64 tokens; within a chunk the
 * work is matrix products and between chunks the state is carried (news
 * digest page on Kimi Linear, section "Algorithme parallele par chunks";
 * course page "Attention lineaire et recurrence", section "Le calcul par
 * blocs").  The chunked form is exact; only the rounding order differs from
 * the token-by-token recurrence.
 *
 *   q, k, log_alpha : [T_total, H, d_k]  dtype
 *   v               : [T_total, H, d_v]  dtype
 *   beta            : [T_total, H]       dtype
 *   init_state      : [N, H, d_k, d_v] fp32, or NULL for zero initial states
 *   cu_seqlens      : device int32 [N + 1], cu_seqlens[0] = 0, non-decreasing,
 *                     cu_seqlens[N] = T_total; or NULL for N sequences of
 *                     equal length T_total / N (T_total % N must be 0).
 *                     Zero-length sequences are allowed: their final state
 *                     is their initial state.
 *   num_seqs (N) >= 1, total_tokens >= 0, H >= 1.
 *   o               : [T_total, H, d_v]  dtype, written
 *   final_state     : [N, H, d_k, d_v] fp32, written, or NULL.  May alias
 *                     init_state exactly (same pointer).
 *   workspace       : device buffer, 256-byte aligned, contents on entry do
 *                     not matter.  At least 256 + 4 N bytes (rounded up to
 *                     256) are required; with kda_prefill_workspace_size(...)
 *                     bytes the bf16 d = 128 case runs the two-kernel path
 *                     (chunk preparation for all chunks in parallel, then the
 *                     state chain), with less it runs the single-kernel path
 *                     (same results, slower).
 *
 * Supported: dtype KDA_BF16 or KDA_FP32 with d_k, d_v in {16, 32, 64, 128}.
 * KDA_BF16 with d_k = d_v = 128 runs the tensor-core (tcgen05) path; every
 * other case runs the fp32 CUDA-core path (KDA_FP32 is the accurate test
 * mode).  o must not overlap any input.
 */
kda_status kda_prefill(const void *q, const void *k, const void *v,
                       const void *log_alpha, const void *beta,
                       const float *init_state, const int32_t *cu_seqlens,
                       int32_t num_seqs, int64_t total_tokens, int32_t H,
                       int32_t d_k, int32_t d_v, kda_dtype dtype, void *o,
                       float *final_state, void *workspace,
                       size_t workspace_bytes, kda_stream_t stream);

/*
 * One decode step for `batch` independent sequences, state updated in place.
 *
 * Per (b, h): S <- Diag(exp(log_alpha)) S;  u = beta (v - S^T k);
 * S <- S + k u^T;  o = S^T q  -- the KDA update for a single token, which is
 * the step form the chunked prefill hands over to (the state is the whole
 * memory of the sequence).
 *
 *   q, k, log_alpha : [batch, H, d_k] dtype;  v, o : [batch, H, d_v] dtype;
 *   beta : [batch, H] dtype;  state : [batch, H, d_k, d_v] fp32, read and
 *   written in place.
 * Supported: dtype KDA_BF16 or KDA_FP32, d_k in {16, 32, 64, 128},
 * d_v in {16, 32, 64, 128}.  o must not overlap the state or the inputs.
 * batch = 0 is a valid no-op.
 */
kda_status kda_decode_step(const void *q, const void *k, const void *v,
                           const void *log_alpha, const void *beta,
                           float *state, int32_t batch, int32_t H,
                           int32_t d_k, int32_t d_v, kda_dtype dtype, void *o,
                           kda_stream_t stream);

/*
 * The same two calls for Gated DeltaNet, whose forget gate is one scalar per
 * token and head (page "Kimi Linear" on docsaid.org, section "KDA : une
 * decroissance propre a chaque canal", the Gated DeltaNet update that opens
 * it; news digest page on Kimi Linear, section "De l'attention lineaire a
 * Gated DeltaNet"):
 *
 *     S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,
 *     o_t = S_t^T q_t,   alpha_t = exp(log_alpha_t) a scalar in (0, 1].
 *
 * A scalar gate commutes with (I - beta k k^T), so this is the KDA update
 * with the gate repeated over the d_k key channels; the kernels take it that
 * way (each 64-token chunk's gate values are spread over the channels in
 * shared memory) and run the same paths as kda_prefill / kda_decode_step.
 *
 * Arguments, layouts, workspace (kda_prefill_workspace_size), alignment and
 * errors are those of kda_prefill / kda_decode_step except:
 *   log_alpha : [T_total, H] (prefill) or [batch, H] (decode), dtype, with
 *               only its element's natural alignment.
 */
kda_status gdn_prefill(const void *q, const void *k, const void *v,
                       const void *log_alpha, const void *beta,
                       const float *init_state, const int32_t *cu_seqlens,
                       int32_t num_seqs, int64_t total_tokens, int32_t H,
                       int32_t d_k, int32_t d_v, kda_dtype dtype, void *o,
                       float *final_state, void *workspace,
                       size_t workspace_bytes, kda_stream_t stream);

kda_status gdn_decode_step(const void *q, const void *k, const void *v,
                           const void *log_alpha, const void *beta,
                           float *state, int32_t batch, int32_t H,
                           int32_t d_k, int32_t d_v, kda_dtype dtype, void *o,
                           kda_stream_t stream);

/*
 * The operator with the layer's prologue and epilogue fused in (page "Kimi
 * Linear" on docsaid.org, section "Les autres pieces": q, k L2-normalised,
 * beta a sigmoid, the decay a GDN / Mamba-like function of a pre-activation,
 * the output RMS-normalised per head and multiplied by a data-dependent
 * sigmoid gate; the course page "Attention lineaire et recurrence" gives
 * Kimi Linear's decay as -e^A Softplus(z)):
 *
 *   q_t <- q_t / sqrt(|q_t|^2 + qk_eps),   k_t <- k_t / sqrt(|k_t|^2 + qk_eps)
 *   log_alpha_t = -exp(A_log[h]) * softplus(gate_z_t)      (per key channel)
 *   beta_t = sigmoid(beta_logit_t)
 *   (the KDA recurrence of kda_prefill / kda_decode_step)
 *   o_t <- o_t / sqrt(mean_j o_tj^2 + norm_eps) * norm_weight_j * sigmoid(out_gate_tj)
 *
 *   q, k, gate_z : [T, H, d_k] raw;  v : [T, H, d_v];  beta_logit : [T, H]
 *   A_log        : [H] fp32 (device), required
 *   out_gate     : [T, H, d_v] pre-sigmoid, or NULL (no output gate); 16-byte
 *                  aligned for kda_layer_prefill
 *   norm_weight  : [d_v] fp32 (device), or NULL (weight 1)
 * Other arguments, layouts and errors as kda_prefill / kda_decode_step.
 * kda_layer_prefill runs on the two-kernel tensor-core path only: bf16,
 * d_k = d_v = 128 and a workspace of at least kda_prefill_workspace_size(...)
 * bytes (else KDA_ERR_UNSUPPORTED / KDA_ERR_WORKSPACE).  With a workspace of
 * kda_layer_prefill_workspace_size(...) bytes its prologue runs as a pass of
 * its own that writes log_alpha and beta (bf16) and the inverse L2 norms of
 * the q and k rows (fp32) into the workspace, then the operator's kernels,
 * whose preparation scales the raw q and k by those norms; with less,
 * the prologue runs inside the chunk preparation (log_alpha kept in fp32
 * there; slower: the arithmetic lands on that kernel's latency-bound path).
 * Either way the epilogue is one pass over o after the state chain.
 * kda_layer_decode_step takes every shape kda_decode_step takes.  Weights of
 * the projections that produce these activations are the caller's.
 */
size_t kda_layer_prefill_workspace_size(int32_t num_seqs, int64_t total_tokens, int32_t H,
                                        int32_t d_k, int32_t d_v);

kda_status kda_layer_prefill(const void *q, const void *k, const void *v, const void *gate_z,
                             const float *A_log, const void *beta_logit, const void *out_gate,
                             const float *norm_weight, float qk_eps, float norm_eps,
                             const float *init_state, const int32_t *cu_seqlens,
                             int32_t num_seqs, int64_t total_tokens, int32_t H, int32_t d_k,
                             int32_t d_v, kda_dtype dtype, void *o, float *final_state,
                             void *workspace, size_t workspace_bytes, kda_stream_t stream);

kda_status kda_layer_decode_step(const void *q, const void *k, const void *v,
                                 const void *gate_z, const float *A_log, const void *beta_logit,
                                 const void *out_gate, const float *norm_weight, float qk_eps,
                                 float norm_eps, float *state, int32_t batch, int32_t H,
                                 int32_t d_k, int32_t d_v, kda_dtype dtype, void *o,
                                 kda_stream_t stream);

/*
 * Context parallelism across devices (course page "Attention lineaire et
 * recurrence", section "Verification de comprehension": a segment of a
 * sequence acts on the state it receives through its cumulative transition
 * M = prod_t (I - beta_t k_t k_t^T) Diag(alpha_t), then adds the state it
 * generates from zero, S~).  A device holding segment r starts from
 *     S_in(0) = S_0,   S_in(i + 1) = M_i S_in(i) + S~_i,   i < r.
 * This call forms S_in(n_prev) from the gathered pairs of the n_prev segments
 * before it:
 *   M       : [n_prev, H, d_k, d_k] fp32;   S_tilde : [n_prev, H, d_k, d_v] fp32
 *   S0      : [H, d_k, d_v] fp32 or NULL (zero);   S_in : [H, d_k, d_v] fp32, written
 * n_prev = 0 copies S0 (or writes zeros).  A segment's (M, S~) come from
 * kda_cp_local below (the Python module context_parallel.py runs the passes
 * and the exchange).  Supported: d_k in
 * {16, 32, 64, 128}, d_v in {32, 64, 128}; 4-byte aligned pointers; S_in must
 * not overlap M or S_tilde.
 */
kda_status kda_cp_combine(const float *M, const float *S_tilde, const float *S0, float *S_in,
                          int32_t n_prev, int32_t H, int32_t d_k, int32_t d_v,
                          kda_stream_t stream);

/*
 * The two passes of one segment (a single sequence of total_tokens tokens,
 * bf16, d_k = d_v = 128, a workspace of kda_prefill_workspace_size(1,
 * total_tokens, H) bytes), sharing one chunk preparation:
 *   kda_cp_local  prepares every chunk (the records stay in `workspace`) and
 *                 runs the state chain twice over them, side by side:
 *                 S_tilde [1, H, d_k, d_v] from a zero state, M [1, H, d_k, d_k]
 *                 from the identity with v counting as zero; o_scratch is not
 *                 written (it stays in the interface; may be NULL).
 *   kda_cp_finish runs the chain once more over the same workspace's records
 *                 from S_in [1, H, d_k, d_v] (NULL: zero), writing o and
 *                 final_state (NULL: not written).  The workspace must not have
 *                 been used for anything else in between, and v must be the
 *                 same tensor.
 */
kda_status kda_cp_local(const void *q, const void *k, const void *v, const void *log_alpha,
                        const void *beta, int64_t total_tokens, int32_t H, int32_t d_k,
                        int32_t d_v, kda_dtype dtype, float *M, float *S_tilde, void *o_scratch,
                        void *workspace, size_t workspace_bytes, kda_stream_t stream);

kda_status kda_cp_finish(const void *v, const float *S_in, int64_t total_tokens, int32_t H,
                         int32_t d_k, int32_t d_v, kda_dtype dtype, void *o, float *final_state,
                         void *workspace, size_t workspace_bytes, kda_stream_t stream);

/*
 * Backward pass (training): the gradients of a loss L through the recurrence
 * of kda_prefill, given dL/do and dL/dS_T (news digest page on Kimi Linear,
 * section "Algorithme parallele par chunks", which organises the operator for
 * training; the derivative is the chain rule through each step of the KDA
 * update of page "Kimi Linear" on docsaid.org, section "KDA : une
 * decroissance propre a chaque canal").
 *
 * Inputs are those of kda_prefill (same layouts, dtype, init_state NULL =
 * zeros, cu_seqlens NULL = num_seqs equal sequences), plus
 *   d_o            [T_total, H, d_v] in `dtype`: dL/do
 *   d_final_state  [N, H, d_k, d_v] fp32 or NULL (zero): dL/dS_T
 * Outputs, fp32, written in full (never accumulated):
 *   dq, dk, dlog_alpha [T_total, H, d_k];  dv [T_total, H, d_v];
 *   dbeta [T_total, H];  d_init_state [N, H, d_k, d_v] or NULL (not wanted).
 * gdn_backward is the same for the Gated DeltaNet gate: log_alpha and
 * dlog_alpha are [T_total, H].
 *
 * Shapes: d_k in {32, 64, 128}; d_v in {32, 64, 96, 128}; else
 * KDA_ERR_UNSUPPORTED.  Alignment: v, d_o, the fp32 states and dv 16 bytes;
 * the other inputs their element; the other outputs 4 bytes.  No output may
 * overlap an input, the workspace or another output (KDA_ERR_INVALID_ARG).
 * The workspace (256-byte aligned, kda_backward_workspace_size bytes) keeps
 * the state entering every 64-token block of every (sequence, head), about
 * T_total * H * d_k * d_v / 16 bytes, plus a per-CTA scratch.  The gradients
 * are summed with fp32 atomic adds, so their last bits may differ from run to
 * run.  A cu_seqlens entry out of order or past T_total skips that sequence
 * and sets the workspace error word (kda_check_workspace_error).
 */
size_t kda_backward_workspace_size(int32_t num_seqs, int64_t total_tokens, int32_t H,
                                   int32_t d_k, int32_t d_v);

kda_status kda_backward(const void *q, const void *k, const void *v, const void *log_alpha,
                        const void *beta, const float *init_state, const int32_t *cu_seqlens,
                        int32_t num_seqs, int64_t total_tokens, int32_t H, int32_t d_k,
                        int32_t d_v, kda_dtype dtype, const void *d_o,
                        const float *d_final_state, float *dq, float *dk, float *dv,
                        float *dlog_alpha, float *dbeta, float *d_init_state, void *workspace,
                        size_t workspace_bytes, kda_stream_t stream);

kda_status gdn_backward(const void *q, const void *k, const void *v, const void *log_alpha,
                        const void *beta, const float *init_state, const int32_t *cu_seqlens,
                        int32_t num_seqs, int64_t total_tokens, int32_t H, int32_t d_k,
                        int32_t d_v, kda_dtype dtype, const void *d_o,
                        const float *d_final_state, float *dq, float *dk, float *dv,
                        float *dlog_alpha, float *dbeta, float *d_init_state, void *workspace,
                        size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_backward for bf16 inputs with d_k = d_v = 128 by chunks (news digest
 * page on Kimi Linear, section "Algorithme parallele par chunks": the chunk
 * algebra, here differentiated): the prefill's chunk preparation, a forward
 * and a reverse scan over its per-chunk transition operands (one grid) for
 * every chunk's entering state and dL/dS at its end, then every (chunk,
 * head) item's gradients at once as products on the tensor cores.  A chunk
 * that decays below e^-80 within itself on some channel (log_alpha summing
 * below -80 over it) takes the token-by-token steps instead.  Same
 * arguments and outputs as kda_backward (bf16, d = 128 implied); the
 * workspace (256-byte aligned,
 * kda_backward_chunked_workspace_size bytes) also holds the prefill's records
 * and two bf16 states per (chunk, head).  The chunk boundary states and the
 * products' operands are bf16: gradients agree with kda_backward to the bf16
 * tolerance, not to fp32 rounding.  Every gradient element is written (the
 * per-channel path needs no zeroed outputs).
 */
size_t kda_backward_chunked_workspace_size(int32_t num_seqs, int64_t total_tokens, int32_t H);

kda_status kda_backward_chunked(const void *q, const void *k, const void *v, const void *log_alpha,
                                const void *beta, const float *init_state,
                                const int32_t *cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                                int32_t H, const void *d_o, const float *d_final_state, float *dq,
                                float *dk, float *dv, float *dlog_alpha, float *dbeta,
                                float *d_init_state, void *workspace, size_t workspace_bytes,
                                kda_stream_t stream);

/*
 * gdn_backward_chunked: kda_backward_chunked for the Gated DeltaNet gate
 * (log_alpha and dlog_alpha one value per token and head, [T_total, H]; the
 * gradient is the channel sum of the per-channel one), the same stages and
 * workspace size.
 */
kda_status gdn_backward_chunked(const void *q, const void *k, const void *v, const void *log_alpha,
                                const void *beta, const float *init_state,
                                const int32_t *cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                                int32_t H, const void *d_o, const float *d_final_state, float *dq,
                                float *dk, float *dv, float *dlog_alpha, float *dbeta,
                                float *d_init_state, void *workspace, size_t workspace_bytes,
                                kda_stream_t stream);

/*
 * Synchronises `stream`, then reads the error word that the prefill and
 * backward kernels leave at the start of `workspace` (non-zero when a
 * device-side check failed, e.g. cu_seqlens not non-decreasing or not ending
 * at T_total).  With workspace NULL it reads the word that
 * kda_prefill_noalloc leaves in its fixed array on the current device.
 * Returns KDA_ERR_INVALID_ARG in that case, KDA_OK otherwise (KDA_ERR_CUDA
 * if the word cannot be read).  Debugging aid; the only call here that
 * blocks.
 */
kda_status kda_check_workspace_error(const void *workspace,
                                     kda_stream_t stream);

/*
 * kda_prefill without a workspace argument, for callers that cannot allocate
 * device memory when they run the operator (an engine whose device memory
 * all belongs to its own pool, a loop that cannot afford cudaMalloc's
 * synchronisation, a plugin host that passes only a stream and tensors).
 * This call has no counterpart in the method's description; it is a
 * deployment convenience.
 *
 * Same arguments, results and errors as kda_prefill, minus the workspace.
 * The scratch it needs (the error word and the sequence-order table) lives
 * in a fixed array of this library's device memory, 256 + 4 *
 * KDA_NOALLOC_MAX_SEQS bytes, which every GPU that loads the library holds
 * until the process exits.  num_seqs above KDA_NOALLOC_MAX_SEQS returns
 * KDA_ERR_UNSUPPORTED.  It calls no allocating function.
 *
 * The first call on a device (with that device current) looks up the
 * array's device address and caches it; make that first call before any
 * stream capture.  All calls share the one array: calls that may overlap on
 * the GPU (different streams, or several host threads) race on it and must
 * be serialised by the caller.  The device-side checks of a call (a bad
 * cu_seqlens) leave their error word in the array: kda_check_workspace_error
 * with a NULL workspace reads it for the current device (it synchronises
 * `stream`).  The array's device address is looked up once per device and
 * kept for the life of the process; a cudaDeviceReset invalidates it, so a
 * process that resets a device must not call this entry point on it again.
 */
#define KDA_NOALLOC_MAX_SEQS 4096

kda_status kda_prefill_noalloc(const void *q, const void *k, const void *v,
                               const void *log_alpha, const void *beta,
                               const float *init_state, const int32_t *cu_seqlens,
                               int32_t num_seqs, int64_t total_tokens, int32_t H,
                               int32_t d_k, int32_t d_v, kda_dtype dtype, void *o,
                               float *final_state, kda_stream_t stream);

#ifdef __cplusplus
} /* extern "C" */
#endif

#endif /* KDA_H_ */
