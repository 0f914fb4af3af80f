// Internal helpers shared by the KDA CUDA kernels (not part of the C ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kda.h"

namespace kda {

// Element I/O for the two supported input/output types.
template <typename T> struct io;

template <> struct io<float> {
    static __device__ __forceinline__ float load(const float *p) { return *p; }
    static __device__ __forceinline__ void store(float *p, float x) { *p = x; }
};

template <> struct io<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16 *p) {
        return __bfloat162float(*p);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, float x) {
        *p = __float2bfloat16_rn(x);
    }
};

// Per-token log-decay floor.  A retention factor exp(-80) ~ 1.8e-35 already
// acts as zero against any state magnitude, and the floor keeps the
// within-chunk running sums finite (so differences of running sums are
// defined even for log_alpha = -inf).
constexpr float kLogAlphaFloor = -80.0f;

__device__ __forceinline__ float clamp_log_alpha(float g) {
    return fmaxf(g, kLogAlphaFloor);
}

// The layer's prologue and epilogue, fused into the kernels for the
// kda_layer_* entry points (page "Kimi Linear" on docsaid.org, section "Les
// autres pieces"; course page "Attention lineaire et recurrence", the gate
// -e^A Softplus(z) of Kimi Linear):
//   q, k <- x / sqrt(sum_c x_c^2 + qk_eps)           (L2 normalisation)
//   log_alpha = -exp(A_log[h]) softplus(z),  beta = sigmoid(beta_logit)
//   o <- o / sqrt(mean_j o_j^2 + norm_eps) * w_j * sigmoid(out_gate_j)
struct LayerArgs {
    const void *gate_z;        // [T, H, d_k], the I/O dtype
    const float *A_log;        // [H] fp32
    const void *beta_logit;    // [T, H], the I/O dtype
    const void *out_gate;      // [T, H, d_v], the I/O dtype, or null (no output gate)
    const float *norm_weight;  // [d_v] fp32, or null (ones)
    float qk_eps, norm_eps;
};

__device__ __forceinline__ float softplus_f(float x) { return x > 20.f ? x : log1pf(expf(x)); }

__device__ __forceinline__ float sigmoid_f(float x) { return 1.f / (1.f + expf(-x)); }

// Error word written by device-side checks into the workspace header.
enum : uint32_t {
    kDevErrNone = 0,
    kDevErrCuSeqlens = 1u << 0,   // cu_seqlens not non-decreasing / bad ends
    kDevErrTimeout = 1u << 1,     // a bounded wait gave up (internal error)
};

// Workspace layout: a 256-byte header holding the error word, then the
// per-kernel scratch areas.
constexpr size_t kWorkspaceHeader = 256;

// Launch set-up cached per (device, kernel) under a lock (kda_launch_setup.cu):
// the dynamic shared-memory limit of `func` on the current device, and the
// current device's SM count (148 if the query fails).
cudaError_t set_max_dynamic_smem(const void *func, int bytes);
int device_sm_count();

// Launchers (defined in the .cu files).  All return cudaGetLastError().
// `scalar_gate`: log_alpha holds one value per (token, head) ([T, H], the
// Gated DeltaNet gate) instead of one per key channel ([T, H, d_k]).
// `layer` (or null): the kda_layer_* prologue and epilogue; then g and beta
// are unused.
cudaError_t launch_decode(const void *q, const void *k, const void *v,
                          const void *g, const void *beta, float *state,
                          int batch, int H, int dk, int dv, kda_dtype dtype,
                          void *o, bool scalar_gate, const LayerArgs *layer,
                          cudaStream_t stream);

cudaError_t launch_prefill_simt(const void *q, const void *k, const void *v,
                                const void *g, const void *beta,
                                const float *init_state, const int32_t *cu,
                                int num_seqs, int64_t total_tokens, int H,
                                int dk, int dv, kda_dtype dtype, void *o,
                                float *final_state, uint32_t *err_word, bool scalar_gate,
                                cudaStream_t stream);

// Tensor-core prefill (bf16, d_k = d_v = 128).
size_t prefill_tc_workspace(int num_seqs);

cudaError_t launch_prefill_tc(const void *q, const void *k, const void *v, const void *g,
                              const void *beta, const float *init_state, const int32_t *cu,
                              int num_seqs, int64_t total_tokens, int H, void *o,
                              float *final_state, void *workspace, bool scalar_gate,
                              cudaStream_t stream);

// Tensor-core prefill split into a chunk-parallel preparation kernel and a
// state-chain kernel; its workspace holds one record per (chunk, head).
size_t prefill_split_workspace(int num_seqs, int64_t total_tokens, int H);

// With `layer`, g is the gate pre-activation and beta the logits (bf16,
// d = 128 only; the chain is then always whole-d_v).
// cp_mode (context parallelism, one segment of a sequence): kCpLocal also
// forms the segment's transition into cp_transition [N, H, d_k, d_k]
// (final_state then receives the state generated from init_state, o is
// scratch); kCpFinish runs only the chain over the records a kCpLocal call
// left in the same workspace.
// kPrepOnly: the plan and the chunk records only (no chain), for the
// backward pass's scans over the records.
enum : int { kCpNone = 0, kCpLocal = 1, kCpFinish = 2, kPrepOnly = 3 };

// The layer with its prologue as a pass of its own (log_alpha, beta and the
// inverse norms of q and k into the workspace), then the split path on the raw
// q and k scaled by those norms, and the epilogue; its workspace is
// layer_prefill_workspace bytes.
size_t layer_prefill_workspace(int num_seqs, int64_t total_tokens, int H);
cudaError_t launch_layer_prefill_split(const void *q, const void *k, const void *v, const LayerArgs &la,
                                       const float *init_state, const int32_t *cu, int num_seqs,
                                       int64_t total_tokens, int H, void *o, float *final_state,
                                       void *workspace, cudaStream_t stream);
cudaError_t launch_prefill_split(const void *q, const void *k, const void *v, const void *g,
                                 const void *beta, const float *init_state, const int32_t *cu,
                                 int num_seqs, int64_t total_tokens, int H, void *o,
                                 float *final_state, void *workspace, bool scalar_gate,
                                 const LayerArgs *layer, cudaStream_t stream,
                                 int cp_mode = kCpNone, float *cp_transition = nullptr,
                                 const float *nrm_in = nullptr);

// Backward pass (fp32 gradients; d_k and d_v multiples of 32 up to 128).
// Its workspace keeps the state entering every 64-step block of every
// (sequence, head) and gives each CTA a 64-state scratch.
size_t backward_workspace(int num_seqs, int64_t total_tokens, int H, int dk, int dv);

cudaError_t launch_backward(const void *q, const void *k, const void *v, const void *g,
                            const void *beta, const float *init_state, const int32_t *cu,
                            int num_seqs, int64_t total_tokens, int H, int dk, int dv,
                            kda_dtype dtype, const void *d_o, const float *d_final_state,
                            float *dq, float *dk_out, float *dv_out, float *dg, float *dbeta,
                            float *d_init_state, void *workspace, bool scalar_gate,
                            cudaStream_t stream);

// Backward pass through the chunk records (bf16, d_k = d_v = 128): the
// prefill's preparation, a forward and a reverse scan over the records for
// each chunk's entering state and dL/dS_next, then every chunk's steps at once.
size_t backward_chunked_workspace(int num_seqs, int64_t total_tokens, int H);
cudaError_t launch_backward_chunked(const void *q, const void *k, const void *v, const void *g,
                                    const void *beta, const float *init_state, const int32_t *cu,
                                    int num_seqs, int64_t total_tokens, int H, const void *d_o,
                                    const float *d_final_state, float *dq, float *dk_out,
                                    float *dv_out, float *dg, float *dbeta, float *d_init_state,
                                    void *workspace, bool scalar_gate, cudaStream_t stream);

// Where a split-path workspace keeps the plan's tables and the records.
struct SplitTables {
    const int32_t *chunk_off;    // [N + 1] first chunk of each sequence
    const int2 *chunk_tab;       // [chunks] (first token, length)
    const uint32_t *total_chunks;
    const uint8_t *recs;         // record (chunk, head) at recs + (chunk * H + head) * rec_stride
    size_t rec_stride;
    size_t max_chunks;
    // record field offsets: MP [128][128], YT [128][64], QP [64][128] bf16
    // (K-major, 128-byte swizzle, 64-column atoms), e^{G_L} 128 fp32
    uint32_t off_mp, off_yt, off_qp, off_egl;
};
SplitTables split_tables(const void *workspace, int num_seqs, int64_t total_tokens, int H);

// The backward pass's two scans over the records a kPrepOnly launch left in
// `workspace`, on the tensor cores (the transposed state chain): every chunk's
// entering state into s_in and dL/dS at every chunk's end into ds_next (both
// bf16 tiles [128 c][128 j] in the 128-byte-swizzled K-major layout of a
// tensor-core operand, two 16 KB K-atoms of 64 j, 32 KB per record, record
// order), dL/dS_0 into d_init_state (or not, when null).
cudaError_t launch_backward_scans(const void *v, const void *d_o, const float *init_state,
                                  const float *d_final_state, const int32_t *cu, int num_seqs,
                                  int64_t total_tokens, int H, void *workspace, void *s_in,
                                  void *ds_next, float *d_init_state, cudaStream_t stream);

// The fixed scratch array of kda_prefill_noalloc on the current device.
void *noalloc_scratch();

// Context parallelism: S_out = the state a segment starts from, given the
// (M_i, S~_i) of the n_prev segments before it and the sequence's S_0 (or null).
cudaError_t launch_cp_combine(const float *M, const float *S_tilde, const float *S0, float *S_out,
                              int n_prev, int H, int dk, int dv, cudaStream_t stream);

}  // namespace kda
