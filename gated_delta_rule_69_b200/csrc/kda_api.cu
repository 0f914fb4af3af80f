// C ABI of libkda.so: host-side validation and dispatch.  Declarations and
// the contract of each entry point are in include/kda.h.
#include <climits>

#include "kda_internal.cuh"

namespace {

constexpr int kVersion = 1 * 10000 + 0 * 100 + 0;

bool supported_dim(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }

bool aligned_to(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool aligned16(const void *p) { return aligned_to(p, 16); }

size_t elem_bytes(kda_dtype t) { return t == KDA_BF16 ? 2 : 4; }

bool overlaps(const void *a, size_t an, const void *b, size_t bn) {
    if (!a || !b || an == 0 || bn == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + bn && b0 < a0 + an;
}

kda_status from_cuda(cudaError_t e) { return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA; }

// The tensor-core path: bf16 I/O with 128 x 128 heads (token coordinates of
// its tensor maps are 32-bit).
bool use_tensor_cores(kda_dtype dtype, int d_k, int d_v, int64_t total_tokens) {
    return dtype == KDA_BF16 && d_k == 128 && d_v == 128 && total_tokens > 0 &&
           total_tokens <= INT_MAX;
}

// The prefill and the decode step for either gate: one log_alpha per key
// channel (KDA) or one per head (Gated DeltaNet).
kda_status prefill_impl(const void *q, const void *k, const void *v,
                        const void *log_alpha, const void *beta,
                        const float *init_state, const int32_t *cu_seqlens,
                        int32_t num_seqs, int64_t total_tokens, int32_t H,
                        int32_t d_k, int32_t d_v, kda_dtype dtype, void *o,
                        float *final_state, void *workspace,
                        size_t workspace_bytes, kda_stream_t stream_, bool scalar_gate,
                        const kda::LayerArgs *layer = nullptr) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (num_seqs < 1 || total_tokens < 0 || H < 1) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_BF16 && dtype != KDA_FP32) return KDA_ERR_INVALID_ARG;
    if (!supported_dim(d_k) || !supported_dim(d_v)) return KDA_ERR_UNSUPPORTED;
    if ((int64_t)num_seqs * H > INT_MAX) return KDA_ERR_UNSUPPORTED;
    if (!cu_seqlens && total_tokens % num_seqs != 0) return KDA_ERR_INVALID_ARG;
    if (total_tokens > 0 && (!q || !k || !v || !log_alpha || !beta || !o))
        return KDA_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, scalar_gate ? nullptr : log_alpha, init_state, o, final_state};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_INVALID_ARG;
    if (beta && !aligned_to(beta, elem_bytes(dtype))) return KDA_ERR_INVALID_ARG;
    if (scalar_gate && log_alpha && !aligned_to(log_alpha, elem_bytes(dtype))) return KDA_ERR_INVALID_ARG;
    if (cu_seqlens && !aligned_to(cu_seqlens, 4)) return KDA_ERR_INVALID_ARG;
    // The least workspace any path accepts; the two-kernel tensor-core path is
    // taken when the workspace also holds its per-chunk records.
    const size_t need = kda::prefill_tc_workspace(num_seqs);
    if (!workspace || workspace_bytes < need) return KDA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KDA_ERR_INVALID_ARG;

    const size_t eb = elem_bytes(dtype);
    const size_t nk = (size_t)total_tokens * H * d_k * eb;
    const size_t nv = (size_t)total_tokens * H * d_v * eb;
    const size_t nb = (size_t)total_tokens * H * eb;
    const size_t ng = scalar_gate ? nb : nk;
    const size_t ns = (size_t)num_seqs * H * d_k * d_v * sizeof(float);
    if (overlaps(o, nv, q, nk) || overlaps(o, nv, k, nk) || overlaps(o, nv, v, nv) ||
        overlaps(o, nv, log_alpha, ng) || overlaps(o, nv, beta, nb) ||
        overlaps(o, nv, init_state, ns) || overlaps(o, nv, final_state, ns) ||
        overlaps(o, nv, workspace, workspace_bytes))
        return KDA_ERR_INVALID_ARG;
    if (init_state && final_state && init_state != final_state &&
        overlaps(init_state, ns, final_state, ns))
        return KDA_ERR_INVALID_ARG;

    if (layer) {   // the fused layer runs on the two-kernel tensor-core path only
        if (total_tokens > 0 && !use_tensor_cores(dtype, d_k, d_v, total_tokens))
            return KDA_ERR_UNSUPPORTED;
        if (total_tokens > 0 &&
            workspace_bytes < kda::prefill_split_workspace(num_seqs, total_tokens, H))
            return KDA_ERR_WORKSPACE;
        if (!layer->A_log || !aligned_to(layer->A_log, 4) ||
            (layer->norm_weight && !aligned_to(layer->norm_weight, 4)) ||
            (layer->out_gate && !aligned16(layer->out_gate)) ||
            !(layer->qk_eps >= 0.f) || !(layer->norm_eps >= 0.f) ||
            overlaps(o, nv, layer->out_gate, nv))
            return KDA_ERR_INVALID_ARG;
    }
    if (layer && total_tokens > 0 &&
        workspace_bytes >= kda::layer_prefill_workspace(num_seqs, total_tokens, H))
        return from_cuda(kda::launch_layer_prefill_split(q, k, v, *layer, init_state, cu_seqlens, num_seqs,
                                                         total_tokens, H, o, final_state, workspace, stream));
    if (use_tensor_cores(dtype, d_k, d_v, total_tokens) &&
        workspace_bytes >= kda::prefill_split_workspace(num_seqs, total_tokens, H))
        return from_cuda(kda::launch_prefill_split(q, k, v, log_alpha, beta, init_state,
                                                   cu_seqlens, num_seqs, total_tokens, H, o,
                                                   final_state, workspace, scalar_gate, layer,
                                                   stream));
    if (use_tensor_cores(dtype, d_k, d_v, total_tokens))
        return from_cuda(kda::launch_prefill_tc(q, k, v, log_alpha, beta, init_state, cu_seqlens,
                                                num_seqs, total_tokens, H, o, final_state,
                                                workspace, scalar_gate, stream));
    uint32_t *err_word = static_cast<uint32_t *>(workspace);
    cudaError_t e = cudaMemsetAsync(err_word, 0, sizeof(uint32_t), stream);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    e = kda::launch_prefill_simt(q, k, v, log_alpha, beta, init_state, cu_seqlens,
                                 num_seqs, total_tokens, H, d_k, d_v, dtype, o,
                                 final_state, err_word, scalar_gate, stream);
    return from_cuda(e);
}

kda_status decode_impl(const void *q, const void *k, const void *v,
                       const void *log_alpha, const void *beta,
                       float *state, int32_t batch, int32_t H,
                       int32_t d_k, int32_t d_v, kda_dtype dtype, void *o,
                       kda_stream_t stream_, bool scalar_gate,
                       const kda::LayerArgs *layer = nullptr) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (batch < 0 || H < 1) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_BF16 && dtype != KDA_FP32) return KDA_ERR_INVALID_ARG;
    if (!supported_dim(d_k) || !supported_dim(d_v)) return KDA_ERR_UNSUPPORTED;
    if ((int64_t)batch * H > INT_MAX) return KDA_ERR_UNSUPPORTED;
    if (batch == 0) return KDA_OK;
    if (!q || !k || !v || !log_alpha || !beta || !state || !o) return KDA_ERR_INVALID_ARG;
    const size_t eb = elem_bytes(dtype);
    const void *ptrs[] = {q, k, v, log_alpha, beta, o};
    for (const void *p : ptrs)
        if (!aligned_to(p, eb)) return KDA_ERR_INVALID_ARG;
    if (!aligned16(state)) return KDA_ERR_INVALID_ARG;
    const size_t nk = (size_t)batch * H * d_k * eb;
    const size_t nv = (size_t)batch * H * d_v * eb;
    const size_t nb = (size_t)batch * H * eb;
    const size_t ng = scalar_gate ? nb : nk;
    const size_t ns = (size_t)batch * H * d_k * d_v * sizeof(float);
    if (overlaps(o, nv, q, nk) || overlaps(o, nv, k, nk) || overlaps(o, nv, v, nv) ||
        overlaps(o, nv, log_alpha, ng) || overlaps(o, nv, beta, nb) ||
        overlaps(o, nv, state, ns))
        return KDA_ERR_INVALID_ARG;
    if (layer && (!layer->A_log || !aligned_to(layer->A_log, 4) ||
                  (layer->norm_weight && !aligned_to(layer->norm_weight, 4)) ||
                  (layer->out_gate && !aligned_to(layer->out_gate, eb)) ||
                  !(layer->qk_eps >= 0.f) || !(layer->norm_eps >= 0.f) ||
                  overlaps(o, nv, layer->out_gate, nv)))
        return KDA_ERR_INVALID_ARG;
    return from_cuda(kda::launch_decode(q, k, v, log_alpha, beta, state, batch, H,
                                        d_k, d_v, dtype, o, scalar_gate, layer, stream));
}

// The backward pass for either gate (gradients in fp32).
kda_status backward_impl(const void *q, const void *k, const void *v, const void *log_alpha,
                         const void *beta, const float *init_state, const int32_t *cu_seqlens,
                         int32_t num_seqs, int64_t total_tokens, int32_t H, int32_t d_k,
                         int32_t d_v, kda_dtype dtype, const void *d_o,
                         const float *d_final_state, float *dq, float *dk, float *dv,
                         float *dlog_alpha, float *dbeta, float *d_init_state, void *workspace,
                         size_t workspace_bytes, kda_stream_t stream_, bool scalar_gate) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (num_seqs < 1 || total_tokens < 0 || H < 1) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_BF16 && dtype != KDA_FP32) return KDA_ERR_INVALID_ARG;
    const bool dims_ok = (d_k == 32 || d_k == 64 || d_k == 128) && d_v % 32 == 0 &&
                         d_v >= 32 && d_v <= 128;
    if (!dims_ok) return KDA_ERR_UNSUPPORTED;
    if ((int64_t)num_seqs * H * (d_v / 32) > INT_MAX) return KDA_ERR_UNSUPPORTED;
    if (!cu_seqlens && total_tokens % num_seqs != 0) return KDA_ERR_INVALID_ARG;
    if (total_tokens > 0 && (!q || !k || !v || !log_alpha || !beta || !d_o || !dq || !dk ||
                             !dv || !dlog_alpha || !dbeta))
        return KDA_ERR_INVALID_ARG;
    const size_t eb = elem_bytes(dtype);
    // v and d_o are read 4 columns at a time; states and dv 16 bytes at a time
    const void *p16[] = {v, d_o, init_state, d_final_state, dv, d_init_state};
    for (const void *p : p16)
        if (p && !aligned16(p)) return KDA_ERR_INVALID_ARG;
    const void *pe[] = {q, k, log_alpha, beta};
    for (const void *p : pe)
        if (p && !aligned_to(p, eb)) return KDA_ERR_INVALID_ARG;
    const void *p4[] = {dq, dk, dlog_alpha, dbeta, cu_seqlens};
    for (const void *p : p4)
        if (p && !aligned_to(p, 4)) return KDA_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < kda::backward_workspace(num_seqs, total_tokens, H, d_k, d_v))
        return KDA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KDA_ERR_INVALID_ARG;

    // no output may overlap an input, the workspace or another output
    const size_t nk = (size_t)total_tokens * H * d_k, nv = (size_t)total_tokens * H * d_v;
    const size_t nb = (size_t)total_tokens * H, ng = scalar_gate ? nb : nk;
    const size_t ns = (size_t)num_seqs * H * d_k * d_v;
    struct Span { const void *p; size_t n; };
    const Span ins[] = {{q, nk * eb}, {k, nk * eb}, {v, nv * eb}, {log_alpha, ng * eb},
                        {beta, nb * eb}, {d_o, nv * eb}, {init_state, ns * 4},
                        {d_final_state, ns * 4}, {cu_seqlens, ((size_t)num_seqs + 1) * 4},
                        {workspace, workspace_bytes}};
    const Span outs[] = {{dq, nk * 4}, {dk, nk * 4}, {dv, nv * 4}, {dlog_alpha, ng * 4},
                         {dbeta, nb * 4}, {d_init_state, ns * 4}};
    for (const Span &o : outs) {
        for (const Span &i : ins)
            if (overlaps(o.p, o.n, i.p, i.n)) return KDA_ERR_INVALID_ARG;
        for (const Span &o2 : outs)
            if (&o2 != &o && overlaps(o.p, o.n, o2.p, o2.n)) return KDA_ERR_INVALID_ARG;
    }
    return from_cuda(kda::launch_backward(q, k, v, log_alpha, beta, init_state, cu_seqlens,
                                          num_seqs, total_tokens, H, d_k, d_v, dtype, d_o,
                                          d_final_state, dq, dk, dv, dlog_alpha, dbeta,
                                          d_init_state, workspace, scalar_gate, stream));
}

}  // namespace

extern "C" {

const char *kda_status_string(kda_status s) {
    switch (s) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG: invalid argument";
        case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED: shape or dtype not supported";
        case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE: workspace missing or too small";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA: CUDA runtime error";
    }
    return "KDA_ERR_UNKNOWN";
}

int kda_version(void) { return kVersion; }

size_t kda_prefill_workspace_size(int32_t num_seqs, int64_t total_tokens,
                                  int32_t H, int32_t d_k, int32_t d_v) {
    if (num_seqs < 1 || total_tokens < 0 || H < 1) return 0;
    if (!supported_dim(d_k) || !supported_dim(d_v)) return 0;
    if (d_k == 128 && d_v == 128 && total_tokens > 0)
        return kda::prefill_split_workspace(num_seqs, total_tokens, H);
    return kda::prefill_tc_workspace(num_seqs);
}

kda_status kda_prefill(const void *q, const void *k, const void *v,
                       const void *log_alpha, const void *beta,
                       const float *init_state, const int32_t *cu_seqlens,
                       int32_t num_seqs, int64_t total_tokens, int32_t H,
                       int32_t d_k, int32_t d_v, kda_dtype dtype, void *o,
                       float *final_state, void *workspace,
                       size_t workspace_bytes, kda_stream_t stream) {
    return prefill_impl(q, k, v, log_alpha, beta, init_state, cu_seqlens, num_seqs, total_tokens,
                        H, d_k, d_v, dtype, o, final_state, workspace, workspace_bytes, stream,
                        false);
}

kda_status gdn_prefill(const void *q, const void *k, const void *v,
                       const void *log_alpha, const void *beta,
                       const float *init_state, const int32_t *cu_seqlens,
                       int32_t num_seqs, int64_t total_tokens, int32_t H,
                       int32_t d_k, int32_t d_v, kda_dtype dtype, void *o,
                       float *final_state, void *workspace,
                       size_t workspace_bytes, kda_stream_t stream) {
    return prefill_impl(q, k, v, log_alpha, beta, init_state, cu_seqlens, num_seqs, total_tokens,
                        H, d_k, d_v, dtype, o, final_state, workspace, workspace_bytes, stream,
                        true);
}

kda_status kda_decode_step(const void *q, const void *k, const void *v,
                           const void *log_alpha, const void *beta,
                           float *state, int32_t batch, int32_t H,
                           int32_t d_k, int32_t d_v, kda_dtype dtype, void *o,
                           kda_stream_t stream) {
    return decode_impl(q, k, v, log_alpha, beta, state, batch, H, d_k, d_v, dtype, o, stream,
                       false);
}

kda_status gdn_decode_step(const void *q, const void *k, const void *v,
                           const void *log_alpha, const void *beta,
                           float *state, int32_t batch, int32_t H,
                           int32_t d_k, int32_t d_v, kda_dtype dtype, void *o,
                           kda_stream_t stream) {
    return decode_impl(q, k, v, log_alpha, beta, state, batch, H, d_k, d_v, dtype, o, stream,
                       true);
}

size_t kda_layer_prefill_workspace_size(int32_t num_seqs, int64_t total_tokens, int32_t H, int32_t d_k,
                                        int32_t d_v) {
    if (num_seqs < 1 || total_tokens < 0 || H < 1 || d_k != 128 || d_v != 128) return 0;
    return kda::layer_prefill_workspace(num_seqs, total_tokens, H);
}

kda_status kda_layer_prefill(const void *q, const void *k, const void *v, const void *gate_z,
                             const float *A_log, const void *beta_logit, const void *out_gate,
                             const float *norm_weight, float qk_eps, float norm_eps,
                             const float *init_state, const int32_t *cu_seqlens,
                             int32_t num_seqs, int64_t total_tokens, int32_t H, int32_t d_k,
                             int32_t d_v, kda_dtype dtype, void *o, float *final_state,
                             void *workspace, size_t workspace_bytes, kda_stream_t stream) {
    const kda::LayerArgs la = {gate_z, A_log, beta_logit, out_gate, norm_weight, qk_eps, norm_eps};
    return prefill_impl(q, k, v, gate_z, beta_logit, init_state, cu_seqlens, num_seqs,
                        total_tokens, H, d_k, d_v, dtype, o, final_state, workspace,
                        workspace_bytes, stream, false, &la);
}

kda_status kda_layer_decode_step(const void *q, const void *k, const void *v,
                                 const void *gate_z, const float *A_log, const void *beta_logit,
                                 const void *out_gate, const float *norm_weight, float qk_eps,
                                 float norm_eps, float *state, int32_t batch, int32_t H,
                                 int32_t d_k, int32_t d_v, kda_dtype dtype, void *o,
                                 kda_stream_t stream) {
    const kda::LayerArgs la = {gate_z, A_log, beta_logit, out_gate, norm_weight, qk_eps, norm_eps};
    return decode_impl(q, k, v, gate_z, beta_logit, state, batch, H, d_k, d_v, dtype, o, stream,
                       false, &la);
}

kda_status kda_cp_combine(const float *M, const float *S_tilde, const float *S0, float *S_in,
                          int32_t n_prev, int32_t H, int32_t d_k, int32_t d_v,
                          kda_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (n_prev < 0 || H < 1) return KDA_ERR_INVALID_ARG;
    if (!supported_dim(d_k) || !supported_dim(d_v) || d_v < 32) return KDA_ERR_UNSUPPORTED;
    if (!S_in || (n_prev > 0 && (!M || !S_tilde))) return KDA_ERR_INVALID_ARG;
    const void *ptrs[] = {M, S_tilde, S0, S_in};
    for (const void *p : ptrs)
        if (p && !aligned_to(p, 4)) return KDA_ERR_INVALID_ARG;
    const size_t ns = (size_t)H * d_k * d_v * sizeof(float);
    const size_t nm = (size_t)n_prev * H * d_k * d_k * sizeof(float);
    if (overlaps(S_in, ns, M, nm) || overlaps(S_in, ns, S_tilde, (size_t)n_prev * ns) ||
        (S0 && S0 != S_in && overlaps(S_in, ns, S0, ns)))
        return KDA_ERR_INVALID_ARG;
    return from_cuda(kda::launch_cp_combine(M, S_tilde, S0, S_in, n_prev, H, d_k, d_v, stream));
}

kda_status kda_cp_local(const void *q, const void *k, const void *v, const void *log_alpha,
                        const void *beta, int64_t total_tokens, int32_t H, int32_t d_k,
                        int32_t d_v, kda_dtype dtype, float *M, float *S_tilde, void *o_scratch,
                        void *workspace, size_t workspace_bytes, kda_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (total_tokens < 1 || H < 1) return KDA_ERR_INVALID_ARG;
    if (!use_tensor_cores(dtype, d_k, d_v, total_tokens)) return KDA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !log_alpha || !beta || !M || !S_tilde)
        return KDA_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, log_alpha, M, S_tilde, o_scratch};
    for (const void *p : ptrs)
        if (!aligned16(p)) return KDA_ERR_INVALID_ARG;
    if (!aligned_to(beta, 2)) return KDA_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < kda::prefill_split_workspace(1, total_tokens, H))
        return KDA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KDA_ERR_INVALID_ARG;
    const size_t nk = (size_t)total_tokens * H * d_k * 2, nb = (size_t)total_tokens * H * 2;
    const size_t ns = (size_t)H * d_k * d_v * sizeof(float);
    const void *ins[] = {q, k, v, log_alpha};
    for (const void *in : ins)
        if (overlaps(M, ns, in, nk) || overlaps(S_tilde, ns, in, nk) || overlaps(o_scratch, nk, in, nk))
            return KDA_ERR_INVALID_ARG;
    if (overlaps(M, ns, S_tilde, ns) || overlaps(M, ns, o_scratch, nk) ||
        overlaps(S_tilde, ns, o_scratch, nk) || overlaps(o_scratch, nk, beta, nb) ||
        overlaps(o_scratch, nk, workspace, workspace_bytes))
        return KDA_ERR_INVALID_ARG;
    return from_cuda(kda::launch_prefill_split(q, k, v, log_alpha, beta, nullptr, nullptr, 1,
                                               total_tokens, H, o_scratch, S_tilde, workspace,
                                               false, nullptr, stream, kda::kCpLocal, M));
}

kda_status kda_cp_finish(const void *v, const float *S_in, int64_t total_tokens, int32_t H,
                         int32_t d_k, int32_t d_v, kda_dtype dtype, void *o, float *final_state,
                         void *workspace, size_t workspace_bytes, kda_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (total_tokens < 1 || H < 1) return KDA_ERR_INVALID_ARG;
    if (!use_tensor_cores(dtype, d_k, d_v, total_tokens)) return KDA_ERR_UNSUPPORTED;
    if (!v || !o) return KDA_ERR_INVALID_ARG;
    const void *ptrs[] = {v, S_in, o, final_state};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < kda::prefill_split_workspace(1, total_tokens, H))
        return KDA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KDA_ERR_INVALID_ARG;
    const size_t nv = (size_t)total_tokens * H * d_v * 2;
    const size_t ns = (size_t)H * d_k * d_v * sizeof(float);
    if (overlaps(o, nv, v, nv) || overlaps(o, nv, S_in, ns) || overlaps(o, nv, final_state, ns) ||
        overlaps(o, nv, workspace, workspace_bytes) ||
        (S_in && final_state && S_in != final_state && overlaps(S_in, ns, final_state, ns)))
        return KDA_ERR_INVALID_ARG;
    return from_cuda(kda::launch_prefill_split(nullptr, nullptr, v, nullptr, nullptr, S_in, nullptr,
                                               1, total_tokens, H, o, final_state, workspace,
                                               false, nullptr, stream, kda::kCpFinish, nullptr));
}

size_t kda_backward_workspace_size(int32_t num_seqs, int64_t total_tokens, int32_t H,
                                   int32_t d_k, int32_t d_v) {
    if (num_seqs < 1 || total_tokens < 0 || H < 1 || d_k < 32 || d_k > 128 || d_v < 32 ||
        d_v > 128 || d_v % 32 != 0)
        return 0;
    return kda::backward_workspace(num_seqs, total_tokens, H, d_k, d_v);
}

kda_status kda_backward(const void *q, const void *k, const void *v, const void *log_alpha,
                        const void *beta, const float *init_state, const int32_t *cu_seqlens,
                        int32_t num_seqs, int64_t total_tokens, int32_t H, int32_t d_k,
                        int32_t d_v, kda_dtype dtype, const void *d_o,
                        const float *d_final_state, float *dq, float *dk, float *dv,
                        float *dlog_alpha, float *dbeta, float *d_init_state, void *workspace,
                        size_t workspace_bytes, kda_stream_t stream) {
    return backward_impl(q, k, v, log_alpha, beta, init_state, cu_seqlens, num_seqs,
                         total_tokens, H, d_k, d_v, dtype, d_o, d_final_state, dq, dk, dv,
                         dlog_alpha, dbeta, d_init_state, workspace, workspace_bytes, stream,
                         false);
}

kda_status gdn_backward(const void *q, const void *k, const void *v, const void *log_alpha,
                        const void *beta, const float *init_state, const int32_t *cu_seqlens,
                        int32_t num_seqs, int64_t total_tokens, int32_t H, int32_t d_k,
                        int32_t d_v, kda_dtype dtype, const void *d_o,
                        const float *d_final_state, float *dq, float *dk, float *dv,
                        float *dlog_alpha, float *dbeta, float *d_init_state, void *workspace,
                        size_t workspace_bytes, kda_stream_t stream) {
    return backward_impl(q, k, v, log_alpha, beta, init_state, cu_seqlens, num_seqs,
                         total_tokens, H, d_k, d_v, dtype, d_o, d_final_state, dq, dk, dv,
                         dlog_alpha, dbeta, d_init_state, workspace, workspace_bytes, stream,
                         true);
}

size_t kda_backward_chunked_workspace_size(int32_t num_seqs, int64_t total_tokens, int32_t H) {
    if (num_seqs < 1 || total_tokens < 0 || H < 1) return 0;
    return kda::backward_chunked_workspace(num_seqs, total_tokens, H);
}

namespace {

kda_status backward_chunked_impl(const void *q, const void *k, const void *v, const void *log_alpha,
                                 const void *beta, const float *init_state,
                                 const int32_t *cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                                 int32_t H, const void *d_o, const float *d_final_state, float *dq,
                                 float *dk, float *dv, float *dlog_alpha, float *dbeta,
                                 float *d_init_state, void *workspace, size_t workspace_bytes,
                                 kda_stream_t stream_, bool scalar_gate) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (num_seqs < 1 || total_tokens < 1 || total_tokens > INT_MAX || H < 1)
        return KDA_ERR_INVALID_ARG;
    if (!cu_seqlens && total_tokens % num_seqs != 0) return KDA_ERR_INVALID_ARG;
    if (!q || !k || !v || !log_alpha || !beta || !d_o || !dq || !dk || !dv || !dlog_alpha || !dbeta)
        return KDA_ERR_INVALID_ARG;
    const void *p16[] = {q, k, v, scalar_gate ? nullptr : log_alpha, d_o, init_state, d_final_state, dv,
                         d_init_state};
    for (const void *p : p16)
        if (p && !aligned16(p)) return KDA_ERR_INVALID_ARG;
    const void *p4[] = {dq, dk, dlog_alpha, dbeta, cu_seqlens};
    for (const void *p : p4)
        if (p && !aligned_to(p, 4)) return KDA_ERR_INVALID_ARG;
    if (beta && !aligned_to(beta, 2)) return KDA_ERR_INVALID_ARG;
    if (scalar_gate && !aligned_to(log_alpha, 2)) return KDA_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < kda::backward_chunked_workspace(num_seqs, total_tokens, H))
        return KDA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KDA_ERR_INVALID_ARG;
    return from_cuda(kda::launch_backward_chunked(q, k, v, log_alpha, beta, init_state, cu_seqlens,
                                                  num_seqs, total_tokens, H, d_o, d_final_state,
                                                  dq, dk, dv, dlog_alpha, dbeta, d_init_state,
                                                  workspace, scalar_gate, stream));
}

}  // namespace

kda_status kda_backward_chunked(const void *q, const void *k, const void *v, const void *log_alpha,
                                const void *beta, const float *init_state,
                                const int32_t *cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                                int32_t H, const void *d_o, const float *d_final_state, float *dq,
                                float *dk, float *dv, float *dlog_alpha, float *dbeta,
                                float *d_init_state, void *workspace, size_t workspace_bytes,
                                kda_stream_t stream) {
    return backward_chunked_impl(q, k, v, log_alpha, beta, init_state, cu_seqlens, num_seqs, total_tokens,
                                 H, d_o, d_final_state, dq, dk, dv, dlog_alpha, dbeta, d_init_state,
                                 workspace, workspace_bytes, stream, false);
}

kda_status gdn_backward_chunked(const void *q, const void *k, const void *v, const void *log_alpha,
                                const void *beta, const float *init_state,
                                const int32_t *cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                                int32_t H, const void *d_o, const float *d_final_state, float *dq,
                                float *dk, float *dv, float *dlog_alpha, float *dbeta,
                                float *d_init_state, void *workspace, size_t workspace_bytes,
                                kda_stream_t stream) {
    return backward_chunked_impl(q, k, v, log_alpha, beta, init_state, cu_seqlens, num_seqs, total_tokens,
                                 H, d_o, d_final_state, dq, dk, dv, dlog_alpha, dbeta, d_init_state,
                                 workspace, workspace_bytes, stream, true);
}

kda_status kda_check_workspace_error(const void *workspace, kda_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (!workspace) {   // the no-workspace entry point's array on the current device
        workspace = kda::noalloc_scratch();
        if (!workspace) return KDA_ERR_CUDA;
    }
    if (cudaStreamSynchronize(stream) != cudaSuccess) return KDA_ERR_CUDA;
    uint32_t word = 0;
    if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
        return KDA_ERR_CUDA;
    return word == kda::kDevErrNone ? KDA_OK : KDA_ERR_INVALID_ARG;
}

}  // extern "C"
