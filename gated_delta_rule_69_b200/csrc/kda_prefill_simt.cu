// KDA chunkwise prefill on CUDA cores, fp32 throughout (the accurate test
// mode, and the path for head sizes the tensor-core kernel does not cover).
//
// The sequence is processed in chunks of C = 64 tokens: within a chunk the
// work is dense linear algebra, and only the d_k x d_v state is carried from
// one chunk to the next (news digest page on Kimi Linear, section
// "Algorithme parallele par chunks"; course page "Attention lineaire et
// recurrence", section "Le calcul par blocs").
//
// Chunk algebra.  With G_t the running sum of log_alpha inside the chunk
// (per key channel) and S0 the state entering the chunk, unrolling
// S_t = D_t S_{t-1} + k_t u_t^T, u_t = beta_t (v_t - (D_t S_{t-1})^T k_t) gives
//     A[t][i] = beta_t sum_c k_tc k_ic exp(G_tc - G_ic)     (i < t)
//     P[t][i] =        sum_c q_tc k_ic exp(G_tc - G_ic)     (i <= t)
//     (I + A) U = diag(beta) (V - Ktil S0),   Ktil = K * exp(G)
//     O = Qtil S0 + P U,                       Qtil = Q * exp(G)
//     S_next = Diag(exp(G_L)) S0 + Kbar^T U,   Kbar = K * exp(G_L - G)
// The lower-triangular system is solved by forward substitution, row after
// row (news digest page, same section: the triangular inverse by forward
// substitution).  Every exponent above is <= 0 because log_alpha <= 0, so no
// factor can overflow (the cumulative-decay trap of the course page, section
// "Le piege numerique de la decroissance cumulee": dividing by the cumulative
// decay overflows; differences of running sums taken pairwise do not).
//
// One CTA per (sequence, head), 256 threads, everything in shared memory.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kChunk = 64;
constexpr int kThreads = 256;

template <int DK, int DV>
struct SimtSmem {
    static constexpr int KP = DK + 1;  // padded row stride of the [C][DK] tiles
    static constexpr int AP = kChunk + 1;
    static constexpr size_t S = 0;                                   // [DK][DV]
    static constexpr size_t K = S + (size_t)DK * DV;                 // [C][KP]
    static constexpr size_t G = K + (size_t)kChunk * KP;             // [C][KP]
    static constexpr size_t Q = G + (size_t)kChunk * KP;             // [C][KP]
    static constexpr size_t V = Q + (size_t)kChunk * KP;             // [C][DV]
    static constexpr size_t A = V + (size_t)kChunk * DV;             // [C][AP]
    static constexpr size_t P = A + (size_t)kChunk * AP;             // [C][AP]
    static constexpr size_t B = P + (size_t)kChunk * AP;             // [C]
    static constexpr size_t GL = B + kChunk;                         // [DK]
    static constexpr size_t floats = GL + DK;
    static constexpr size_t bytes = floats * sizeof(float);
};

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(kThreads)
kda_prefill_simt_kernel(const T *__restrict__ q, const T *__restrict__ k,
                        const T *__restrict__ v, const T *__restrict__ g,
                        const T *__restrict__ beta,
                        const float *init_state, const int32_t *__restrict__ cu,
                        int num_seqs, int64_t total_tokens, int H,
                        T *__restrict__ o, float *final_state,
                        uint32_t *err_word, int scalar_gate) {
    using L = SimtSmem<DK, DV>;
    constexpr int KP = L::KP, AP = L::AP;
    extern __shared__ __align__(16) float sm[];
    float *S = sm + L::S, *Ks = sm + L::K, *Gs = sm + L::G, *Qs = sm + L::Q;
    float *Vs = sm + L::V, *As = sm + L::A, *Ps = sm + L::P;
    float *Bs = sm + L::B, *GLs = sm + L::GL;

    const int tid = threadIdx.x;
    const int seq = blockIdx.x / H;
    const int h = blockIdx.x % H;
    int64_t bos, eos;
    if (cu) {
        bos = cu[seq];
        eos = cu[seq + 1];
        const bool bad = bos < 0 || eos < bos || eos > total_tokens ||
                         (seq == 0 && bos != 0) ||
                         (seq == num_seqs - 1 && eos != total_tokens);
        if (bad) {
            if (tid == 0) atomicOr(err_word, kDevErrCuSeqlens);
            bos = eos = 0;  // process nothing; the state passes through
        }
    } else {
        const int64_t len = total_tokens / num_seqs;
        bos = (int64_t)seq * len;
        eos = bos + len;
    }

    const size_t state_off = ((size_t)seq * H + h) * (size_t)(DK * DV);
    for (int idx = tid; idx < DK * DV; idx += kThreads)
        S[idx] = init_state ? init_state[state_off + idx] : 0.f;
    // (the first __syncthreads of the chunk loop orders these writes)

    for (int64_t cs = bos; cs < eos; cs += kChunk) {
        const int Lc = (int)min((int64_t)kChunk, eos - cs);
        __syncthreads();  // previous chunk fully consumed
        for (int idx = tid; idx < Lc * DK; idx += kThreads) {
            const int t = idx / DK, c = idx % DK;
            const size_t gi = ((size_t)(cs + t) * H + h) * DK + c;
            Ks[t * KP + c] = io<T>::load(k + gi);
            Qs[t * KP + c] = io<T>::load(q + gi);
            const size_t gg = scalar_gate ? (size_t)(cs + t) * H + h : gi;
            Gs[t * KP + c] = clamp_log_alpha(io<T>::load(g + gg));
        }
        for (int idx = tid; idx < Lc * DV; idx += kThreads) {
            const int t = idx / DV, j = idx % DV;
            Vs[t * DV + j] = io<T>::load(v + ((size_t)(cs + t) * H + h) * DV + j);
        }
        for (int t = tid; t < Lc; t += kThreads)
            Bs[t] = io<T>::load(beta + (size_t)(cs + t) * H + h);
        __syncthreads();

        // Running sum of log_alpha along the chunk, per key channel.
        for (int c = tid; c < DK; c += kThreads) {
            float run = 0.f;
            for (int t = 0; t < Lc; ++t) {
                run += Gs[t * KP + c];
                Gs[t * KP + c] = run;
            }
            GLs[c] = run;
        }
        __syncthreads();

        // A (strictly lower, with beta) and P (lower) from pairwise decays.
        for (int p = tid; p < Lc * Lc; p += kThreads) {
            const int r = p / Lc, i = p % Lc;
            if (i > r) continue;
            float ak = 0.f, aq = 0.f;
            const float *kr = Ks + r * KP, *ki = Ks + i * KP, *qr = Qs + r * KP;
            const float *gr = Gs + r * KP, *gi = Gs + i * KP;
#pragma unroll 8
            for (int c = 0; c < DK; ++c) {
                const float kd = ki[c] * expf(gr[c] - gi[c]);
                ak = fmaf(kr[c], kd, ak);
                aq = fmaf(qr[c], kd, aq);
            }
            As[r * AP + i] = (i < r) ? Bs[r] * ak : 0.f;
            Ps[r * AP + i] = aq;
        }
        __syncthreads();

        // Gated operands, in place: K -> Ktil, G -> Kbar, Q -> Qtil.
        for (int idx = tid; idx < Lc * DK; idx += kThreads) {
            const int t = idx / DK, c = idx % DK;
            const float kv = Ks[t * KP + c], gv = Gs[t * KP + c];
            const float e = expf(gv);
            Ks[t * KP + c] = kv * e;
            Gs[t * KP + c] = kv * expf(GLs[c] - gv);
            Qs[t * KP + c] *= e;
        }
        __syncthreads();

        // Right-hand side: diag(beta) (V - Ktil S0), in place in V.
        for (int idx = tid; idx < Lc * DV; idx += kThreads) {
            const int t = idx / DV, j = idx % DV;
            float acc = Vs[t * DV + j];
            const float *kt = Ks + t * KP;
#pragma unroll 8
            for (int c = 0; c < DK; ++c) acc = fmaf(-kt[c], S[c * DV + j], acc);
            Vs[t * DV + j] = Bs[t] * acc;
        }
        __syncthreads();

        // Forward substitution (I + A) U = RHS, column by column: each thread
        // owns whole columns, so rows need no barrier between them.
        for (int j = tid; j < DV; j += kThreads) {
            for (int r = 1; r < Lc; ++r) {
                float acc = Vs[r * DV + j];
                const float *ar = As + r * AP;
                for (int i = 0; i < r; ++i) acc = fmaf(-ar[i], Vs[i * DV + j], acc);
                Vs[r * DV + j] = acc;
            }
        }
        __syncthreads();

        // O = Qtil S0 + P U.
        for (int idx = tid; idx < Lc * DV; idx += kThreads) {
            const int t = idx / DV, j = idx % DV;
            float acc = 0.f;
            const float *qt = Qs + t * KP;
#pragma unroll 8
            for (int c = 0; c < DK; ++c) acc = fmaf(qt[c], S[c * DV + j], acc);
            const float *pt = Ps + t * AP;
            for (int i = 0; i <= t; ++i) acc = fmaf(pt[i], Vs[i * DV + j], acc);
            io<T>::store(o + ((size_t)(cs + t) * H + h) * DV + j, acc);
        }
        __syncthreads();

        // S <- Diag(exp(G_L)) S + Kbar^T U.
        for (int idx = tid; idx < DK * DV; idx += kThreads) {
            const int c = idx / DV, j = idx % DV;
            float acc = S[idx] * expf(GLs[c]);
            for (int t = 0; t < Lc; ++t) acc = fmaf(Gs[t * KP + c], Vs[t * DV + j], acc);
            S[idx] = acc;
        }
    }
    __syncthreads();
    if (final_state)
        for (int idx = tid; idx < DK * DV; idx += kThreads)
            final_state[state_off + idx] = S[idx];
}

template <typename T, int DK, int DV>
cudaError_t launch_typed(const void *q, const void *k, const void *v,
                         const void *g, const void *beta, const float *init,
                         const int32_t *cu, int n, int64_t T_tot, int H,
                         void *o, float *fin, uint32_t *err, bool sg, cudaStream_t st) {
    constexpr size_t smem = SimtSmem<DK, DV>::bytes;
    auto kern = kda_prefill_simt_kernel<T, DK, DV>;
    cudaError_t e = set_max_dynamic_smem((const void *)kern, (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned blocks = (unsigned)((size_t)n * (size_t)H);
    kern<<<blocks, kThreads, smem, st>>>(
        static_cast<const T *>(q), static_cast<const T *>(k),
        static_cast<const T *>(v), static_cast<const T *>(g),
        static_cast<const T *>(beta), init, cu, n, T_tot, H,
        static_cast<T *>(o), fin, err, sg ? 1 : 0);
    return cudaGetLastError();
}

template <typename T, int DK>
cudaError_t dispatch_dv(int dv, const void *q, const void *k, const void *v,
                        const void *g, const void *beta, const float *init,
                        const int32_t *cu, int n, int64_t T_tot, int H,
                        void *o, float *fin, uint32_t *err, bool sg, cudaStream_t st) {
    switch (dv) {
        case 16: return launch_typed<T, DK, 16>(q, k, v, g, beta, init, cu, n, T_tot, H, o, fin, err, sg, st);
        case 32: return launch_typed<T, DK, 32>(q, k, v, g, beta, init, cu, n, T_tot, H, o, fin, err, sg, st);
        case 64: return launch_typed<T, DK, 64>(q, k, v, g, beta, init, cu, n, T_tot, H, o, fin, err, sg, st);
        case 128: return launch_typed<T, DK, 128>(q, k, v, g, beta, init, cu, n, T_tot, H, o, fin, err, sg, st);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t dispatch_dk(int dk, int dv, const void *q, const void *k,
                        const void *v, const void *g, const void *beta,
                        const float *init, const int32_t *cu, int n,
                        int64_t T_tot, int H, void *o, float *fin,
                        uint32_t *err, bool sg, cudaStream_t st) {
    switch (dk) {
        case 16: return dispatch_dv<T, 16>(dv, q, k, v, g, beta, init, cu, n, T_tot, H, o, fin, err, sg, st);
        case 32: return dispatch_dv<T, 32>(dv, q, k, v, g, beta, init, cu, n, T_tot, H, o, fin, err, sg, st);
        case 64: return dispatch_dv<T, 64>(dv, q, k, v, g, beta, init, cu, n, T_tot, H, o, fin, err, sg, st);
        case 128: return dispatch_dv<T, 128>(dv, q, k, v, g, beta, init, cu, n, T_tot, H, o, fin, err, sg, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_prefill_simt(const void *q, const void *k, const void *v,
                                const void *g, const void *beta,
                                const float *init_state, const int32_t *cu,
                                int num_seqs, int64_t total_tokens, int H,
                                int dk, int dv, kda_dtype dtype, void *o,
                                float *final_state, uint32_t *err_word, bool scalar_gate,
                                cudaStream_t stream) {
    if (dtype == KDA_BF16)
        return dispatch_dk<__nv_bfloat16>(dk, dv, q, k, v, g, beta, init_state, cu, num_seqs,
                                          total_tokens, H, o, final_state, err_word, scalar_gate,
                                          stream);
    return dispatch_dk<float>(dk, dv, q, k, v, g, beta, init_state, cu, num_seqs,
                              total_tokens, H, o, final_state, err_word, scalar_gate, stream);
}

}  // namespace kda
