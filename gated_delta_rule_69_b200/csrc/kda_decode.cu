// KDA decode step: one token per sequence, the fp32 state updated in place.
//
// Per (b, h), with D = Diag(exp(log_alpha)):
//     S <- D S;   u = beta (v - S^T k);   S <- S + k u^T;   o = S^T q
// which is the KDA update (page "Kimi Linear" on docsaid.org, section "KDA :
// une decroissance propre a chaque canal") applied to a single token, read
// out with the updated state.  The read-out is expanded as
//     o = (D S)^T q + u (k . q)
// so the state is read once and written once: the step is bound by HBM
// bandwidth (one fp32 d_k x d_v read + write per head).
//
// Layout: one CTA per (b, h).  A warp spans d_v with one float4 per lane, so
// every warp-wide load or store touches whole 512-byte rows; the CTA's row
// groups split d_k.  The whole d_k x d_v tile stays in registers between the
// read and the write (64 fp32 per thread at d = 128).  State traffic uses
// streaming cache hints: each element is touched once per step and the
// state of a large batch does not fit in L2.
#include "kda_internal.cuh"

namespace kda {
namespace {

template <int DK, int DV>
struct DecodeShape {
    static constexpr int LX = DV / 4;                        // lanes along d_v
    static constexpr int NT = (LX * DK < 256) ? LX * DK : 256;  // threads
    static constexpr int R = NT / LX;                        // row groups
    static constexpr int RPT = DK / R;                       // rows per thread
    static_assert(DV % 4 == 0 && NT % LX == 0 && DK % R == 0, "bad shape");
};

__device__ __forceinline__ float4 fma4(float4 a, float s, float4 acc) {
    acc.x = fmaf(a.x, s, acc.x);
    acc.y = fmaf(a.y, s, acc.y);
    acc.z = fmaf(a.z, s, acc.z);
    acc.w = fmaf(a.w, s, acc.w);
    return acc;
}

// LAYER: the layer prologue / epilogue (kda_layer_decode_step); a separate
// instantiation keeps the plain step as lean as before.
template <typename T, int DK, int DV, bool LAYER>
__global__ void __launch_bounds__(DecodeShape<DK, DV>::NT)
kda_decode_kernel(const T *__restrict__ q, const T *__restrict__ k,
                  const T *__restrict__ v, const T *__restrict__ g,
                  const T *__restrict__ beta, float *__restrict__ state,
                  T *__restrict__ o, int g_bh, int g_c, int H, const LayerArgs la) {
    using Sh = DecodeShape<DK, DV>;
    constexpr int LX = Sh::LX, NT = Sh::NT, R = Sh::R, RPT = Sh::RPT;
    __shared__ float sk[DK], sq[DK], sa[DK], sv[DV], su[DV];
    __shared__ __align__(16) float red_k[R][DV];
    __shared__ __align__(16) float red_q[R][DV];
    __shared__ float s_kq, s_nk, s_nq, s_no;
    __shared__ float so[LAYER ? DV : 1];
    constexpr bool layer = LAYER;

    const int tid = threadIdx.x;
    const int lx = tid % LX;
    const int ry = tid / LX;
    const size_t bh = blockIdx.x;
    float4 *Sp = reinterpret_cast<float4 *>(state + bh * (size_t)(DK * DV));

    // Issue every state load first: RPT independent 16-byte loads per thread.
    float4 s[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) s[i] = __ldcs(Sp + (ry + i * R) * LX + lx);

    for (int i = tid; i < DK; i += NT) {
        sk[i] = io<T>::load(k + bh * DK + i);
        sq[i] = io<T>::load(q + bh * DK + i);
        if (layer) {
            const float z = io<T>::load(static_cast<const T *>(la.gate_z) + bh * DK + i);
            sa[i] = expf(-expf(la.A_log[bh % (size_t)H]) * softplus_f(z));
        } else {
            sa[i] = expf(io<T>::load(g + bh * g_bh + i * g_c));
        }
    }
    for (int i = tid; i < DV; i += NT) sv[i] = io<T>::load(v + bh * DV + i);
    __syncthreads();
    if (layer) {   // L2-normalise q and k
        if (tid < 32) {
            float ak = 0.f, aq = 0.f;
            for (int c = tid; c < DK; c += 32) {
                ak = fmaf(sk[c], sk[c], ak);
                aq = fmaf(sq[c], sq[c], aq);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                ak += __shfl_xor_sync(0xffffffffu, ak, off);
                aq += __shfl_xor_sync(0xffffffffu, aq, off);
            }
            if (tid == 0) {
                s_nk = rsqrtf(ak + la.qk_eps);
                s_nq = rsqrtf(aq + la.qk_eps);
            }
        }
        __syncthreads();
        for (int i = tid; i < DK; i += NT) {
            sk[i] *= s_nk;
            sq[i] *= s_nq;
        }
        __syncthreads();
    }

    if (tid < 32) {  // k . q by one warp
        float acc = 0.f;
        for (int c = tid; c < DK; c += 32) acc = fmaf(sk[c], sq[c], acc);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (tid == 0) s_kq = acc;
    }

    // D S, and the partial column sums of (D S)^T k and (D S)^T q.
    float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pq = pk;
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int c = ry + i * R;
        const float a = sa[c];
        s[i].x *= a; s[i].y *= a; s[i].z *= a; s[i].w *= a;
        pk = fma4(s[i], sk[c], pk);
        pq = fma4(s[i], sq[c], pq);
    }
    reinterpret_cast<float4 *>(red_k[ry])[lx] = pk;
    reinterpret_cast<float4 *>(red_q[ry])[lx] = pq;
    __syncthreads();

    if (tid < DV) {
        float rk = 0.f, rq = 0.f;
#pragma unroll
        for (int y = 0; y < R; ++y) {
            rk += red_k[y][tid];
            rq += red_q[y][tid];
        }
        const float b = layer ? sigmoid_f(io<T>::load(static_cast<const T *>(la.beta_logit) + bh))
                              : io<T>::load(beta + bh);
        const float u = b * (sv[tid] - rk);
        su[tid] = u;
        const float ov = fmaf(u, s_kq, rq);
        if (layer) so[tid] = ov;
        else io<T>::store(o + bh * DV + tid, ov);
    }
    __syncthreads();
    if (layer) {   // RMSNorm over d_v, weight, sigmoid output gate
        if (tid < 32) {
            float a = 0.f;
            for (int j = tid; j < DV; j += 32) a = fmaf(so[j], so[j], a);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
            if (tid == 0) s_no = rsqrtf(a / (float)DV + la.norm_eps);
        }
        __syncthreads();
        if (tid < DV) {
            float y = so[tid] * s_no;
            if (la.norm_weight) y *= la.norm_weight[tid];
            if (la.out_gate)
                y *= sigmoid_f(io<T>::load(static_cast<const T *>(la.out_gate) + bh * DV + tid));
            io<T>::store(o + bh * DV + tid, y);
        }
    }

    const float4 u4 = reinterpret_cast<const float4 *>(su)[lx];
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int c = ry + i * R;
        s[i] = fma4(u4, sk[c], s[i]);
        __stcs(Sp + c * LX + lx, s[i]);
    }
}

template <typename T, int DK, int DV>
cudaError_t launch_typed(const void *q, const void *k, const void *v,
                         const void *g, const void *beta, float *state,
                         int batch, int H, void *o, bool sg, const LayerArgs *layer,
                         cudaStream_t stream) {
    const unsigned blocks = (unsigned)((size_t)batch * (size_t)H);
    LayerArgs la = {};
    if (layer) {
        la = *layer;
        kda_decode_kernel<T, DK, DV, true><<<blocks, DecodeShape<DK, DV>::NT, 0, stream>>>(
            static_cast<const T *>(q), static_cast<const T *>(k),
            static_cast<const T *>(v), static_cast<const T *>(g),
            static_cast<const T *>(beta), state, static_cast<T *>(o), sg ? 1 : DK, sg ? 0 : 1, H, la);
    } else {
        kda_decode_kernel<T, DK, DV, false><<<blocks, DecodeShape<DK, DV>::NT, 0, stream>>>(
            static_cast<const T *>(q), static_cast<const T *>(k),
            static_cast<const T *>(v), static_cast<const T *>(g),
            static_cast<const T *>(beta), state, static_cast<T *>(o), sg ? 1 : DK, sg ? 0 : 1, H, la);
    }
    return cudaGetLastError();
}

template <typename T, int DK>
cudaError_t dispatch_dv(int dv, const void *q, const void *k, const void *v,
                        const void *g, const void *beta, float *state,
                        int batch, int H, void *o, bool sg, const LayerArgs *la,
                        cudaStream_t stream) {
    switch (dv) {
        case 16: return launch_typed<T, DK, 16>(q, k, v, g, beta, state, batch, H, o, sg, la, stream);
        case 32: return launch_typed<T, DK, 32>(q, k, v, g, beta, state, batch, H, o, sg, la, stream);
        case 64: return launch_typed<T, DK, 64>(q, k, v, g, beta, state, batch, H, o, sg, la, stream);
        case 128: return launch_typed<T, DK, 128>(q, k, v, g, beta, state, batch, H, o, sg, la, stream);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t dispatch_dk(int dk, int dv, const void *q, const void *k,
                        const void *v, const void *g, const void *beta,
                        float *state, int batch, int H, void *o, bool sg,
                        const LayerArgs *la, cudaStream_t stream) {
    switch (dk) {
        case 16: return dispatch_dv<T, 16>(dv, q, k, v, g, beta, state, batch, H, o, sg, la, stream);
        case 32: return dispatch_dv<T, 32>(dv, q, k, v, g, beta, state, batch, H, o, sg, la, stream);
        case 64: return dispatch_dv<T, 64>(dv, q, k, v, g, beta, state, batch, H, o, sg, la, stream);
        case 128: return dispatch_dv<T, 128>(dv, q, k, v, g, beta, state, batch, H, o, sg, la, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_decode(const void *q, const void *k, const void *v,
                          const void *g, const void *beta, float *state,
                          int batch, int H, int dk, int dv, kda_dtype dtype,
                          void *o, bool scalar_gate, const LayerArgs *layer,
                          cudaStream_t stream) {
    if (dtype == KDA_BF16)
        return dispatch_dk<__nv_bfloat16>(dk, dv, q, k, v, g, beta, state, batch, H, o, scalar_gate,
                                          layer, stream);
    return dispatch_dk<float>(dk, dv, q, k, v, g, beta, state, batch, H, o, scalar_gate, layer,
                              stream);
}

}  // namespace kda
