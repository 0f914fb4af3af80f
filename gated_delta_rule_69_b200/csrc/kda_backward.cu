// KDA backward pass (training): the reverse-mode derivative of the recurrence
//
//     Sp = Diag(exp(g_t)) S_{t-1},  r = Sp^T k_t,  u = beta_t (v_t - r),
//     S_t = Sp + k_t u^T,           o_t = S_t^T q_t
//
// (page "Kimi Linear" on docsaid.org, section "KDA : une decroissance propre
// a chaque canal", the KDA update; the news digest page on Kimi Linear,
// section "Algorithme parallele par chunks", organises the operator for
// training).  Step t read backwards, with dS = dL/dS_t:
//
//     dS += q do^T;         dq = S_t do
//     du  = dS^T k;         dk = dS u
//     dbeta = du . (v - r); dv = beta du;   dr = -beta du
//     dS += k dr^T;         dk += Sp dr          (dS is now dL/dSp)
//     dg[c] = sum_j Sp[c][j] dS[c][j];      dS = Diag(exp(g_t)) dS
//
// Layout.  Every column of the state follows its own recurrence (the step
// reads column j only through r_j and u_j), so a CTA owns a 32-column slice of
// one (sequence, head) and runs the whole sequence: 8 warps of 4 columns, a
// lane holding d_k/32 key rows of its warp's columns (16 fp32 of S and 16 of
// dS at d_k = 128, in registers).  Column sums over the key rows (r, du) are
// warp shuffles; row sums over the columns (dq, dk, dg, dbeta) are partials
// per warp, summed over the CTA's warps in shared memory every 4 steps and
// over the head's slices by fp32 atomic adds into the zeroed gradients.
//
// States entering the steps come from a forward pass that keeps the state
// entering every block of 64 steps in the workspace; each block is then run
// forward once more from its kept state, writing the 64 states entering its
// steps into the CTA's own scratch (L2-resident), and backward from its end.
// The same thread writes and reads every scratch element, so no barrier
// orders them.
#include "kda_internal.cuh"

namespace kda {

// kda_backward_tc.cu: the chunk-local gradients on the tensor cores
size_t backward_tc_scratch(int grid);
cudaError_t launch_backward_tc(const void *q, const void *k, const void *v, const void *g, const void *beta,
                               const void *d_o, int64_t total_tokens, int H, const int2 *chunk_tab,
                               const uint32_t *total_chunks, const uint8_t *s_in, const uint8_t *ds_next, float *dq,
                               float *dk, float *dv, float *dg, float *dbeta, uint32_t *slow, float *gscr,
                               uint32_t *err_word, int grid, bool scalar_gate, cudaStream_t stream);

namespace {

constexpr int kBwdWarps = 8;
constexpr int kBwdThreads = 32 * kBwdWarps;
constexpr int kBwdCols = 4;                        // d_v columns per warp
constexpr int kBwdSlice = kBwdWarps * kBwdCols;    // d_v columns per CTA
constexpr int kBwdBlock = 64;                      // steps between kept states
constexpr int kBwdGroup = 4;                       // steps per shared-memory reduction
constexpr int kBwdMaxCtas = 2 * 148;               // resident CTAs on a B200 (2 per SM)
constexpr int kBwdTcMaxCtas = 148;                 // tensor-core chunk kernel: one CTA per SM
// Sub-block of the chunk-parallel kernel's recompute: the whole 64-step block
// (16-step sub-blocks with kept states cut its scratch from 1 MB to 330 KB a CTA
// but their second forward pass made the call 20 % slower on a B200).
constexpr int kBwdChunkSub = kBwdBlock;

template <int DK>
struct BwdShape {
    static constexpr int RPL = DK / 32;                  // key rows per lane
    static constexpr int E = 3 * DK + 2;                 // a warp's partials of one step
    static constexpr int STATE4 = DK * kBwdSlice / 4;    // float4s in a state slice
    static constexpr size_t SMEM = 2ull * kBwdGroup * kBwdWarps * E * sizeof(float);
    static_assert(DK % 32 == 0, "d_k must be a multiple of 32");
};

struct BwdArgs {
    const void *q, *k, *v, *g, *beta, *d_o;
    const float *init_state, *d_final_state;
    const int32_t *cu_seqlens;
    float *dq, *dk, *dv, *dg, *dbeta, *d_init_state;
    float4 *ckpt, *scratch;
    uint32_t *err_word;
    int64_t seq_len;     // tokens per sequence when cu_seqlens is null
    int64_t total_tokens;
    int H, dv_total, nslices, units, scalar_gate;
};

__device__ __forceinline__ float4 f4(float x) { return make_float4(x, x, x, x); }

// Byte offset of element (row, col) in a 128-byte-swizzled K-atom of 64
// bf16 columns (the layout the backward scans write the states in).
__device__ __forceinline__ uint32_t sw128_tile_off(uint32_t row, uint32_t col) {
    return row * 128u + (((col >> 3) ^ (row & 7u)) << 4) + (col & 7u) * 2u;
}
__device__ __forceinline__ float4 sub4(float4 a, float4 b) {
    return make_float4(a.x - b.x, a.y - b.y, a.z - b.z, a.w - b.w);
}
__device__ __forceinline__ float4 mul4(float4 a, float s) {
    return make_float4(a.x * s, a.y * s, a.z * s, a.w * s);
}
// acc + a * s
__device__ __forceinline__ float4 fma4s(float4 a, float s, float4 acc) {
    return make_float4(fmaf(a.x, s, acc.x), fmaf(a.y, s, acc.y), fmaf(a.z, s, acc.z),
                       fmaf(a.w, s, acc.w));
}
__device__ __forceinline__ float dot4(float4 a, float4 b) {
    return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, a.w * b.w)));
}
__device__ __forceinline__ float4 warp_sum4(float4 x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        x.x += __shfl_xor_sync(0xffffffffu, x.x, off);
        x.y += __shfl_xor_sync(0xffffffffu, x.y, off);
        x.z += __shfl_xor_sync(0xffffffffu, x.z, off);
        x.w += __shfl_xor_sync(0xffffffffu, x.w, off);
    }
    return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

// One step's inputs as a lane needs them: its key rows of k, q and the decay,
// its warp's 4 columns of v and do, and beta.
template <int RPL>
struct StepIn {
    float k[RPL], q[RPL], a[RPL];
    float4 v, d;
    float b;
};

// The same inputs as loaded, unconverted: a load issued a step ahead is then
// first waited for in the step that uses it (converting at the load would
// wait for it there).
template <typename T> struct Raw4;
template <> struct Raw4<float> { using type = float4; };
template <> struct Raw4<__nv_bfloat16> { using type = uint2; };

template <typename T, int RPL>
struct StepRaw {
    T k[RPL], q[RPL], g[RPL];
    typename Raw4<T>::type v, d;
    T b;
};

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float4 to_f4(float4 x) { return x; }
__device__ __forceinline__ float4 to_f4(uint2 w) {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w.y));
    return make_float4(a.x, a.y, b.x, b.y);
}

template <typename T, int DK, bool BWD>
__device__ __forceinline__ void load_step(StepRaw<T, DK / 32> &s, const BwdArgs &p, int64_t t,
                                          int h, int lane, int j0) {
    constexpr int RPL = DK / 32;
    using R4 = typename Raw4<T>::type;
    const size_t row = (size_t)t * p.H + h;
    const T *kp = static_cast<const T *>(p.k) + row * DK + lane;
#pragma unroll
    for (int i = 0; i < RPL; ++i) s.k[i] = kp[32 * i];
    if (p.scalar_gate) {
        s.g[0] = static_cast<const T *>(p.g)[row];
    } else {
        const T *gp = static_cast<const T *>(p.g) + row * DK + lane;
#pragma unroll
        for (int i = 0; i < RPL; ++i) s.g[i] = gp[32 * i];
    }
    s.v = *reinterpret_cast<const R4 *>(static_cast<const T *>(p.v) + row * p.dv_total + j0);
    s.b = static_cast<const T *>(p.beta)[row];
    if (BWD) {
        const T *qp = static_cast<const T *>(p.q) + row * DK + lane;
#pragma unroll
        for (int i = 0; i < RPL; ++i) s.q[i] = qp[32 * i];
        s.d = *reinterpret_cast<const R4 *>(static_cast<const T *>(p.d_o) + row * p.dv_total + j0);
    }
}

template <typename T, int RPL, bool BWD>
__device__ __forceinline__ void decode_step(StepIn<RPL> &s, const StepRaw<T, RPL> &r,
                                            int scalar_gate) {
#pragma unroll
    for (int i = 0; i < RPL; ++i) s.k[i] = to_f(r.k[i]);
    if (scalar_gate) {
        const float a = __expf(to_f(r.g[0]));
#pragma unroll
        for (int i = 0; i < RPL; ++i) s.a[i] = a;
    } else {
#pragma unroll
        for (int i = 0; i < RPL; ++i) s.a[i] = __expf(to_f(r.g[i]));
    }
    s.v = to_f4(r.v);
    s.b = to_f(r.b);
    if (BWD) {
#pragma unroll
        for (int i = 0; i < RPL; ++i) s.q[i] = to_f(r.q[i]);
        s.d = to_f4(r.d);
    }
}

// S <- S_t from S_{t-1}; returns r = (Diag(a) S_{t-1})^T k.
template <int RPL>
__device__ __forceinline__ float4 forward_step(float4 (&S)[RPL], const StepIn<RPL> &in) {
    float4 rp = f4(0.f);
#pragma unroll
    for (int i = 0; i < RPL; ++i) {
        S[i] = mul4(S[i], in.a[i]);
        rp = fma4s(S[i], in.k[i], rp);
    }
    const float4 r = warp_sum4(rp);
    const float4 u = mul4(sub4(in.v, r), in.b);
#pragma unroll
    for (int i = 0; i < RPL; ++i) S[i] = fma4s(u, in.k[i], S[i]);
    return r;
}

// A step's record in a CTA's scratch: the state slice entering it, then r of
// each warp's 4 columns.
template <int DK>
constexpr int scratch_step4() { return BwdShape<DK>::STATE4 + kBwdWarps; }

// Forward over steps [t0, t1) with the next step's inputs loaded one step ahead;
// with `keep`, each step's record (entering state, r) is written to
// keep[step - t0].
template <typename T, int DK>
__device__ __forceinline__ void forward_run(float4 (&S)[DK / 32], const BwdArgs &p, int64_t t0,
                                            int64_t t1, int h, int lane, int j0, float4 *keep,
                                            int idx) {
    constexpr int RPL = DK / 32;
    constexpr int R4 = scratch_step4<DK>();
    StepRaw<T, RPL> nxt;
    if (t0 < t1) load_step<T, DK, false>(nxt, p, t0, h, lane, j0);
#pragma unroll 1
    for (int64_t t = t0; t < t1; ++t) {
        StepIn<RPL> cur;
        decode_step<T, RPL, false>(cur, nxt, p.scalar_gate);
        if (t + 1 < t1) load_step<T, DK, false>(nxt, p, t + 1, h, lane, j0);
        float4 *rec = keep ? keep + (size_t)(t - t0) * R4 : nullptr;
        if (rec) {
#pragma unroll
            for (int i = 0; i < RPL; ++i) rec[idx + i * kBwdThreads] = S[i];
        }
        const float4 r = forward_step<RPL>(S, cur);
        if (rec && lane == 0) rec[BwdShape<DK>::STATE4 + (idx >> 5)] = r;
    }
}

// Sums the group's per-warp partials over the warps and adds them to the
// gradients (count steps, the first of them at token t_hi, then t_hi - 1, ...).
template <int DK>
__device__ __forceinline__ void flush_group(const float *red, int count, int64_t t_hi, int h,
                                            const BwdArgs &p) {
    constexpr int E = BwdShape<DK>::E;
    for (int idx = threadIdx.x; idx < count * E; idx += kBwdThreads) {
        const int gi = idx / E, e = idx - gi * E;
        const float *src = red + (size_t)gi * kBwdWarps * E + e;
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < kBwdWarps; ++w) acc += src[w * E];
        const size_t row = (size_t)(t_hi - gi) * p.H + h;
        if (e < DK) {
            atomicAdd(p.dq + row * DK + e, acc);
        } else if (e < 2 * DK) {
            atomicAdd(p.dk + row * DK + (e - DK), acc);
        } else if (e < 3 * DK) {
            if (!p.scalar_gate) atomicAdd(p.dg + row * DK + (e - 2 * DK), acc);
        } else if (e == 3 * DK) {
            atomicAdd(p.dbeta + row, acc);
        } else if (p.scalar_gate) {
            atomicAdd(p.dg + row, acc);
        }
    }
}

// One range of steps [tb, te) backwards, from dS = dL/dS_te: the range run
// forward again from its entering state S (overwritten) into the scratch,
// then the backward steps; the row partials are flushed every kBwdGroup
// steps and at t == t_stop (the first step of the unit).
template <typename T, int DK>
__device__ __forceinline__ void range_backward(float4 (&S)[DK / 32], float4 (&dS)[DK / 32],
                                               const BwdArgs &p, int64_t tb, int64_t te,
                                               int64_t t_stop, int h, int warp, int lane, int j0,
                                               int idx, float4 *scratch, float *red, int &buf,
                                               int &gi, int64_t &g_hi) {
    using Sh = BwdShape<DK>;
    constexpr int RPL = Sh::RPL, E = Sh::E, S4 = Sh::STATE4;
    forward_run<T, DK>(S, p, tb, te, h, lane, j0, scratch, idx);

    // Lane 0 wrote each step's r; the warp's lanes read it below.
    __syncwarp();
    // Backward over the block, the next step's inputs and record
    // loaded one step ahead.
    constexpr int R4 = scratch_step4<DK>();
    StepRaw<T, RPL> nxt;
    float4 Sn[RPL], rn;
    load_step<T, DK, true>(nxt, p, te - 1, h, lane, j0);
    {
        const float4 *rec = scratch + (size_t)(te - 1 - tb) * R4;
#pragma unroll
        for (int i = 0; i < RPL; ++i) Sn[i] = rec[idx + i * kBwdThreads];
        rn = rec[S4 + warp];
    }
#pragma unroll 1
    for (int64_t t = te - 1; t >= tb; --t) {
        StepIn<RPL> cur;
        decode_step<T, RPL, true>(cur, nxt, p.scalar_gate);
        float4 sp[RPL];
#pragma unroll
        for (int i = 0; i < RPL; ++i) sp[i] = Sn[i];
        const float4 r = rn;
        if (t - 1 >= tb) {
            load_step<T, DK, true>(nxt, p, t - 1, h, lane, j0);
            const float4 *rec = scratch + (size_t)(t - 1 - tb) * R4;
#pragma unroll
            for (int i = 0; i < RPL; ++i) Sn[i] = rec[idx + i * kBwdThreads];
            rn = rec[S4 + warp];
        }
        // Sp = Diag(a) S_{t-1}; r and u as the forward had them
#pragma unroll
        for (int i = 0; i < RPL; ++i) sp[i] = mul4(sp[i], cur.a[i]);
        const float4 vr = sub4(cur.v, r);
        const float4 uu = mul4(vr, cur.b);
        // o_t = S_t^T q, S_t = Sp + k u^T
        float dq_r[RPL], dk_r[RPL], dg_r[RPL];
        float4 dup = f4(0.f);
#pragma unroll
        for (int i = 0; i < RPL; ++i) {
            dS[i] = fma4s(cur.d, cur.q[i], dS[i]);
            dq_r[i] = dot4(fma4s(uu, cur.k[i], sp[i]), cur.d);
            dup = fma4s(dS[i], cur.k[i], dup);
            dk_r[i] = dot4(dS[i], uu);
        }
        const float4 du = warp_sum4(dup);
        const float dbeta = dot4(du, vr);
        const size_t row = (size_t)t * p.H + h;
        if (lane == 0)
            *reinterpret_cast<float4 *>(p.dv + row * p.dv_total + j0) = mul4(du, cur.b);
        const float4 dr = mul4(du, -cur.b);
        float gsum = 0.f;
#pragma unroll
        for (int i = 0; i < RPL; ++i) {
            dS[i] = fma4s(dr, cur.k[i], dS[i]);
            dk_r[i] += dot4(sp[i], dr);
            dg_r[i] = dot4(sp[i], dS[i]);
            gsum += dg_r[i];
            dS[i] = mul4(dS[i], cur.a[i]);
        }
        // this warp's row partials of the step
        float *slot = red + ((size_t)(buf * kBwdGroup + gi) * kBwdWarps + warp) * E;
#pragma unroll
        for (int i = 0; i < RPL; ++i) {
            slot[lane + 32 * i] = dq_r[i];
            slot[DK + lane + 32 * i] = dk_r[i];
            slot[2 * DK + lane + 32 * i] = dg_r[i];
        }
        if (p.scalar_gate) gsum = warp_sum(gsum);
        if (lane == 0) {
            slot[3 * DK] = dbeta;
            slot[3 * DK + 1] = gsum;
        }
        if (gi == 0) g_hi = t;
        ++gi;
        if (gi == kBwdGroup || t == t_stop) {
            // One barrier per group: the two buffers alternate, and a
            // buffer is written again only after the next group's
            // barrier, which every thread reaches after this flush.
            __syncthreads();
            flush_group<DK>(red + (size_t)buf * kBwdGroup * kBwdWarps * E, gi, g_hi, h, p);
            buf ^= 1;
            gi = 0;
        }
    }
}

// One block of steps [tb, te) backwards (te - tb <= kBwdBlock).  SUB =
// kBwdBlock: the whole block is run forward into the scratch (kBwdBlock step
// records), then backwards.  SUB < kBwdBlock: a first forward pass keeps only
// the state entering each SUB-step sub-block (after the SUB step records in
// the scratch), then each sub-block from the last is run forward again from
// its kept state and backwards: SUB + kBwdBlock / SUB state records instead
// of kBwdBlock, for one more forward pass.  The chunk-parallel kernel keeps
// many units in flight at once, and the smaller scratch stays in L2.
template <int SUB>
constexpr int scratch_records() { return SUB >= kBwdBlock ? kBwdBlock : SUB + kBwdBlock / SUB; }

template <typename T, int DK, int SUB>
__device__ __forceinline__ void block_backward(float4 (&S)[DK / 32], float4 (&dS)[DK / 32],
                                               const BwdArgs &p, int64_t tb, int64_t te,
                                               int64_t t_stop, int h, int warp, int lane, int j0,
                                               int idx, float4 *scratch, float *red, int &buf,
                                               int &gi, int64_t &g_hi) {
    if (SUB >= kBwdBlock) {
        range_backward<T, DK>(S, dS, p, tb, te, t_stop, h, warp, lane, j0, idx, scratch, red, buf,
                              gi, g_hi);
        return;
    }
    constexpr int RPL = DK / 32;
    constexpr int R4 = scratch_step4<DK>();
    float4 *kept = scratch + (size_t)SUB * R4;   // the state entering sub-block s at kept + s R4
#pragma unroll 1
    for (int64_t sb = tb; sb < te; sb += SUB) {
        float4 *ks = kept + (size_t)((sb - tb) / SUB) * R4;
#pragma unroll
        for (int i = 0; i < RPL; ++i) ks[idx + i * kBwdThreads] = S[i];
        forward_run<T, DK>(S, p, sb, sb + SUB < te ? sb + SUB : te, h, lane, j0, nullptr, idx);
    }
#pragma unroll 1
    for (int64_t sb = tb + ((te - tb - 1) / SUB) * SUB; sb >= tb; sb -= SUB) {
        const float4 *ks = kept + (size_t)((sb - tb) / SUB) * R4;
#pragma unroll
        for (int i = 0; i < RPL; ++i) S[i] = ks[idx + i * kBwdThreads];
        range_backward<T, DK>(S, dS, p, sb, sb + SUB < te ? sb + SUB : te, t_stop, h, warp, lane, j0,
                              idx, scratch, red, buf, gi, g_hi);
    }
}

template <typename T, int DK>
__global__ void __launch_bounds__(kBwdThreads, 2) kda_backward_kernel(const BwdArgs p) {
    using Sh = BwdShape<DK>;
    constexpr int RPL = Sh::RPL, S4 = Sh::STATE4;
    extern __shared__ float red[];   // [2][kBwdGroup][kBwdWarps][E]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // a thread's float4 i of a state slice: key row lane + 32 i, its warp's columns
    const int idx = warp * 32 + lane;
    float4 *scratch = p.scratch + (size_t)blockIdx.x * kBwdBlock * scratch_step4<DK>();
    int buf = 0;

#pragma unroll 1
    for (int u = blockIdx.x; u < p.units; u += gridDim.x) {
        const int s = u % p.nslices;
        const int h = (u / p.nslices) % p.H;
        const int n = u / (p.nslices * p.H);
        int64_t bos, eos;
        if (p.cu_seqlens) {
            bos = p.cu_seqlens[n];
            eos = p.cu_seqlens[n + 1];
            if (bos < 0 || eos < bos || eos > p.total_tokens) {   // uniform over the CTA
                if (threadIdx.x == 0) atomicOr(p.err_word, kDevErrCuSeqlens);
                continue;
            }
        } else {
            bos = (int64_t)n * p.seq_len;
            eos = bos + p.seq_len;
        }
        const int j0 = s * kBwdSlice + warp * kBwdCols;
        const int64_t nb = (eos - bos + kBwdBlock - 1) / kBwdBlock;
        // Kept states: sequence n's blocks start at slot bos / 64 + n, which
        // leaves the slot ranges of consecutive sequences disjoint.
        const int64_t slot0 = bos / kBwdBlock + n;
        const size_t st = ((size_t)n * p.H + h) * DK * p.dv_total + j0;   // [N, H, d_k, d_v]

        float4 S[RPL];
#pragma unroll
        for (int i = 0; i < RPL; ++i)
            S[i] = p.init_state ? *reinterpret_cast<const float4 *>(
                                      p.init_state + st + (size_t)(lane + 32 * i) * p.dv_total)
                                : f4(0.f);
        // Forward: keep the state entering every block.
#pragma unroll 1
        for (int64_t b = 0; b < nb; ++b) {
            float4 *ck = p.ckpt + (((size_t)(slot0 + b) * p.H + h) * p.nslices + s) * S4;
#pragma unroll
            for (int i = 0; i < RPL; ++i) ck[idx + i * kBwdThreads] = S[i];
            if (b == nb - 1) break;
            const int64_t t0 = bos + b * kBwdBlock;
            forward_run<T, DK>(S, p, t0, t0 + kBwdBlock, h, lane, j0, nullptr, idx);
        }

        float4 dS[RPL];
#pragma unroll
        for (int i = 0; i < RPL; ++i)
            dS[i] = p.d_final_state ? *reinterpret_cast<const float4 *>(
                                          p.d_final_state + st + (size_t)(lane + 32 * i) * p.dv_total)
                                    : f4(0.f);
        int gi = 0;
        int64_t g_hi = 0;
#pragma unroll 1
        for (int64_t b = nb - 1; b >= 0; --b) {
            const int64_t tb = bos + b * kBwdBlock;
            const int64_t te = (tb + kBwdBlock < eos) ? tb + kBwdBlock : eos;
            const float4 *ck = p.ckpt + (((size_t)(slot0 + b) * p.H + h) * p.nslices + s) * S4;
#pragma unroll
            for (int i = 0; i < RPL; ++i) S[i] = ck[idx + i * kBwdThreads];
            block_backward<T, DK, kBwdBlock>(S, dS, p, tb, te, bos, h, warp, lane, j0, idx, scratch, red,
                                             buf, gi, g_hi);
        }
        if (p.d_init_state) {
#pragma unroll
            for (int i = 0; i < RPL; ++i)
                *reinterpret_cast<float4 *>(p.d_init_state + st + (size_t)(lane + 32 * i) * p.dv_total) = dS[i];
        }
    }
}

template <typename T, int DK>
cudaError_t launch_dk(const BwdArgs &p, int grid, cudaStream_t stream) {
    const size_t smem = BwdShape<DK>::SMEM;
    cudaError_t e = set_max_dynamic_smem((const void *)kda_backward_kernel<T, DK>, (int)smem);
    if (e != cudaSuccess) return e;
    kda_backward_kernel<T, DK><<<grid, kBwdThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

// ---- chunk-parallel variant (bf16, d = 128): the chunk records of the
// prefill's preparation give every chunk's entering state (a forward scan,
// S <- Diag(e^{G_L}) S + MP S + YT V) and every chunk's dL/dS_next (a
// reverse scan, dS <- Diag(e^{G_L}) dS + MP^T dS + QP^T dO: the transpose of
// the forward transition), both run as the prefill's transposed state chain
// on the tensor cores; the chunks' steps then run independently.

struct ChunkArgs {
    SplitTables tab;
    const uint8_t *s_in;     // entering states, bf16 tiles (launch_backward_scans)
    const uint8_t *ds_next;  // dL/dS at each chunk's end, bf16 tiles
    const uint32_t *only;  // [max_chunks * H] or null: run only the (chunk, head) items flagged 1
    int num_seqs;
};

// One unit per (chunk, head, slice): the block_backward of the chunk from its
// entering state and dL/dS_next; a sequence's first chunk writes dL/dS_0.
template <typename T, int DK>
__global__ void __launch_bounds__(kBwdThreads, 2) kda_backward_chunk_kernel(const BwdArgs p,
                                                                          const ChunkArgs c) {
    using Sh = BwdShape<DK>;
    constexpr int RPL = Sh::RPL;
    extern __shared__ float red[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int idx = warp * 32 + lane;
    float4 *scratch = p.scratch + (size_t)blockIdx.x * scratch_records<kBwdChunkSub>() * scratch_step4<DK>();
    int buf = 0, gi = 0;
    int64_t g_hi = 0;
    const int units = (int)*c.tab.total_chunks * p.H * p.nslices;
#pragma unroll 1
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
        const int s = u % p.nslices;
        const int h = (u / p.nslices) % p.H;
        const int ch = u / (p.nslices * p.H);
        if (c.only && !c.only[(size_t)ch * p.H + h]) continue;
        const int2 ct = c.tab.chunk_tab[ch];
        const int64_t tb = ct.x, te = (int64_t)ct.x + ct.y;
        const int j0 = s * kBwdSlice + warp * kBwdCols;
        // the 4 columns j0 .. j0 + 3 of row c share one 16-byte piece of the tile
        const size_t tile = ((size_t)ch * p.H + h) * 32768 + (size_t)(j0 >> 6) * 16384;
        float4 S[RPL], dS[RPL];
#pragma unroll
        for (int i = 0; i < RPL; ++i) {
            const uint32_t off = sw128_tile_off(lane + 32 * i, j0 & 63);
            S[i] = to_f4(*reinterpret_cast<const uint2 *>(c.s_in + tile + off));
            dS[i] = to_f4(*reinterpret_cast<const uint2 *>(c.ds_next + tile + off));
        }
        block_backward<T, DK, kBwdChunkSub>(S, dS, p, tb, te, tb, h, warp, lane, j0, idx, scratch, red,
                                            buf, gi, g_hi);
        if (p.d_init_state) {
            int lo = 0, hi = c.num_seqs;   // the last sequence whose first chunk is <= ch
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (c.tab.chunk_off[mid] <= ch) lo = mid;
                else hi = mid;
            }
            if (c.tab.chunk_off[lo] == ch) {
                const size_t st = ((size_t)lo * p.H + h) * DK * p.dv_total + j0;
#pragma unroll
                for (int i = 0; i < RPL; ++i)
                    *reinterpret_cast<float4 *>(p.d_init_state + st + (size_t)(lane + 32 * i) * p.dv_total) = dS[i];
            }
        }
    }
}

size_t bwd_slots(int num_seqs, int64_t total_tokens) {
    return (size_t)(total_tokens / kBwdBlock) + (size_t)num_seqs + 1;
}

int bwd_grid(int num_seqs, int H, int d_v) {
    const int64_t units = (int64_t)num_seqs * H * (d_v / kBwdSlice);
    return (int)(units < kBwdMaxCtas ? units : kBwdMaxCtas);
}

}  // namespace

size_t backward_workspace(int num_seqs, int64_t total_tokens, int H, int dk, int dv) {
    const size_t state = (size_t)dk * kBwdSlice * sizeof(float);   // one slice
    const size_t record = state + kBwdWarps * sizeof(float4);       // state and r per step
    const size_t nsl = (size_t)(dv / kBwdSlice);
    return kWorkspaceHeader + bwd_slots(num_seqs, total_tokens) * H * nsl * state +
           (size_t)bwd_grid(num_seqs, H, dv) * kBwdBlock * record;
}

cudaError_t launch_backward(const void *q, const void *k, const void *v, const void *g,
                            const void *beta, const float *init_state, const int32_t *cu,
                            int num_seqs, int64_t total_tokens, int H, int dk, int dv,
                            kda_dtype dtype, const void *d_o, const float *d_final_state,
                            float *dq, float *dk_out, float *dv_out, float *dg, float *dbeta,
                            float *d_init_state, void *workspace, bool scalar_gate,
                            cudaStream_t stream) {
    const size_t ng = (size_t)total_tokens * H * (scalar_gate ? 1 : dk);
    const size_t nk = (size_t)total_tokens * H * dk;
    uint32_t *err_word = static_cast<uint32_t *>(workspace);
    cudaError_t e;
    if ((e = cudaMemsetAsync(err_word, 0, sizeof(uint32_t), stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dq, 0, nk * sizeof(float), stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dk_out, 0, nk * sizeof(float), stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dg, 0, ng * sizeof(float), stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dbeta, 0, (size_t)total_tokens * H * sizeof(float), stream)) != cudaSuccess)
        return e;

    BwdArgs p;
    p.q = q; p.k = k; p.v = v; p.g = g; p.beta = beta; p.d_o = d_o;
    p.init_state = init_state;
    p.d_final_state = d_final_state;
    p.cu_seqlens = cu;
    p.dq = dq; p.dk = dk_out; p.dv = dv_out; p.dg = dg; p.dbeta = dbeta;
    p.d_init_state = d_init_state;
    p.err_word = err_word;
    p.seq_len = cu ? 0 : total_tokens / num_seqs;
    p.total_tokens = total_tokens;
    p.H = H;
    p.dv_total = dv;
    p.nslices = dv / kBwdSlice;
    p.units = num_seqs * H * p.nslices;
    p.scalar_gate = scalar_gate ? 1 : 0;
    const size_t state = (size_t)dk * kBwdSlice * sizeof(float);
    uint8_t *base = static_cast<uint8_t *>(workspace) + kWorkspaceHeader;
    p.ckpt = reinterpret_cast<float4 *>(base);
    p.scratch = reinterpret_cast<float4 *>(base + bwd_slots(num_seqs, total_tokens) * H * p.nslices * state);
    const int grid = bwd_grid(num_seqs, H, dv);
    if (grid == 0) return cudaGetLastError();
    const bool bf = dtype == KDA_BF16;
    switch (dk) {
        case 32: return bf ? launch_dk<__nv_bfloat16, 32>(p, grid, stream) : launch_dk<float, 32>(p, grid, stream);
        case 64: return bf ? launch_dk<__nv_bfloat16, 64>(p, grid, stream) : launch_dk<float, 64>(p, grid, stream);
        case 128: return bf ? launch_dk<__nv_bfloat16, 128>(p, grid, stream) : launch_dk<float, 128>(p, grid, stream);
        default: return cudaErrorInvalidValue;
    }
}

namespace {

struct ChunkedLayout {
    size_t split, s_in, ds_next, scratch, slow, gscr, total;
    size_t max_chunks;
    int grid, grid_tc;
};

ChunkedLayout chunked_layout(int num_seqs, int64_t total_tokens, int H) {
    ChunkedLayout l;
    l.max_chunks = (size_t)(total_tokens / kBwdBlock) + (size_t)num_seqs;
    const size_t state = (size_t)128 * 128 * sizeof(__nv_bfloat16);   // a bf16 tile per record
    const int64_t units = (int64_t)l.max_chunks * H * (128 / kBwdSlice);
    l.grid = (int)(units < kBwdMaxCtas ? units : kBwdMaxCtas);
    l.split = 0;
    l.s_in = (prefill_split_workspace(num_seqs, total_tokens, H) + 1023) & ~(size_t)1023;
    l.ds_next = l.s_in + l.max_chunks * H * state;
    l.scratch = l.ds_next + l.max_chunks * H * state;
    l.slow = l.scratch + (size_t)l.grid * scratch_records<kBwdChunkSub>() * scratch_step4<128>() * sizeof(float4);
    l.gscr = (l.slow + l.max_chunks * H * sizeof(uint32_t) + 255) & ~(size_t)255;
    const size_t items = l.max_chunks * (size_t)H;
    l.grid_tc = (int)(items < (size_t)kBwdTcMaxCtas ? items : (size_t)kBwdTcMaxCtas);
    l.total = l.gscr + backward_tc_scratch(l.grid_tc);
    return l;
}

}  // namespace

size_t backward_chunked_workspace(int num_seqs, int64_t total_tokens, int H) {
    return chunked_layout(num_seqs, total_tokens, H).total;
}

cudaError_t launch_backward_chunked(const void *q, const void *k, const void *v, const void *g,
                                    const void *beta, const float *init_state, const int32_t *cu,
                                    int num_seqs, int64_t total_tokens, int H, const void *d_o,
                                    const float *d_final_state, float *dq, float *dk_out,
                                    float *dv_out, float *dg, float *dbeta, float *d_init_state,
                                    void *workspace, bool scalar_gate, cudaStream_t stream) {
    const ChunkedLayout l = chunked_layout(num_seqs, total_tokens, H);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const size_t nk = (size_t)total_tokens * H * 128;
    const size_t ng = scalar_gate ? (size_t)total_tokens * H : nk;
    // no zeroing: the tensor-core kernel writes every row of its items and
    // zeroes those of the items it leaves, into which the step kernel adds
    (void)nk;
    (void)ng;
    cudaError_t e;
    // 1. the plan and the chunk records (the prefill's preparation, no chain)
    e = launch_prefill_split(q, k, v, g, beta, nullptr, cu, num_seqs, total_tokens, H, nullptr,
                             nullptr, ws + l.split, scalar_gate, nullptr, stream, kPrepOnly);
    if (e != cudaSuccess) return e;
    const SplitTables tab = split_tables(ws + l.split, num_seqs, total_tokens, H);
    // 2. the scans over the records on the tensor cores (the transposed state
    // chain, forward and reverse): every chunk's entering state and dL/dS at
    // its end, and a first dL/dS_0 per sequence
    e = launch_backward_scans(v, d_o, init_state, d_final_state, cu, num_seqs, total_tokens, H,
                              ws + l.split, ws + l.s_in, ws + l.ds_next, d_init_state, stream);
    if (e != cudaSuccess) return e;
    // 3. the chunk-local gradients: on the tensor cores for every chunk that
    // decays within e^80, then the token-by-token kernel for the rest
    uint32_t *slow = reinterpret_cast<uint32_t *>(ws + l.slow);
    if ((e = cudaMemsetAsync(slow, 0, l.max_chunks * H * sizeof(uint32_t), stream)) != cudaSuccess) return e;
    e = launch_backward_tc(q, k, v, g, beta, d_o, total_tokens, H, tab.chunk_tab, tab.total_chunks,
                           ws + l.s_in, ws + l.ds_next, dq, dk_out, dv_out, dg, dbeta,
                           slow, reinterpret_cast<float *>(ws + l.gscr), reinterpret_cast<uint32_t *>(ws),
                           l.grid_tc, scalar_gate, stream);
    if (e != cudaSuccess) return e;
    BwdArgs p = {};
    p.q = q; p.k = k; p.v = v; p.g = g; p.beta = beta; p.d_o = d_o;
    p.dq = dq; p.dk = dk_out; p.dv = dv_out; p.dg = dg; p.dbeta = dbeta;
    p.d_init_state = d_init_state;
    p.scratch = reinterpret_cast<float4 *>(ws + l.scratch);
    p.err_word = reinterpret_cast<uint32_t *>(ws);
    p.total_tokens = total_tokens;
    p.H = H;
    p.dv_total = 128;
    p.nslices = 128 / kBwdSlice;
    p.scalar_gate = scalar_gate ? 1 : 0;
    ChunkArgs ca;
    ca.tab = tab;
    ca.s_in = ws + l.s_in;
    ca.ds_next = ws + l.ds_next;
    ca.only = slow;
    ca.num_seqs = num_seqs;
    const size_t smem = BwdShape<128>::SMEM;
    if ((e = set_max_dynamic_smem((const void *)kda_backward_chunk_kernel<__nv_bfloat16, 128>, (int)smem)) !=
        cudaSuccess)
        return e;
    kda_backward_chunk_kernel<__nv_bfloat16, 128><<<l.grid, kBwdThreads, smem, stream>>>(p, ca);
    return cudaGetLastError();
}

}  // namespace kda
