// KDA chunkwise prefill on the sm_100a tensor cores (bf16 I/O, d_k = d_v =
// 128, chunk C = 64, fp32 state).
//
// Chunk algebra (news digest page on Kimi Linear, section "Algorithme
// parallele par chunks"; course page "Attention lineaire et recurrence",
// section "Le calcul par blocs").  Inside a chunk, with G_t the running sum of
// log_alpha (per key channel, from the chunk start) and S the state entering
// the chunk (d_k x d_v):
//     Ktil = K e^{G}, Qtil = Q e^{G}, Khat = K e^{-G}, Kbar = K e^{G_L - G}
//     A = diag(beta) strict_tril(Ktil Khat^T)    P = tril(Qtil Khat^T)
//     T = (I + A)^{-1}        (blocked forward substitution, fp32)
//     W = T diag(beta) Ktil   U' = T diag(beta) V        (the WY / UT form)
//     U = U' - W S            O = Qtil S + P U
//     S_next = Diag(e^{G_L}) S + Kbar^T U
// KDA ties both low-rank factors of its diagonal-plus-low-rank transition
// to k, so only two intra-chunk products (A and P, stacked into one M = 128
// product) are needed (news digest page, section "Un volume de calcul reduit
// par rapport au DPLR general").
//
// Numerics: every exponent is <= 0 except in Khat, whose exponent -G is at
// most the chunk's total log-decay.  When some channel decays by more than
// e^{-60} inside one chunk (the cumulative-decay trap of the course page,
// section "Le piege numerique de la decroissance cumulee"), A and P for that
// chunk are instead computed pairwise in fp32 from differences of running
// sums, which never overflow.
//
// Work decomposition: one CTA per (sequence, head, 32-column slice of d_v);
// the columns of the state evolve independently, so the four slices of a
// head run concurrently on four SMs (the S-independent chunk work is redone
// per slice).  Roles inside the CTA, synchronised by mbarriers:
//   warp 0      : TMA producer for q, k, log_alpha, v (two-stage ring)
//   warps 1-4   : state chain: S -> bf16 operand, decay, U read-out,
//                 outputs and final state; issues the state-path MMAs
//   warps 5-12  : chunk preparation: running sums, gated operands, A/P
//                 read-out, triangular solve, W read-out; issues the
//                 chunk-local MMAs
// so the preparation of chunk n+1 overlaps the state chain of chunk n.
#include <cuda.h>

#include "kda_internal.cuh"
#include "kda_sm100.cuh"

namespace kda {
namespace tc {

using namespace sm100;

constexpr int C = 64;          // chunk length
constexpr int DK = 128;
constexpr int DV = 128;
constexpr int DVT = 32;        // d_v columns per CTA
constexpr int NTILE = DV / DVT;
constexpr int kThreads = 416;  // 13 warps
constexpr int kChainWarp0 = 1, kChainThreads = 128;
constexpr int kPrepWarp0 = 5, kPrepThreads = 256;
constexpr uint32_t kBarChain = 1, kBarPrep = 2;
constexpr uint32_t kTmemCols = 512;
constexpr float kSlowPathLogDecay = -60.0f;   // chunk log-decay below this -> pairwise path

// TMEM column map (lane = row of the accumulator)
constexpr uint32_t kColAP = 0;     // [Ktil;Qtil] Khat^T : M=128, N=64
constexpr uint32_t kColW = 64;     // T_beta Ktil        : M=64,  N=128
constexpr uint32_t kColUp = 192;   // U' (x2 stages)     : M=128, N=32 (rows 0-63 used)
constexpr uint32_t kColUO = 256;   // [-W S; O] (x2)     : M=128, N=32 (rows 0-63: -W S, 64-127: O)
constexpr uint32_t kColS = 320;    // state              : M=128, N=32

// Shared memory map (bytes from a 1024-aligned base)
struct Smem {
    static constexpr uint32_t STACK = 0;          // 2 x 32 KB: [Ktil rows 0-63 | Qtil rows 64-127] x 2 K-atoms
    static constexpr uint32_t KBAR = 65536;       // 2 x 16 KB: Kbar [64 t][128 c], 2 K-atoms of 8 KB
    static constexpr uint32_t KHAT = 98304;       // 16 KB Khat [64 i][128 c]
    static constexpr uint32_t AF = 114688;        // 16 KB: A fp32 64x64 (row-XOR layout)
    static constexpr uint32_t TF = 131072;        // 16 KB: T fp32 64x64
    static constexpr uint32_t GRAW = 147456;      // 2 x 16 KB: raw log_alpha [64 t][128 c]
    static constexpr uint32_t TB = 180224;        // 8 KB: T diag(beta), bf16 [64 t][64 i]
    static constexpr uint32_t PB = 188416;        // 2 x 8 KB: P bf16 [64 t][64 i]
    // TB, PB[0], PB[1] are contiguous: an M = 128 operand that starts 64 rows
    // before PB[s] (or at TB) reads rows 64-127 from PB[s] (or PB[0]); the
    // first 64 rows only feed accumulator rows that are never read.
    static constexpr uint32_t SB = 204800;        // 8 KB: S bf16 [128 c][32 j] (64-byte rows)
    static constexpr uint32_t VT = 212992;        // 2 x 4 KB: V [64 t][32 j]
    static constexpr uint32_t UB = 221184;        // 4 KB: U bf16 [64 t][32 j]
    static constexpr uint32_t BETA = 225280;      // 2 x 64 fp32: beta per stage (zero past the end)
    static constexpr uint32_t EGL = 225792;       // 2 x 128 fp32: exp(G_L) per stage
    static constexpr uint32_t CSUM = 226816;      // 4 x 128 fp32: running-sum partials
    static constexpr uint32_t BARS = 228864;      // mbarriers
    static constexpr uint32_t MISC = 229120;      // tmem base, flags
    static constexpr uint32_t SIZE = 229184;
    static constexpr uint32_t ALLOC = SIZE + 1024;  // room to align the base
};
static_assert(Smem::ALLOC <= 232448, "shared memory budget");

// mbarrier slots (uint64 each) inside Smem::BARS
enum Bar : int {
    RAW_FULL = 0,     // [2] TMA -> prep
    RAW_EMPTY = 2,    // [2] prep + state-path MMAs -> TMA (2 arrivals)
    GATE_READY = 4,   // [2] prep -> chain (exp(G_L) ready; Ktil/Qtil/Kbar written)
    AP_FULL = 6,      // product [A;P] done -> prep
    W_FULL = 7,       // W and U' products done -> prep
    WB_READY = 8,     // -W written over Ktil in STACK[s] -> chain
    ACCU_EMPTY = 9,   // [2] chain read U' -> prep may write U' again
    U_FULL = 11,      // [2] [-W; Qtil] S done -> chain
    CHAIN_DONE = 13,  // [2] state update + output products done -> chain, prep
    FINAL = 15,       // end-of-kernel drain of this thread's MMAs
    FINAL2 = 16,
    kNumBars = 17
};

struct Params {
    const __nv_bfloat16 *k, *q, *beta;            // raw pointers for the pairwise path
    const __nv_bfloat16 *g;                       // log_alpha [T, H] when scalar_gate
    int scalar_gate;
    const float *init_state;
    float *final_state;
    __nv_bfloat16 *o;
    const int32_t *cu;                            // may be null: equal lengths
    const int32_t *perm;                          // sequence order (longest first) or null
    uint32_t *err_word;
    int64_t total_tokens;
    int num_seqs, H;
};


constexpr float kLog2e = 1.4426950408889634f;

// e^x through the hardware base-2 exponential (ex2.approx, flush-to-zero):
// its relative error (~2^-22) is far below the bf16 rounding of the operands
// it scales.
__device__ __forceinline__ float exp_f(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x * kLog2e));
    return y;
}

__device__ __forceinline__ uint64_t *bars(uint8_t *sm) {
    return reinterpret_cast<uint64_t *>(sm + Smem::BARS);
}

// Per-CTA flags in Smem::MISC: [0] TMEM base, [1] abort, [2] pairwise-path flag.
__device__ __forceinline__ uint32_t *misc(uint8_t *sm) {
    return reinterpret_cast<uint32_t *>(sm + Smem::MISC);
}

// Index of A / T element (t, i) in the 64x64 fp32 tiles: rows of 64 floats,
// column XORed with the row's low 5 bits so that row-parallel accesses hit
// distinct banks.
__device__ __forceinline__ int fidx(int t, int i) { return t * 64 + (i ^ (t & 31)); }

// ---- preparation step 1: running sums of log_alpha and the gated operands.
// Thread pt (0..255) owns channels c, c+1 (c = 2 (pt mod 64)) for the 16
// tokens of group pt / 64; a warp covers one 64-channel K-atom of one token
// group, so every shared-memory access below is a full 128-byte row.
// Returns whether the chunk takes the pairwise path.
__device__ bool prep_gate(uint8_t *__restrict__ sm, int pt, int s, int L) {
    const int c = 2 * (pt & 63);
    const int tg = pt >> 6;
    const int t0 = tg * 16;
    float *csum = reinterpret_cast<float *>(sm + Smem::CSUM);
    uint32_t *flags = misc(sm);
    const uint8_t *graw = sm + Smem::GRAW + s * 16384;
    const int katom = c >> 6, cc = c & 63;
    uint8_t *stack = sm + Smem::STACK + s * 32768 + katom * 16384;
    uint8_t *khat = sm + Smem::KHAT + katom * 8192;
    uint8_t *kbar = sm + Smem::KBAR + s * 16384 + katom * 8192;

    // issue every load of this thread's slice first
    uint32_t graw_v[16], k_v[16], q_v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int t = t0 + i;
        graw_v[i] = *reinterpret_cast<const uint32_t *>(graw + t * 256 + c * 2);
        k_v[i] = *reinterpret_cast<const uint32_t *>(stack + sw128_off(t, cc));
        q_v[i] = *reinterpret_cast<const uint32_t *>(stack + sw128_off(64 + t, cc));
    }
    float g0[16], g1[16];
    float r0 = 0.f, r1 = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const bool valid = t0 + i < L;
        const __nv_bfloat162 gv = *reinterpret_cast<const __nv_bfloat162 *>(&graw_v[i]);
        r0 += valid ? clamp_log_alpha(__low2float(gv)) : 0.f;
        r1 += valid ? clamp_log_alpha(__high2float(gv)) : 0.f;
        g0[i] = r0;
        g1[i] = r1;
    }
    csum[tg * 128 + c] = r0;
    csum[tg * 128 + c + 1] = r1;
    if (pt == 0) flags[2] = 0u;
    named_barrier(kBarPrep, kPrepThreads);

    float off0 = 0.f, off1 = 0.f, GL0 = 0.f, GL1 = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float a = csum[j * 128 + c], b = csum[j * 128 + c + 1];
        if (j < tg) { off0 += a; off1 += b; }
        GL0 += a;
        GL1 += b;
    }
    if (tg == 0 && (GL0 < kSlowPathLogDecay || GL1 < kSlowPathLogDecay)) flags[2] = 1u;
    named_barrier(kBarPrep, kPrepThreads);
    const bool slow = flags[2] != 0u;

    const float eL0 = exp_f(GL0), eL1 = exp_f(GL1);
    if (tg == 0) {
        float *egl = reinterpret_cast<float *>(sm + Smem::EGL) + s * 128;
        egl[c] = eL0;
        egl[c + 1] = eL1;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int t = t0 + i;
        const bool valid = t < L;
        const __nv_bfloat162 kv = *reinterpret_cast<const __nv_bfloat162 *>(&k_v[i]);
        const __nv_bfloat162 qv = *reinterpret_cast<const __nv_bfloat162 *>(&q_v[i]);
        const float k0 = valid ? __low2float(kv) : 0.f, k1 = valid ? __high2float(kv) : 0.f;
        const float q0 = valid ? __low2float(qv) : 0.f, q1 = valid ? __high2float(qv) : 0.f;
        const float G0 = g0[i] + off0, G1 = g1[i] + off1;
        const float e0 = exp_f(G0), e1 = exp_f(G1);
        const float ih0 = exp_f(fminf(-G0, 80.f)), ih1 = exp_f(fminf(-G1, 80.f));
        float b0, b1;
        if (slow) {
            b0 = exp_f(GL0 - G0);
            b1 = exp_f(GL1 - G1);
        } else {
            b0 = eL0 * ih0;
            b1 = eL1 * ih1;
        }
        const uint32_t ok = sw128_off(t, cc);
        *reinterpret_cast<uint32_t *>(stack + ok) = pack_bf16x2(k0 * e0, k1 * e1);
        *reinterpret_cast<uint32_t *>(stack + sw128_off(64 + t, cc)) = pack_bf16x2(q0 * e0, q1 * e1);
        *reinterpret_cast<uint32_t *>(khat + ok) = pack_bf16x2(k0 * ih0, k1 * ih1);
        *reinterpret_cast<uint32_t *>(kbar + ok) = pack_bf16x2(k0 * b0, k1 * b1);
    }
    return slow;
}

// 32 consecutive bf16 of a global row as fp32 (zeros when !valid).
__device__ __forceinline__ void row32_f(const __nv_bfloat16 *src, float (&v)[32], bool valid) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        if (valid) w = reinterpret_cast<const uint4 *>(src)[q];
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 h2 = *reinterpret_cast<const __nv_bfloat162 *>(&ww[e]);
            v[8 * q + 2 * e] = __low2float(h2);
            v[8 * q + 2 * e + 1] = __high2float(h2);
        }
    }
}

// ---- pairwise fallback for A and P when a chunk decays too fast for the
// product form.  A quad of lanes (four groups of 32 channels) owns column i
// and walks the rows t = i .. 63 in order, carrying d = G_t - G_i (the sum of
// log_alpha over tokens i+1 .. t) per channel, so every exponent is a
// difference of running sums taken in fp32 and is <= 0; the quad's partial
// sums are combined with shuffles.  All lanes of a warp walk the same rows
// (from the warp's first column), so the shuffles stay converged.
__device__ void prep_pairwise(uint8_t *sm, int pt, int s, int L, const Params &p,
                              int64_t tok0, int h) {
    const uint8_t *graw = sm + Smem::GRAW + s * 16384;
    const float *beta = reinterpret_cast<const float *>(sm + Smem::BETA) + s * C;
    float *AF = reinterpret_cast<float *>(sm + Smem::AF);
    uint8_t *pb = sm + Smem::PB + s * 8192;
    const size_t row_stride = (size_t)p.H * DK;
    const __nv_bfloat16 *kt0 = p.k + ((size_t)tok0 * p.H + h) * DK;
    const __nv_bfloat16 *qt0 = p.q + ((size_t)tok0 * p.H + h) * DK;
    const int i = pt >> 2, cg = pt & 3, c0 = 32 * cg;
    const bool lead = cg == 0;
    const int t_first = (pt >> 5) * 8;
    float ki[32], d[32];
    row32_f(kt0 + (size_t)i * row_stride + c0, ki, i < L);
#pragma unroll
    for (int c = 0; c < 32; ++c) d[c] = 0.f;
    if (lead) {   // rows above the diagonal
        for (int t = 0; t < i; ++t) {
            AF[fidx(t, i)] = 0.f;
            *reinterpret_cast<__nv_bfloat16 *>(pb + sw128_off(t, i)) = __float2bfloat16_rn(0.f);
        }
    }
    for (int t = t_first; t < C; ++t) {
        const bool active = t >= i;
        if (t > i) {
            const uint4 *gr = reinterpret_cast<const uint4 *>(graw + t * 256 + c0 * 2);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 w = gr[q];
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const __nv_bfloat162 h2 = *reinterpret_cast<const __nv_bfloat162 *>(&ww[e]);
                    d[8 * q + 2 * e] += clamp_log_alpha(__low2float(h2));
                    d[8 * q + 2 * e + 1] += clamp_log_alpha(__high2float(h2));
                }
            }
        }
        float kt[32], qt[32];
        row32_f(kt0 + (size_t)t * row_stride + c0, kt, active && t < L);
        row32_f(qt0 + (size_t)t * row_stride + c0, qt, active && t < L);
        float a = 0.f, pq = 0.f;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
            const float w = ki[c] * exp_f(d[c]);
            a = fmaf(kt[c], w, a);
            pq = fmaf(qt[c], w, pq);
        }
        a += __shfl_xor_sync(0xffffffffu, a, 1);
        a += __shfl_xor_sync(0xffffffffu, a, 2);
        pq += __shfl_xor_sync(0xffffffffu, pq, 1);
        pq += __shfl_xor_sync(0xffffffffu, pq, 2);
        if (lead && active) {
            AF[fidx(t, i)] = (t > i) ? beta[t] * a : 0.f;
            *reinterpret_cast<__nv_bfloat16 *>(pb + sw128_off(t, i)) = __float2bfloat16_rn(pq);
        }
    }
}

// ---- preparation step 2: read [A; P] from TMEM.  Warp w of the preparation
// group reads TMEM lanes 32 (w mod 4) .. +31 (rows 0-63 are Ktil Khat^T,
// rows 64-127 are Qtil Khat^T) and 32 of the 64 columns.
__device__ void prep_read_ap(uint8_t *sm, uint32_t tmem, int warp, int lane, int s) {
    const int quad = warp & 3, half = (warp - kPrepWarp0) >> 2;
    float v[32];
    tmem_ld32(tmem_addr(tmem, 32 * quad, kColAP + 32 * half), v);
    tmem_wait_ld();
    const float *beta = reinterpret_cast<const float *>(sm + Smem::BETA) + s * C;
    if (quad < 2) {
        float *AF = reinterpret_cast<float *>(sm + Smem::AF);
        const int t = 32 * quad + lane;
        const float bt = beta[t];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int i = 32 * half + j;
            AF[fidx(t, i)] = (i < t) ? bt * v[j] : 0.f;
        }
    } else {
        uint8_t *pb = sm + Smem::PB + s * 8192;
        const int t = 32 * (quad - 2) + lane;
#pragma unroll
        for (int j = 0; j < 32; j += 8) {
            float w[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) w[e] = (32 * half + j + e <= t) ? v[j + e] : 0.f;
            uint4 pk;
            pk.x = pack_bf16x2(w[0], w[1]);
            pk.y = pack_bf16x2(w[2], w[3]);
            pk.z = pack_bf16x2(w[4], w[5]);
            pk.w = pack_bf16x2(w[6], w[7]);
            *reinterpret_cast<uint4 *>(pb + sw128_off(t, 32 * half + j)) = pk;
        }
    }
}

// ---- preparation step 3: T = (I + A)^{-1} for the unit lower-triangular
// 64x64 system by recursive doubling: the sixteen 4x4 diagonal blocks in
// closed form (forward substitution written out), then four merge levels that
// combine neighbouring m x m inverses into 2m x 2m ones,
//     [[T1, 0], [T21, T2]],   T21 = -T2 (A21 T1),
// for m = 4, 8, 16, 32.  Each level is two fully parallel products (one 1x4
// row segment per thread).  Writes T diag(beta) as bf16 into TB.

// T tile layout: rows of 64 floats; the float4 group index is XORed with
// (row mod 16), so that row segments load as float4 and threads on
// different rows hit different banks.
__device__ __forceinline__ int tfi(int row, int col) {
    return row * 64 + ((((col >> 2) ^ (row & 15))) << 2) + (col & 3);
}

template <int M>
__device__ __forceinline__ void solve_merge(const float *__restrict__ AF, float *__restrict__ TF,
                                            float *__restrict__ XF, int pt) {
    // (64 / 2M) merges, each M x M outputs in 1x4 segments: 8M threads.
    // Thread layout for X = A21 T1: a warp shares one 4-column group, lanes
    // run over rows, so the loop can start at k = c4 (T1 is lower
    // triangular).  For T21 = -T2 X: a warp shares a group of rows, so the
    // loop can stop after the group's last row (T2 is lower triangular).
    constexpr int kThr = 8 * M;
    constexpr int SEG = M / 4;                // 4-column groups per row
    constexpr int PER = M * SEG;              // threads per merge
    constexpr int XS = M + 4;                 // padded row stride of X (bank spread)
    if (pt < kThr) {   // X = A21 T1
        const int merge = pt / PER, rem = pt % PER;
        const int c4 = (rem / M) * 4, r = rem % M;   // column group outer, row inner
        const int base = merge * 2 * M;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
        for (int k = c4; k < M; ++k) {
            const float av = AF[fidx(base + M + r, base + k)];
            const float4 tv = *reinterpret_cast<const float4 *>(&TF[tfi(base + k, base + c4)]);
            acc.x = fmaf(av, tv.x, acc.x);
            acc.y = fmaf(av, tv.y, acc.y);
            acc.z = fmaf(av, tv.z, acc.z);
            acc.w = fmaf(av, tv.w, acc.w);
        }
        *reinterpret_cast<float4 *>(&XF[(merge * M + r) * XS + c4]) = acc;
    }
    named_barrier(kBarPrep, kPrepThreads);
    if (pt < kThr) {   // T21 = -T2 X
        const int merge = pt / PER, rem = pt % PER;
        const int r = rem / SEG, c4 = (rem % SEG) * 4;   // row outer, column group inner
        const int base = merge * 2 * M;
        const int rlast = (pt | 31) % PER / SEG;          // last row handled by this warp
        // warps of the M >= 16 levels hold whole row groups of one merge
        const int kend = (M >= 16) ? ((rlast >> 2) + 1) * 4 : M;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int k4 = 0; k4 < kend; k4 += 4) {
            const float4 tr = *reinterpret_cast<const float4 *>(&TF[tfi(base + M + r, base + M + k4)]);
            const float tk[4] = {tr.x, tr.y, tr.z, tr.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float4 xv = *reinterpret_cast<const float4 *>(&XF[(merge * M + k4 + e) * XS + c4]);
                acc.x = fmaf(tk[e], xv.x, acc.x);
                acc.y = fmaf(tk[e], xv.y, acc.y);
                acc.z = fmaf(tk[e], xv.z, acc.z);
                acc.w = fmaf(tk[e], xv.w, acc.w);
            }
        }
        *reinterpret_cast<float4 *>(&TF[tfi(base + M + r, base + c4)]) =
            make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
    }
    named_barrier(kBarPrep, kPrepThreads);
}

__device__ void prep_solve(uint8_t *__restrict__ sm, int pt, int s) {
    const float *__restrict__ AF = reinterpret_cast<const float *>(sm + Smem::AF);
    float *__restrict__ TF = reinterpret_cast<float *>(sm + Smem::TF);
    float *__restrict__ XF = reinterpret_cast<float *>(sm + Smem::GRAW + s * 16384);  // raw g is spent
    const float *__restrict__ beta = reinterpret_cast<const float *>(sm + Smem::BETA) + s * C;

    // zero every float4 group of T outside the 4x4 diagonal blocks
    for (int v = pt; v < 1024; v += kPrepThreads) {
        const int row = v >> 4, g4 = v & 15;
        if (g4 != (row >> 2))
            *reinterpret_cast<float4 *>(&TF[tfi(row, 4 * g4)]) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    // 4x4 diagonal blocks: T = L^{-1} for unit lower-triangular L = I + N
    if (pt < 16) {
        const int b0 = 4 * pt;
        const float n10 = AF[fidx(b0 + 1, b0)];
        const float n20 = AF[fidx(b0 + 2, b0)], n21 = AF[fidx(b0 + 2, b0 + 1)];
        const float n30 = AF[fidx(b0 + 3, b0)], n31 = AF[fidx(b0 + 3, b0 + 1)],
                    n32 = AF[fidx(b0 + 3, b0 + 2)];
        const float t10 = -n10, t21 = -n21, t32 = -n32;
        const float t20 = -(n20 + n21 * t10);
        const float t31 = -(n31 + n32 * t21);
        const float t30 = -(n30 + n31 * t10 + n32 * t20);
        *reinterpret_cast<float4 *>(&TF[tfi(b0 + 0, b0)]) = make_float4(1.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4 *>(&TF[tfi(b0 + 1, b0)]) = make_float4(t10, 1.f, 0.f, 0.f);
        *reinterpret_cast<float4 *>(&TF[tfi(b0 + 2, b0)]) = make_float4(t20, t21, 1.f, 0.f);
        *reinterpret_cast<float4 *>(&TF[tfi(b0 + 3, b0)]) = make_float4(t30, t31, t32, 1.f);
    }
    named_barrier(kBarPrep, kPrepThreads);
    solve_merge<4>(AF, TF, XF, pt);
    solve_merge<8>(AF, TF, XF, pt);
    solve_merge<16>(AF, TF, XF, pt);
    solve_merge<32>(AF, TF, XF, pt);

    // T diag(beta) -> bf16, K-major 128-byte-swizzled [64 t][64 i]
    uint8_t *tb = sm + Smem::TB;
    const int t = pt >> 2, i0 = (pt & 3) * 16;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const float4 u0 = *reinterpret_cast<const float4 *>(&TF[tfi(t, i0 + 8 * hh)]);
        const float4 u1 = *reinterpret_cast<const float4 *>(&TF[tfi(t, i0 + 8 * hh + 4)]);
        const float *bb = beta + i0 + 8 * hh;
        uint4 pk;
        pk.x = pack_bf16x2(u0.x * bb[0], u0.y * bb[1]);
        pk.y = pack_bf16x2(u0.z * bb[2], u0.w * bb[3]);
        pk.z = pack_bf16x2(u1.x * bb[4], u1.y * bb[5]);
        pk.w = pack_bf16x2(u1.z * bb[6], u1.w * bb[7]);
        *reinterpret_cast<uint4 *>(tb + sw128_off(t, i0 + 8 * hh)) = pk;
    }
}

// ---- preparation step 4: -W from TMEM (M = 64 layout: row r sits in lane
// (r mod 16) + 32 (r / 16)) as bf16 over Ktil, i.e. rows 0-63 of STACK[s]
// (K-major, 64 channels per K-atom), so that [-W; Qtil] is one M = 128 operand.
__device__ void prep_read_w(uint8_t *sm, uint32_t tmem, int warp, int lane, int s) {
    const int quad = warp & 3, half = (warp - kPrepWarp0) >> 2;
    uint8_t *wdst = sm + Smem::STACK + s * 32768 + half * 16384;
    const int t = 16 * quad + lane;
#pragma unroll
    for (int part = 0; part < 2; ++part) {
        float v[32];
        tmem_ld32(tmem_addr(tmem, 32 * quad, kColW + 64 * half + 32 * part), v);
        tmem_wait_ld();
        if (lane < 16) {
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
                uint4 pk;
                pk.x = pack_bf16x2(-v[j + 0], -v[j + 1]);
                pk.y = pack_bf16x2(-v[j + 2], -v[j + 3]);
                pk.z = pack_bf16x2(-v[j + 4], -v[j + 5]);
                pk.w = pack_bf16x2(-v[j + 6], -v[j + 7]);
                *reinterpret_cast<uint4 *>(wdst + sw128_off(t, 32 * part + j)) = pk;
            }
        }
    }
}

// Bounded wait used only while draining at the end of the kernel: it ignores
// the abort flag (the copies and products it waits for are already issued).
__device__ __forceinline__ void mbar_wait_drain(uint64_t *bar, uint32_t parity) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > 1000000000ull) return;
    }
}

constexpr uint32_t kRawBytes = 2 * 8192 + 2 * 8192 + 16384 + C * DVT * 2;

// ---- chain step helpers ---------------------------------------------------------

// O rows of chunk m from TMEM (rows 64-127 of the M = 128 accumulator
// [-W S; O], i.e. lanes 64-127: the warps of quadrants 2 and 3) to global
// memory, bf16.
__device__ __forceinline__ void chain_store_o(uint32_t tmem, int quad, int lane, int m,
                                              int64_t bos, int64_t len, int h, int j0,
                                              const Params &p) {
    if (quad < 2) return;
    const int st = m & 1;
    float v[32];
    tmem_ld32(tmem_addr(tmem, 32 * quad, kColUO + 32 * st), v);
    tmem_wait_ld();
    const int t = 32 * (quad - 2) + lane;
    const int64_t tok = bos + (int64_t)m * C + t;
    if ((int64_t)m * C + t < len) {
        uint4 *dst = reinterpret_cast<uint4 *>(p.o + ((size_t)tok * p.H + h) * DV + j0);
#pragma unroll
        for (int j = 0; j < 32; j += 8) {
            uint4 pk;
            pk.x = pack_bf16x2(v[j + 0], v[j + 1]);
            pk.y = pack_bf16x2(v[j + 2], v[j + 3]);
            pk.z = pack_bf16x2(v[j + 4], v[j + 5]);
            pk.w = pack_bf16x2(v[j + 6], v[j + 7]);
            dst[j / 8] = pk;
        }
    }
}

__device__ __forceinline__ void store_bf16_row_sw64(uint8_t *tile, int row, const float (&v)[32]) {
#pragma unroll
    for (int j = 0; j < 32; j += 8) {
        uint4 pk;
        pk.x = pack_bf16x2(v[j + 0], v[j + 1]);
        pk.y = pack_bf16x2(v[j + 2], v[j + 3]);
        pk.z = pack_bf16x2(v[j + 4], v[j + 5]);
        pk.w = pack_bf16x2(v[j + 6], v[j + 7]);
        *reinterpret_cast<uint4 *>(tile + sw64_off(row, j)) = pk;
    }
}

// ---- the kernel ------------------------------------------------------------------

__global__ void __launch_bounds__(kThreads, 1)
kda_prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_g,
                      const __grid_constant__ CUtensorMap tm_v, const Params p) {
    extern __shared__ uint8_t dyn_smem[];
    uint8_t *sm = dyn_smem + ((1024u - (smem_addr(dyn_smem) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    const int item = blockIdx.x;
    const int tile = item % NTILE;
    const int h = (item / NTILE) % p.H;
    const int rank = item / (NTILE * p.H);
    const int seq = p.perm ? p.perm[rank] : rank;
    int64_t bos, eos;
    if (p.cu) {
        bos = p.cu[seq];
        eos = p.cu[seq + 1];
        if (bos < 0 || eos < bos || eos > p.total_tokens) bos = eos = 0;  // flagged by the plan kernel
    } else {
        const int64_t len = p.total_tokens / p.num_seqs;
        bos = (int64_t)seq * len;
        eos = bos + len;
    }
    const int64_t len = eos - bos;
    const int nchunks = (int)((len + C - 1) / C);
    const int j0 = tile * DVT;

    uint64_t *B = bars(sm);
    uint32_t *flags = misc(sm);
    volatile uint32_t *abort_flag = flags + 1;
    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i)
            mbar_init(&B[i], (i == RAW_EMPTY || i == RAW_EMPTY + 1 || i == RAW_FULL ||
                                  i == RAW_FULL + 1) ? 2u : 1u);
        flags[1] = 0u;
        flags[2] = 0u;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&flags[0], kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = flags[0];

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        // Lane 0 issues the tensor copies; the whole warp then loads the
        // chunk's 64 beta values (a strided gather TMA cannot do) into the
        // matching ring slot and lane 0 adds the second arrival.
        if (nchunks > 0) {
            if (lane == 0) {
                tma_prefetch_desc(&tm_k);
                tma_prefetch_desc(&tm_q);
                tma_prefetch_desc(&tm_g);
                tma_prefetch_desc(&tm_v);
            }
            float *betar = reinterpret_cast<float *>(sm + Smem::BETA);
            int issued = 0;
            for (int n = 0; n < nchunks; ++n) {
                const int s = n & 1;
                int stop = 0;
                if (lane == 0) {
                    if (n >= 2) mbar_wait(&B[RAW_EMPTY + s], ((n - 2) >> 1) & 1, abort_flag);
                    stop = *abort_flag ? 1 : 0;
                }
                stop = __shfl_sync(0xffffffffu, stop, 0);
                if (stop) break;
                __syncwarp();   // lane 0's wait for the free slot orders the warp's stores below
                const int tok = (int)(bos + (int64_t)n * C);
                if (lane == 0) {
                    mbar_arrive_expect_tx(&B[RAW_FULL + s], p.scalar_gate ? kRawBytes - 16384 : kRawBytes);
                    uint8_t *stk = sm + Smem::STACK + s * 32768;
                    tma_load_3d(stk, &tm_k, &B[RAW_FULL + s], 0, h, tok);
                    tma_load_3d(stk + 16384, &tm_k, &B[RAW_FULL + s], 64, h, tok);
                    tma_load_3d(stk + 8192, &tm_q, &B[RAW_FULL + s], 0, h, tok);
                    tma_load_3d(stk + 16384 + 8192, &tm_q, &B[RAW_FULL + s], 64, h, tok);
                    if (!p.scalar_gate)
                        tma_load_3d(sm + Smem::GRAW + s * 16384, &tm_g, &B[RAW_FULL + s], 0, h, tok);
                    tma_load_3d(sm + Smem::VT + s * 4096, &tm_v, &B[RAW_FULL + s], j0, h, tok);
                }
                const int64_t rem = len - (int64_t)n * C;
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int t = lane + 32 * e;
                    float b = 0.f;
                    if (t < rem) b = __bfloat162float(p.beta[(size_t)(tok + t) * p.H + h]);
                    betar[s * C + t] = b;
                    if (p.scalar_gate) {   // one log_alpha per token: broadcast over its 128 channels
                        __nv_bfloat16 gv = __float2bfloat16(0.f);
                        if (t < rem) gv = p.g[(size_t)(tok + t) * p.H + h];
                        const __nv_bfloat162 g2 = __halves2bfloat162(gv, gv);
                        const uint32_t gw = *reinterpret_cast<const uint32_t *>(&g2);
                        uint4 *row = reinterpret_cast<uint4 *>(sm + Smem::GRAW + s * 16384 + t * 256);
#pragma unroll
                        for (int i = 0; i < 16; ++i) row[i] = make_uint4(gw, gw, gw, gw);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&B[RAW_FULL + s]);
                issued = n + 1;
            }
            // every issued copy must have landed before the CTA's memory is released
            if (lane == 0)
                for (int n = (issued > 2 ? issued - 2 : 0); n < issued; ++n)
                    mbar_wait_drain(&B[RAW_FULL + (n & 1)], (n >> 1) & 1);
        }
    } else if (warp < kPrepWarp0) {
        // ------------------------------------------------ state chain
        const int ct = tid - 32 * kChainWarp0;
        const bool leader = ct == 0;
        const int quad = warp & 3;
        const int crow = 32 * quad + lane;
        const size_t soff = ((size_t)seq * p.H + h) * (size_t)(DK * DV) + (size_t)crow * DV + j0;
        float S[32];
        if (p.init_state) {
            const float4 *src = reinterpret_cast<const float4 *>(p.init_state + soff);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 v = src[i];
                S[4 * i] = v.x; S[4 * i + 1] = v.y; S[4 * i + 2] = v.z; S[4 * i + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) S[i] = 0.f;
        }
        const float *egl = reinterpret_cast<const float *>(sm + Smem::EGL);
        for (int n = 0; n < nchunks; ++n) {
            const int s = n & 1;
            if (n >= 1) {
                mbar_wait(&B[CHAIN_DONE + ((n - 1) & 1)], ((n - 1) >> 1) & 1, abort_flag);
                tc_fence_after();
                tmem_ld32(tmem_addr(tmem, 32 * quad, kColS), S);
                tmem_wait_ld();
            }
            store_bf16_row_sw64(sm + Smem::SB, crow, S);
            mbar_wait(&B[GATE_READY + s], (n >> 1) & 1, abort_flag);
            const float d = egl[s * 128 + crow];
#pragma unroll
            for (int i = 0; i < 32; ++i) S[i] *= d;
            tmem_st32(tmem_addr(tmem, 32 * quad, kColS), S);
            tmem_wait_st();
            fence_async_smem();
            tc_fence_before();
            named_barrier(kBarChain, kChainThreads);
            if (leader) {
                tc_fence_after();
                mbar_wait(&B[WB_READY], n & 1, abort_flag);
                const uint32_t aWQ = smem_addr(sm + Smem::STACK + s * 32768);
                const uint32_t bS = smem_addr(sm + Smem::SB);
                const uint32_t id = idesc_bf16(128, DVT, false, true);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)   // [-W S; Qtil S] = [-W; Qtil] S
                    mma_bf16(tmem + kColUO + 32 * s,
                             smem_desc(aWQ + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kLayoutSW128),
                             smem_desc(bS + ks * 1024, 16, 512, kLayoutSW64), id, ks > 0 ? 1u : 0u);
                mma_commit(&B[U_FULL + s]);
                mma_commit(&B[RAW_EMPTY + s]);
            }
            if (n >= 1) chain_store_o(tmem, quad, lane, n - 1, bos, len, h, j0, p);

            mbar_wait(&B[U_FULL + s], (n >> 1) & 1, abort_flag);
            tc_fence_after();
            float U[32];
            if (quad < 2) {   // U = U' - W S for rows 0-63 (lanes 0-63)
                float Wp[32];
                tmem_ld32(tmem_addr(tmem, 32 * quad, kColUO + 32 * s), U);
                tmem_ld32(tmem_addr(tmem, 32 * quad, kColUp + 32 * s), Wp);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) U[i] += Wp[i];
                store_bf16_row_sw64(sm + Smem::UB, 32 * quad + lane, U);
            }
            fence_async_smem();
            tc_fence_before();
            named_barrier(kBarChain, kChainThreads);
            if (leader) {
                tc_fence_after();
                mbar_arrive(&B[ACCU_EMPTY + s]);
                const uint32_t aK = smem_addr(sm + Smem::KBAR + s * 16384);
                const uint32_t aP = smem_addr(sm + Smem::PB + s * 8192 - 8192);
                const uint32_t bU = smem_addr(sm + Smem::UB);
                const uint32_t idS = idesc_bf16(128, DVT, true, true);
                const uint32_t idO = idesc_bf16(128, DVT, false, true);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)   // S += Kbar^T U
                    mma_bf16(tmem + kColS, smem_desc(aK + ks * 2048, 8192, 1024, kLayoutSW128),
                             smem_desc(bU + ks * 1024, 16, 512, kLayoutSW64), idS, 1u);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)   // O += P U (rows 64-127 of an M = 128 product)
                    mma_bf16(tmem + kColUO + 32 * s, smem_desc(aP + ks * 32, 16, 1024, kLayoutSW128),
                             smem_desc(bU + ks * 1024, 16, 512, kLayoutSW64), idO, 1u);
                mma_commit(&B[CHAIN_DONE + s]);
            }
        }
        if (nchunks > 0) {
            const int n = nchunks - 1;
            mbar_wait(&B[CHAIN_DONE + (n & 1)], (n >> 1) & 1, abort_flag);
            tc_fence_after();
            chain_store_o(tmem, quad, lane, n, bos, len, h, j0, p);
            tmem_ld32(tmem_addr(tmem, 32 * quad, kColS), S);
            tmem_wait_ld();
            if (leader) {
                mma_commit(&B[FINAL2]);
                mbar_wait_drain(&B[FINAL2], 0);
            }
        }
        if (p.final_state) {
            float4 *dst = reinterpret_cast<float4 *>(p.final_state + soff);
#pragma unroll
            for (int i = 0; i < 8; ++i)
                dst[i] = make_float4(S[4 * i], S[4 * i + 1], S[4 * i + 2], S[4 * i + 3]);
        }
    } else {
        // ------------------------------------------------ chunk preparation
        const int pt = tid - 32 * kPrepWarp0;
        const bool leader = pt == 0;
        for (int n = 0; n < nchunks; ++n) {
            const int s = n & 1;
            const int L = (int)min((int64_t)C, len - (int64_t)n * C);
            const int64_t tok0 = bos + (int64_t)n * C;
            mbar_wait(&B[RAW_FULL + s], (n >> 1) & 1, abort_flag);
            if (n >= 2) mbar_wait(&B[CHAIN_DONE + s], ((n - 2) >> 1) & 1, abort_flag);
            const bool slow = prep_gate(sm, pt, s, L);
            fence_async_smem();
            named_barrier(kBarPrep, kPrepThreads);
            if (leader) {
                tc_fence_after();
                const uint32_t a0 = smem_addr(sm + Smem::STACK + s * 32768);
                const uint32_t b0 = smem_addr(sm + Smem::KHAT);
                const uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)   // [Ktil; Qtil] Khat^T
                    mma_bf16(tmem + kColAP,
                             smem_desc(a0 + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kLayoutSW128),
                             smem_desc(b0 + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024, kLayoutSW128),
                             id, ks > 0 ? 1u : 0u);
                mma_commit(&B[AP_FULL]);
                mbar_arrive(&B[GATE_READY + s]);
            }
            mbar_wait(&B[AP_FULL], n & 1, abort_flag);
            tc_fence_after();
            if (!slow) prep_read_ap(sm, tmem, warp, lane, s);
            else prep_pairwise(sm, pt, s, L, p, tok0, h);
            tc_fence_before();
            named_barrier(kBarPrep, kPrepThreads);
            prep_solve(sm, pt, s);
            fence_async_smem();
            named_barrier(kBarPrep, kPrepThreads);
            if (leader) {
                tc_fence_after();
                if (n >= 2) mbar_wait(&B[ACCU_EMPTY + s], ((n - 2) >> 1) & 1, abort_flag);
                const uint32_t aT = smem_addr(sm + Smem::TB);
                const uint32_t bK = smem_addr(sm + Smem::STACK + s * 32768);
                const uint32_t bV = smem_addr(sm + Smem::VT + s * 4096);
                const uint32_t idW = idesc_bf16(64, DK, false, true);
                const uint32_t idU = idesc_bf16(128, DVT, false, true);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)   // W = T diag(beta) Ktil
                    mma_bf16(tmem + kColW, smem_desc(aT + ks * 32, 16, 1024, kLayoutSW128),
                             smem_desc(bK + ks * 2048, 16384, 1024, kLayoutSW128), idW,
                             ks > 0 ? 1u : 0u);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)   // U' = T diag(beta) V (rows 0-63 of an M = 128 product)
                    mma_bf16(tmem + kColUp + 32 * s, smem_desc(aT + ks * 32, 16, 1024, kLayoutSW128),
                             smem_desc(bV + ks * 1024, 16, 512, kLayoutSW64), idU,
                             ks > 0 ? 1u : 0u);
                mma_commit(&B[W_FULL]);
            }
            mbar_wait(&B[W_FULL], n & 1, abort_flag);
            tc_fence_after();
            prep_read_w(sm, tmem, warp, lane, s);
            tc_fence_before();
            fence_async_smem();
            named_barrier(kBarPrep, kPrepThreads);
            if (leader) {
                mbar_arrive(&B[WB_READY]);
                mbar_arrive(&B[RAW_EMPTY + s]);
            }
        }
        if (leader && nchunks > 0) {
            mma_commit(&B[FINAL]);
            mbar_wait_drain(&B[FINAL], 0);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    if (tid == 0 && *abort_flag) atomicOr(p.err_word, kDevErrTimeout);
}

// ---- plan kernel: checks cu_seqlens (writing the workspace error word, which
// it also clears) and orders sequences longest first, so that the longest
// chains start in the first wave.
constexpr int kPlanThreads = 1024;
constexpr int kMaxSortedSeqs = 4096;

__global__ void __launch_bounds__(kPlanThreads)
kda_plan_kernel(const int32_t *cu, int n, int64_t total, int32_t *perm, uint32_t *err) {
    int bad = 0;
    if (cu) {
        for (int i = threadIdx.x; i < n; i += kPlanThreads) {
            const int64_t a = cu[i], b = cu[i + 1];
            if (a < 0 || b < a || b > total) bad = 1;
        }
        if (threadIdx.x == 0 && (cu[0] != 0 || cu[n] != total)) bad = 1;
    }
    bad = __syncthreads_or(bad);
    if (threadIdx.x == 0) *err = bad ? kDevErrCuSeqlens : kDevErrNone;
    if (!perm) return;
    for (int i = threadIdx.x; i < n; i += kPlanThreads) {
        if (!cu || n > kMaxSortedSeqs) {
            perm[i] = i;
            continue;
        }
        const int64_t li = (int64_t)cu[i + 1] - cu[i];
        int r = 0;
        for (int j = 0; j < n; ++j) {
            const int64_t lj = (int64_t)cu[j + 1] - cu[j];
            r += (lj > li) || (lj == li && j < i);
        }
        perm[r] = i;
    }
}

}  // namespace tc

// ---- host side -------------------------------------------------------------------

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's encoder, looked up once per process (a function-local static
// is initialised once even when several threads arrive together).
EncodeTiledFn encode_fn() {
    static const EncodeTiledFn fn = []() -> EncodeTiledFn {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiledFn>(ptr);
        return nullptr;
    }();
    return fn;
}

// 3-D bf16 view [T][H][inner] of a token-major tensor, box (box_inner, 1, 64).
bool make_map(CUtensorMap *m, const void *base, int64_t T, int H, int inner, int box_inner,
              CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)H, (cuuint64_t)T};
    const cuuint64_t strides[2] = {(cuuint64_t)inner * 2, (cuuint64_t)inner * 2 * H};
    const cuuint32_t box[3] = {(cuuint32_t)box_inner, 1, (cuuint32_t)tc::C};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t prefill_tc_workspace(int num_seqs) {
    return kWorkspaceHeader + (((size_t)num_seqs * sizeof(int32_t) + 255) & ~(size_t)255);
}

cudaError_t launch_prefill_tc(const void *q, const void *k, const void *v, const void *g,
                              const void *beta, const float *init_state, const int32_t *cu,
                              int num_seqs, int64_t total_tokens, int H, void *o,
                              float *final_state, void *workspace, bool scalar_gate,
                              cudaStream_t stream) {
    using namespace tc;
    uint32_t *err = static_cast<uint32_t *>(workspace);
    int32_t *perm = cu ? reinterpret_cast<int32_t *>(static_cast<uint8_t *>(workspace) +
                                                      kWorkspaceHeader)
                       : nullptr;
    CUtensorMap mk, mq, mg, mv;
    if (!make_map(&mk, k, total_tokens, H, DK, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mq, q, total_tokens, H, DK, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        // with a scalar gate the map is never used (log_alpha comes in by plain loads)
        !make_map(&mg, scalar_gate ? k : g, total_tokens, H, DK, 128, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&mv, v, total_tokens, H, DV, DVT, CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    kda_plan_kernel<<<1, kPlanThreads, 0, stream>>>(cu, num_seqs, total_tokens, perm, err);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = set_max_dynamic_smem((const void *)kda_prefill_tc_kernel, (int)Smem::ALLOC);
    if (e != cudaSuccess) return e;
    Params prm;
    prm.k = static_cast<const __nv_bfloat16 *>(k);
    prm.q = static_cast<const __nv_bfloat16 *>(q);
    prm.beta = static_cast<const __nv_bfloat16 *>(beta);
    prm.g = static_cast<const __nv_bfloat16 *>(g);
    prm.scalar_gate = scalar_gate ? 1 : 0;
    prm.init_state = init_state;
    prm.final_state = final_state;
    prm.o = static_cast<__nv_bfloat16 *>(o);
    prm.cu = cu;
    prm.perm = perm;
    prm.err_word = err;
    prm.total_tokens = total_tokens;
    prm.num_seqs = num_seqs;
    prm.H = H;
    const unsigned blocks = (unsigned)((size_t)num_seqs * H * NTILE);
    kda_prefill_tc_kernel<<<blocks, kThreads, Smem::ALLOC, stream>>>(mk, mq, mg, mv, prm);
    return cudaGetLastError();
}

}  // namespace kda
