// Chunk preparation for the tensor-core KDA prefill: everything that does not
// depend on the carried state.  For one chunk of C = 64 tokens of one head,
// with G the running sum of log_alpha from the chunk start:
//     Ktil = K e^G, Qtil = Q e^G, Khat = K e^-G, Kbar = K e^{G_L - G}
//     [A; P] = [Ktil; Qtil] Khat^T  (tensor cores)
//     A = diag(beta) strict_tril(.),  P = tril(.)
//     T = (I + A)^-1 (fp32, recursive doubling),  T_beta = T diag(beta)
// (news digest page on Kimi Linear, section "Algorithme parallele par
// chunks": WY/UT packing of the chunk's rank-1 updates and the triangular
// inverse by forward substitution).  The routines take explicit buffer
// pointers so that kernels with different shared-memory maps can use them;
// the threads of one 256-thread group call each routine together.
#pragma once

#include "kda_internal.cuh"
#include "kda_sm100.cuh"

namespace kda {
namespace prep {

using namespace sm100;

constexpr int C = 64;
constexpr int DK = 128;
constexpr int kGroupThreads = 256;
// A chunk whose log-decay on some channel is below this takes the pairwise
// path: above it, e^{G} and e^{-G} (<= e^80 ~ 5.5e34) are normal numbers in
// bf16 and fp32, so the product form keeps its relative precision.
constexpr float kSlowPathLogDecay = -80.0f;
constexpr float kLog2e = 1.4426950408889634f;

// e^x through the hardware base-2 exponential (ex2.approx, flush-to-zero):
// its relative error (~2^-22) is far below the bf16 rounding of the operands
// it scales.
__device__ __forceinline__ float exp2_f(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float exp_f(float x) { return exp2_f(x * kLog2e); }

// Shared-memory buffers of one chunk's preparation.
struct Bufs {
    uint8_t *stk;        // [Ktil rows 0-63 | Qtil rows 64-127], 2 K-atoms of 16 KB (128-byte swizzle);
                         // raw k / q on entry
    uint8_t *khat;       // Khat [64][128], 2 K-atoms of 8 KB
    uint8_t *kbar;       // Kbar [64][128], 2 K-atoms of 8 KB
    const uint8_t *graw; // raw log_alpha [64][128] bf16, 256-byte rows
    float *af;           // A, fp32 64x64, rows of 65 (16,640 bytes); may alias khat after the product
    float *tf;           // T, fp32 64x64, rows of 68 (17,408 bytes)
    float *xf;           // solve scratch, >= 4608 bytes; may alias graw after gating
    uint8_t *tb;         // T diag(beta) bf16 [64 t][64 i] (one K-atom)
    uint8_t *pb;         // P bf16 [64 t][64 i]
    const float *beta;   // 64 fp32, zero past the chunk end
    float *egl;          // 128 fp32: exp(G_L)
    float *csum;         // 4 x 128 fp32 scratch
    uint32_t *slow_flag; // one word
    // The layer prologue (null nrm: off).  graw then holds the gate
    // pre-activation z on entry and log_alpha = neg_eA softplus(z) (bf16) on
    // exit; q and k are L2-normalised with the factors left in nrm
    // (1 / |k_t| at t, 1 / |q_t| at 64 + t).
    float *nrm;          // 128 fp32, or null
    float neg_eA;        // -exp(A_log[h])
    float qk_eps;
    // The scalar (Gated DeltaNet) gate: one raw log_alpha per token, 64 fp32
    // (zero past the chunk end), or null for the per-channel gate in graw.
    const float *gsc;
    // gate<BAR, LAYER, true> also writes the running sums G (base-2 units,
    // fp32 [64 t][128 c] row-major) here, gate_scalar<BAR, true> the 64 per
    // token, for the backward pass
    float *gout;
};

// Index of A element (t, i): rows padded to 65 floats, so that a warp
// reading one column across 32 rows hits 32 distinct banks, and a thread
// walking a row or a column steps by a constant.
constexpr int kAStride = 65;
__device__ __forceinline__ int fidx(int t, int i) { return t * kAStride + i; }

// T layout: rows padded to 68 floats (float4-aligned); the four rows a warp
// reads at once in the second product of a merge fall in distinct banks.
constexpr int kTStride = 68;
__device__ __forceinline__ int tfi(int row, int col) { return row * kTStride + col; }

// ---- running sums and gated operands.  Thread pt (0..255) owns channels
// c, c+1 (c = 2 (pt mod 64)) for the 16 tokens of group pt / 64; a warp covers
// one 64-channel K-atom of one token group.  Rows past the chunk's end (a
// sequence's last chunk) are zeroed first, so that they add nothing to the
// running sums and give zero operand rows.  The running sums are kept in
// base-2 units (log_alpha log2(e)).  Returns how [A; P] is to be formed:
// kProductForm (one reference, the chunk start), kSecondary (the chunk
// decays below e^-80 on some channel, but no 16-token block does: one
// reference per block) or kPairwise.
enum : int { kProductForm = 0, kSecondary = 1, kPairwise = 2 };

// LAYER: 0 plain; 1 the layer prologue (z -> log_alpha, the norms of the raw
// q and k rows formed here and left in b.nrm); 2 raw q and k scaled by the
// inverse norms already in b.nrm.
template <int BAR, int LAYER, bool GOUT = false>
__device__ int gate(const Bufs &b, int pt, int L) {
    const int c = 2 * (pt & 63);
    const int tg = pt >> 6;
    const int t0 = tg * 16;
    const int katom = c >> 6, cc = c & 63;
    uint8_t *stack = b.stk + katom * 16384;
    uint8_t *khat = b.khat + katom * 8192;
    uint8_t *kbar = b.kbar + katom * 8192;

    if (L < C) {   // uniform over the group
        uint8_t *graw = const_cast<uint8_t *>(b.graw);
        for (int v = pt; v < (C - L) * 16; v += kGroupThreads) {   // 16-byte pieces of a 256-byte row
            const int t = L + (v >> 4), piece = v & 15;
            const uint4 z = make_uint4(0u, 0u, 0u, 0u);
            *reinterpret_cast<uint4 *>(graw + t * 256 + piece * 16) = z;
            uint8_t *atom = b.stk + (piece >> 3) * 16384;
            *reinterpret_cast<uint4 *>(atom + sw128_off(t, (piece & 7) * 8)) = z;
            *reinterpret_cast<uint4 *>(atom + sw128_off(64 + t, (piece & 7) * 8)) = z;
        }
        named_barrier(BAR, kGroupThreads);
    }

    constexpr bool layer = LAYER == 1;    // the prologue
    constexpr bool scaled = LAYER != 0;   // q and k scaled by b.nrm
    uint32_t graw_v[16], k_v[16], q_v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int t = t0 + i;
        k_v[i] = *reinterpret_cast<const uint32_t *>(stack + sw128_off(t, cc));
        q_v[i] = *reinterpret_cast<const uint32_t *>(stack + sw128_off(64 + t, cc));
    }
    if (layer) {
        // Sums of squares of k and q per token: this warp's 64 channels by a
        // reduce-scatter over the lanes (slot s = lane: k of token s for
        // s < 16, q of token s - 16), the two channel halves added after
        // the next barrier.
        const int lane = pt & 31;
        float v[32];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const __nv_bfloat162 kv = *reinterpret_cast<const __nv_bfloat162 *>(&k_v[i]);
            const __nv_bfloat162 qv = *reinterpret_cast<const __nv_bfloat162 *>(&q_v[i]);
            v[i] = __low2float(kv) * __low2float(kv) + __high2float(kv) * __high2float(kv);
            v[16 + i] = __low2float(qv) * __low2float(qv) + __high2float(qv) * __high2float(qv);
        }
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) {
            const bool up = (lane & m) != 0;
#pragma unroll
            for (int j = 0; j < m; ++j) {
                const float lo = v[j], hi = v[j + m];
                const float send = up ? lo : hi;
                const float keep = up ? hi : lo;
                v[j] = keep + __shfl_xor_sync(0xffffffffu, send, m);
            }
        }
        b.xf[katom * 128 + tg * 32 + lane] = v[0];
    }
#pragma unroll
    for (int i = 0; i < 16; ++i)
        graw_v[i] = *reinterpret_cast<const uint32_t *>(b.graw + (t0 + i) * 256 + c * 2);
    float g0[16], g1[16];
    float r0 = 0.f, r1 = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const __nv_bfloat162 gv = *reinterpret_cast<const __nv_bfloat162 *>(&graw_v[i]);
        float x0 = __low2float(gv), x1 = __high2float(gv);
        if (layer) {   // log_alpha = -e^A softplus(z); rows past the chunk end decay nothing
            const bool valid = t0 + i < L;
            x0 = valid ? b.neg_eA * (x0 > 15.f ? x0 : __logf(1.f + __expf(x0))) : 0.f;
            x1 = valid ? b.neg_eA * (x1 > 15.f ? x1 : __logf(1.f + __expf(x1))) : 0.f;
            *reinterpret_cast<uint32_t *>(const_cast<uint8_t *>(b.graw) + (t0 + i) * 256 + c * 2) =
                pack_bf16x2(x0, x1);
        }
        r0 = fmaf(clamp_log_alpha(x0), kLog2e, r0);
        r1 = fmaf(clamp_log_alpha(x1), kLog2e, r1);
        g0[i] = r0;
        g1[i] = r1;
    }
    b.csum[tg * 128 + c] = r0;
    b.csum[tg * 128 + c + 1] = r1;
    if (pt == 0) *b.slow_flag = 0u;
    named_barrier(BAR, kGroupThreads);
    if (layer && katom == 0) {   // one lane per (token, k / q): the inverse norm
        const int lane = pt & 31;
        const float tot = b.xf[tg * 32 + lane] + b.xf[128 + tg * 32 + lane];
        b.nrm[(lane < 16 ? 0 : 64) + t0 + (lane & 15)] = rsqrtf(tot + b.qk_eps);
    }

    float off0 = 0.f, off1 = 0.f, GL0 = 0.f, GL1 = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float a = b.csum[j * 128 + c], bb = b.csum[j * 128 + c + 1];
        if (j < tg) { off0 += a; off1 += bb; }
        GL0 += a;
        GL1 += bb;
    }
    constexpr float kSlow2 = kSlowPathLogDecay * kLog2e;
    if (tg == 0 && (GL0 < kSlow2 || GL1 < kSlow2)) atomicOr(b.slow_flag, 1u);
    if (r0 < kSlow2 || r1 < kSlow2) atomicOr(b.slow_flag, 2u);   // this 16-token block alone
    named_barrier(BAR, kGroupThreads);
    const uint32_t flag = *b.slow_flag;
    const bool slow = (flag & 1u) != 0u;

    const float eL0 = exp2_f(GL0), eL1 = exp2_f(GL1);
    if (tg == 0) {
        b.egl[c] = eL0;
        b.egl[c + 1] = eL1;
    }
    constexpr float kMaxInv2 = 80.f * kLog2e;   // Khat's factor is capped at e^80
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int t = t0 + i;
        const __nv_bfloat162 kv = *reinterpret_cast<const __nv_bfloat162 *>(&k_v[i]);
        const __nv_bfloat162 qv = *reinterpret_cast<const __nv_bfloat162 *>(&q_v[i]);
        const float nk = scaled ? b.nrm[t] : 1.f, nq = scaled ? b.nrm[64 + t] : 1.f;
        const float k0 = __low2float(kv) * nk, k1 = __high2float(kv) * nk;
        const float q0 = __low2float(qv) * nq, q1 = __high2float(qv) * nq;
        const float G0 = g0[i] + off0, G1 = g1[i] + off1;
        if (GOUT) *reinterpret_cast<float2 *>(b.gout + t * 128 + c) = make_float2(G0, G1);
        const float e0 = exp2_f(G0), e1 = exp2_f(G1);
        const float ih0 = exp2_f(fminf(-G0, kMaxInv2)), ih1 = exp2_f(fminf(-G1, kMaxInv2));
        // Kbar's factor e^{G_L - G}: a product of two factors, or (pairwise
        // path, where e^{-G} may be capped) one exponential
        const float b0 = slow ? exp2_f(GL0 - G0) : eL0 * ih0;
        const float b1 = slow ? exp2_f(GL1 - G1) : eL1 * ih1;
        const uint32_t ok = sw128_off(t, cc);
        *reinterpret_cast<uint32_t *>(stack + ok) = pack_bf16x2(k0 * e0, k1 * e1);
        *reinterpret_cast<uint32_t *>(stack + sw128_off(64 + t, cc)) = pack_bf16x2(q0 * e0, q1 * e1);
        *reinterpret_cast<uint32_t *>(khat + ok) = pack_bf16x2(k0 * ih0, k1 * ih1);
        *reinterpret_cast<uint32_t *>(kbar + ok) = pack_bf16x2(k0 * b0, k1 * b1);
    }
    return !slow ? kProductForm : ((flag & 2u) ? kPairwise : kSecondary);
}

// ---- the same for a scalar gate (b.gsc: one log_alpha per token, every
// channel decaying alike).  The running sums and the factors e^{G_t},
// e^{-G_t} and e^{G_L - G_t} are per token, so they are formed once per token
// (64 exponentials of each kind instead of one per element) and every thread
// only scales its elements.  Each sum and factor is taken by the very
// operations, in the same order, that gate() applies per channel, so the
// operands equal those of the per-channel gate fed the scalar repeated over
// the channels, bit for bit.  A chunk that takes a slow path also gets the
// gate spread over the channels in b.graw and the 16-token block sums in
// b.csum, which those paths read.  Scratch: b.xf (the solve's, free here).
template <int BAR, bool GOUT = false>
__device__ int gate_scalar(const Bufs &b, int pt, int L) {
    const int c = 2 * (pt & 63);
    const int tg = pt >> 6;
    const int t0 = tg * 16;
    const int katom = c >> 6, cc = c & 63;
    uint8_t *stack = b.stk + katom * 16384;
    uint8_t *khat = b.khat + katom * 8192;
    uint8_t *kbar = b.kbar + katom * 8192;
    float *part = b.xf;                                        // [64] sums within each block
    float *bsum = b.xf + 64;                                   // [4] block sums
    float4 *fac = reinterpret_cast<float4 *>(b.xf + 128);     // [64] (e^G, e^-G, Kbar's factor, -)

    if (L < C) {   // rows past the chunk's end: zero operand rows (uniform over the group)
        for (int v = pt; v < (C - L) * 16; v += kGroupThreads) {
            const int t = L + (v >> 4), piece = v & 15;
            const uint4 z = make_uint4(0u, 0u, 0u, 0u);
            uint8_t *atom = b.stk + (piece >> 3) * 16384;
            *reinterpret_cast<uint4 *>(atom + sw128_off(t, (piece & 7) * 8)) = z;
            *reinterpret_cast<uint4 *>(atom + sw128_off(64 + t, (piece & 7) * 8)) = z;
        }
    }
    if (pt < 4) {   // block pt's running sum, in token order from zero (base-2 units)
        float r = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            r = fmaf(clamp_log_alpha(b.gsc[16 * pt + i]), kLog2e, r);
            part[16 * pt + i] = r;
        }
        bsum[pt] = r;
    }
    if (pt == 0) *b.slow_flag = 0u;
    named_barrier(BAR, kGroupThreads);
    constexpr float kSlow2 = kSlowPathLogDecay * kLog2e;
    float GL = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) GL += bsum[j];
    const bool slow = GL < kSlow2;
    bool pairwise = false;
#pragma unroll
    for (int j = 0; j < 4; ++j) pairwise |= bsum[j] < kSlow2;
    const float eL = exp2_f(GL);
    constexpr float kMaxInv2 = 80.f * kLog2e;   // Khat's factor is capped at e^80
    if (pt < C) {   // token pt's factors
        const int j = pt >> 4;
        float off = 0.f;
#pragma unroll
        for (int jj = 0; jj < 3; ++jj)
            if (jj < j) off += bsum[jj];
        const float G = part[pt] + off;
        if (GOUT) b.gout[pt] = G;   // one running sum per token (base-2 units)
        const float ih = exp2_f(fminf(-G, kMaxInv2));
        fac[pt] = make_float4(exp2_f(G), ih, slow ? exp2_f(GL - G) : eL * ih, 0.f);
    }
    if (pt < 128) b.egl[pt] = eL;
    if (slow) {   // what the slow paths read: the gate per channel and the block sums
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const __nv_bfloat16 gv = __float2bfloat16_rn(b.gsc[t0 + i]);   // exact: a bf16 value
            *reinterpret_cast<__nv_bfloat162 *>(const_cast<uint8_t *>(b.graw) + (t0 + i) * 256 + c * 2) =
                __halves2bfloat162(gv, gv);
        }
        b.csum[tg * 128 + c] = bsum[tg];
        b.csum[tg * 128 + c + 1] = bsum[tg];
    }
    named_barrier(BAR, kGroupThreads);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int t = t0 + i;
        const float4 f = fac[t];
        const __nv_bfloat162 kv = *reinterpret_cast<const __nv_bfloat162 *>(stack + sw128_off(t, cc));
        const __nv_bfloat162 qv = *reinterpret_cast<const __nv_bfloat162 *>(stack + sw128_off(64 + t, cc));
        const float k0 = __low2float(kv), k1 = __high2float(kv);
        const float q0 = __low2float(qv), q1 = __high2float(qv);
        const uint32_t ok = sw128_off(t, cc);
        *reinterpret_cast<uint32_t *>(stack + ok) = pack_bf16x2(k0 * f.x, k1 * f.x);
        *reinterpret_cast<uint32_t *>(stack + sw128_off(64 + t, cc)) = pack_bf16x2(q0 * f.x, q1 * f.x);
        *reinterpret_cast<uint32_t *>(khat + ok) = pack_bf16x2(k0 * f.y, k1 * f.y);
        *reinterpret_cast<uint32_t *>(kbar + ok) = pack_bf16x2(k0 * f.z, k1 * f.z);
    }
    return !slow ? kProductForm : (pairwise ? kPairwise : kSecondary);
}

// ---- secondary chunking, for a chunk that decays too fast for one reference
// but not within any 16-token block.  For each column block bb, with the
// running sum just before the block as reference (off_bb, per channel), the
// rows t >= 16 bb scaled by e^{G_t - off_bb} (<= 1) and the block's columns
// by e^{off_bb - G_i} (<= e^80) give columns 16 bb .. + 15 of
// [Ktil Khat^T; Qtil Khat^T] as one M = 128, N = 16 product; rows above the
// block hold leftovers of earlier blocks, which the read-out masks.  The four
// products fill the TMEM columns the one-reference product does, so the same
// read-out follows.  Operand tiles: rows [k; q] in two K-atoms at opa0 and
// opa1 (16 KB each), the block's columns in two 2 KB K-atoms at opc; raw g
// is read from b.graw before opa1 may overwrite it; raw k and q come from
// global memory (kt0 / qt0, as for the pairwise path).  `round` counts the
// phases of `bar` across calls.
template <int BAR>
__device__ void secondary(const Bufs &b, int pt, int L, const __nv_bfloat16 *kt0,
                          const __nv_bfloat16 *qt0, size_t row_stride, uint8_t *opa0,
                          uint8_t *opa1, uint8_t *opc, uint32_t tmem_ap, bool issue_warp,
                          uint64_t *bar, uint32_t &round, volatile uint32_t *abort) {
    const int c = 2 * (pt & 63);
    const int tg = pt >> 6;
    const int t0 = tg * 16;
    const int katom = c >> 6, cc = c & 63;
    uint8_t *atom_a = katom ? opa1 : opa0;
    uint8_t *atom_c = opc + katom * 2048;
    float G0[16], G1[16];
    {
        float r0 = 0.f, r1 = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const __nv_bfloat162 gv =
                *reinterpret_cast<const __nv_bfloat162 *>(b.graw + (t0 + i) * 256 + c * 2);
            r0 = fmaf(clamp_log_alpha(__low2float(gv)), kLog2e, r0);
            r1 = fmaf(clamp_log_alpha(__high2float(gv)), kLog2e, r1);
            G0[i] = r0;
            G1[i] = r1;
        }
    }
    float off0[4], off1[4];   // running sum before each block
    off0[0] = off1[0] = 0.f;
#pragma unroll
    for (int j = 1; j < 4; ++j) {
        off0[j] = off0[j - 1] + b.csum[(j - 1) * 128 + c];
        off1[j] = off1[j - 1] + b.csum[(j - 1) * 128 + c + 1];
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        G0[i] += off0[tg];
        G1[i] += off1[tg];
    }
    uint32_t kv[16], qv[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int t = t0 + i;
        kv[i] = t < L ? *reinterpret_cast<const uint32_t *>(kt0 + (size_t)t * row_stride + c) : 0u;
        qv[i] = t < L ? *reinterpret_cast<const uint32_t *>(qt0 + (size_t)t * row_stride + c) : 0u;
    }
    named_barrier(BAR, kGroupThreads);   // raw g read everywhere before opa1 is written
    for (int bb = 0; bb < 4; ++bb) {
        const float ob0 = off0[bb], ob1 = off1[bb];
        if (tg >= bb) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int t = t0 + i;
                const __nv_bfloat162 k2 = *reinterpret_cast<const __nv_bfloat162 *>(&kv[i]);
                const __nv_bfloat162 q2 = *reinterpret_cast<const __nv_bfloat162 *>(&qv[i]);
                const float nk = b.nrm ? b.nrm[t] : 1.f, nq = b.nrm ? b.nrm[64 + t] : 1.f;
                const float e0 = exp2_f(G0[i] - ob0), e1 = exp2_f(G1[i] - ob1);
                *reinterpret_cast<uint32_t *>(atom_a + sw128_off(t, cc)) =
                    pack_bf16x2(__low2float(k2) * (e0 * nk), __high2float(k2) * (e1 * nk));
                *reinterpret_cast<uint32_t *>(atom_a + sw128_off(64 + t, cc)) =
                    pack_bf16x2(__low2float(q2) * (e0 * nq), __high2float(q2) * (e1 * nq));
                if (tg == bb) {
                    const float f0 = exp2_f(ob0 - G0[i]), f1 = exp2_f(ob1 - G1[i]);
                    *reinterpret_cast<uint32_t *>(atom_c + sw128_off(i, cc)) =
                        pack_bf16x2(__low2float(k2) * (f0 * nk), __high2float(k2) * (f1 * nk));
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        named_barrier(BAR, kGroupThreads);
        if (issue_warp) {
            tc_fence_after();
            const uint32_t a0 = smem_addr(opa0), a1 = smem_addr(opa1), c0 = smem_addr(opc);
            const uint32_t id = idesc_bf16(128, 16, false, false);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16_warp(tmem_ap + 16 * bb,
                              smem_desc((ks >> 2 ? a1 : a0) + (ks & 3) * 32, 16, 1024, kLayoutSW128),
                              smem_desc(c0 + (ks >> 2) * 2048 + (ks & 3) * 32, 16, 1024, kLayoutSW128),
                              id, ks > 0 ? 1u : 0u);
            mma_commit_warp(bar);
        }
        mbar_wait(bar, round & 1u, abort);   // this block's operands are free again
        ++round;
        tc_fence_after();
    }
}

// 32 consecutive bf16 of a global row as fp32 (zeros when !valid).
__device__ __forceinline__ void load_row32(const __nv_bfloat16 *src, float (&v)[32], bool valid) {
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
// product form (a factor e^{-G} would overflow).  A quad of lanes (four
// groups of 32 channels) owns column i and walks the rows t = i .. 63 in
// order, carrying d = G_t - G_i (the sum of log_alpha over tokens i+1 .. t,
// base-2 units) per channel, so every exponent is a difference of running
// sums taken in fp32 and is <= 0; the quad's partial sums are combined with
// shuffles.  Raw k and q rows come from global memory (kt0 / qt0: token 0 of
// the chunk for this head; row_stride is H * d_k elements).  All lanes of a
// warp walk the same rows (from the warp's first column), so the shuffles
// stay converged.
__device__ inline void pairwise(const Bufs &b, int pt, int L, const __nv_bfloat16 *kt0,
                         const __nv_bfloat16 *qt0, size_t row_stride) {
    const int i = pt >> 2, cg = pt & 3, c0 = 32 * cg;
    const bool lead = cg == 0;
    const int t_first = (pt >> 5) * 8;   // the warp's first column
    float ki[32], d[32];
    load_row32(kt0 + (size_t)i * row_stride + c0, ki, i < L);
#pragma unroll
    for (int c = 0; c < 32; ++c) d[c] = 0.f;
    if (lead) {   // rows above the diagonal
        for (int t = 0; t < i; ++t) {
            b.af[fidx(t, i)] = 0.f;
            *reinterpret_cast<__nv_bfloat16 *>(b.pb + sw128_off(t, i)) = __float2bfloat16_rn(0.f);
        }
    }
    for (int t = t_first; t < C; ++t) {
        const bool active = t >= i;
        if (t > i) {   // d += log_alpha of token t (rows past the chunk end are zero)
            const uint4 *gr = reinterpret_cast<const uint4 *>(b.graw + t * 256 + c0 * 2);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 w = gr[q];
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const __nv_bfloat162 h2 = *reinterpret_cast<const __nv_bfloat162 *>(&ww[e]);
                    d[8 * q + 2 * e] = fmaf(clamp_log_alpha(__low2float(h2)), kLog2e, d[8 * q + 2 * e]);
                    d[8 * q + 2 * e + 1] =
                        fmaf(clamp_log_alpha(__high2float(h2)), kLog2e, d[8 * q + 2 * e + 1]);
                }
            }
        }
        float kt[32], qt[32];
        load_row32(kt0 + (size_t)t * row_stride + c0, kt, active && t < L);
        load_row32(qt0 + (size_t)t * row_stride + c0, qt, active && t < L);
        float a = 0.f, pq = 0.f;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
            const float w = ki[c] * exp2_f(d[c]);
            a = fmaf(kt[c], w, a);
            pq = fmaf(qt[c], w, pq);
        }
        a += __shfl_xor_sync(0xffffffffu, a, 1);
        a += __shfl_xor_sync(0xffffffffu, a, 2);
        pq += __shfl_xor_sync(0xffffffffu, pq, 1);
        pq += __shfl_xor_sync(0xffffffffu, pq, 2);
        if (lead && active) {
            if (b.nrm) {   // the dot products of the raw rows, scaled to the normalised ones
                a *= b.nrm[t] * b.nrm[i];
                pq *= b.nrm[64 + t] * b.nrm[i];
            }
            b.af[fidx(t, i)] = (t > i) ? b.beta[t] * a : 0.f;
            *reinterpret_cast<__nv_bfloat16 *>(b.pb + sw128_off(t, i)) = __float2bfloat16_rn(pq);
        }
    }
}

// ---- [A; P] from TMEM.  A warp of TMEM quadrant `quad` (lanes 32 quad ..)
// reads 32 of the 64 columns (`half`): rows 0-63 are Ktil Khat^T -> A (fp32,
// beta-scaled, strictly lower), rows 64-127 are Qtil Khat^T -> P (bf16, lower).
__device__ __forceinline__ void read_ap(const Bufs &b, uint32_t tmem_ap, int quad, int half,
                                        int lane) {
    float v[32];
    tmem_ld32(tmem_addr(tmem_ap, 32 * quad, 32 * half), v);
    tmem_wait_ld();
    if (quad < 2) {
        const int t = 32 * quad + lane;
        const float bt = b.beta[t];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int i = 32 * half + j;
            b.af[fidx(t, i)] = (i < t) ? bt * v[j] : 0.f;
        }
    } else {
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
            *reinterpret_cast<uint4 *>(b.pb + sw128_off(t, 32 * half + j)) = pk;
        }
    }
}

// ---- one merge level of the recursive-doubling inverse: neighbouring M x M
// lower-triangular inverses T1, T2 become [[T1, 0], [T21, T2]] with
// T21 = -T2 (A21 T1).  1x4 row segments per thread; warps share a column
// group (first product) or a row group (second product) so that the loops
// skip the triangular zeros.
template <int M, int BAR>
__device__ __forceinline__ void merge(const float *__restrict__ AF, float *__restrict__ TF,
                                      float *__restrict__ XF, int pt) {
    constexpr int kThr = 8 * M;
    constexpr int SEG = M / 4;
    constexpr int PER = M * SEG;
    constexpr int XS = M + 4;
    if (pt < kThr) {   // X = A21 T1
        const int merge_id = pt / PER, rem = pt % PER;
        const int c4 = (rem / M) * 4, r = rem % M;
        const int base = merge_id * 2 * M;
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
        *reinterpret_cast<float4 *>(&XF[(merge_id * M + r) * XS + c4]) = acc;
    }
    named_barrier(BAR, kGroupThreads);
    if (pt < kThr) {   // T21 = -T2 X
        const int merge_id = pt / PER, rem = pt % PER;
        const int r = rem / SEG, c4 = (rem % SEG) * 4;
        const int base = merge_id * 2 * M;
        const int rlast = (pt | 31) % PER / SEG;
        const int kend = (M >= 16) ? ((rlast >> 2) + 1) * 4 : M;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int k4 = 0; k4 < kend; k4 += 4) {
            const float4 tr = *reinterpret_cast<const float4 *>(&TF[tfi(base + M + r, base + M + k4)]);
            const float tk[4] = {tr.x, tr.y, tr.z, tr.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float4 xv =
                    *reinterpret_cast<const float4 *>(&XF[(merge_id * M + k4 + e) * XS + c4]);
                acc.x = fmaf(tk[e], xv.x, acc.x);
                acc.y = fmaf(tk[e], xv.y, acc.y);
                acc.z = fmaf(tk[e], xv.z, acc.z);
                acc.w = fmaf(tk[e], xv.w, acc.w);
            }
        }
        *reinterpret_cast<float4 *>(&TF[tfi(base + M + r, base + c4)]) =
            make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
    }
    named_barrier(BAR, kGroupThreads);
}

// ---- T = (I + A)^-1: the 16 x 16 diagonal blocks by forward substitution,
// then recursive doubling (merges at 16 and 32); writes T diag(beta) as bf16
// into b.tb.  Starts and ends with every
// thread of the group past a barrier on its buffers.
template <int BAR>
__device__ void solve(const Bufs &b, int pt) {
    const float *__restrict__ AF = b.af;
    float *__restrict__ TF = b.tf;
    float *__restrict__ XF = b.xf;
    if (pt < 64) {
        // The four 16 x 16 diagonal blocks of T, one column per lane (two warps,
        // a half-warp per block), by forward substitution in fp32: for rows
        // i > j of column j, x_i = -sum_{k < i} A_ik x_k with x_j = 1 and
        // x_k = 0 above it.  The half-warp's lanes read the same A element at
        // once (a broadcast), and only the last term of each row waits for the
        // row before.
        const int b0 = 16 * (pt >> 4), j = pt & 15;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = (i == j) ? 1.f : 0.f;
#pragma unroll
        for (int i = 1; i < 16; ++i) {
            float acc = 0.f;
#pragma unroll
            for (int k = 0; k < i; ++k) acc = fmaf(AF[fidx(b0 + i, b0 + k)], x[k], acc);
            if (i > j) x[i] = -acc;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) TF[tfi(b0 + i, b0 + j)] = x[i];
    } else {   // zero outside the 16 x 16 diagonal blocks
        for (int v = pt - 64; v < 768; v += kGroupThreads - 64) {
            const int row = v / 12, g = v % 12;               // 12 float4 off the block per row
            const int g4 = g + (g >= 4 * (row >> 4) ? 4 : 0);  // skip the row's diagonal block
            *reinterpret_cast<float4 *>(&TF[tfi(row, 4 * g4)]) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    named_barrier(BAR, kGroupThreads);
    merge<16, BAR>(AF, TF, XF, pt);
    merge<32, BAR>(AF, TF, XF, pt);

    const int t = pt >> 2, i0 = (pt & 3) * 16;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const float4 u0 = *reinterpret_cast<const float4 *>(&TF[tfi(t, i0 + 8 * hh)]);
        const float4 u1 = *reinterpret_cast<const float4 *>(&TF[tfi(t, i0 + 8 * hh + 4)]);
        const float *bb = b.beta + i0 + 8 * hh;
        uint4 pk;
        pk.x = pack_bf16x2(u0.x * bb[0], u0.y * bb[1]);
        pk.y = pack_bf16x2(u0.z * bb[2], u0.w * bb[3]);
        pk.z = pack_bf16x2(u1.x * bb[4], u1.y * bb[5]);
        pk.w = pack_bf16x2(u1.z * bb[6], u1.w * bb[7]);
        *reinterpret_cast<uint4 *>(b.tb + sw128_off(t, i0 + 8 * hh)) = pk;
    }
}

}  // namespace prep
}  // namespace kda
