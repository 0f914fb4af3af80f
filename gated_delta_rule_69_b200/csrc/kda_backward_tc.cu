// Chunk-local gradients of the KDA backward pass on the tensor cores (bf16,
// d_k = d_v = 128, C = 64).
//
// The backward pass runs in three stages (the prefill's own chunk algebra,
// news digest page on Kimi Linear, section "Algorithme parallele par chunks"):
// the chunk records, a forward scan for each chunk's entering state S and a
// reverse scan for dL/dS at each chunk's end (dS_C), both on the tensor cores
// (kda_prefill_split.cu).  This file holds the third: with S and dS_C known,
// every (chunk, head) item is independent, and its gradients are products of
// 64 x 64 and 64 x 128 matrices.  Per item, with the gated operands of the
// prefill (Ktil = K e^G, Qtil = Q e^G, Khat = K e^-G, Kbar = K e^{G_L - G}),
// A = strict_tril(diag(beta) Ktil Khat^T) (KK = Ktil Khat^T unscaled),
// T = (I + A)^-1, T_beta = T diag(beta), P = tril(Qtil Khat^T):
//
//   R = V - Ktil S,           U = T_beta R            (the forward's values)
//   dU = Kbar dS_C + P^T dO,  dR = T_beta^T dU = dL/dV
//   dT_beta = dU R^T,         dbeta_i += sum_t dT_beta[t][i] T[t][i]
//   dT = dT_beta diag(beta),  dA = -strict_tril(T^T (dT T^T))
//   dbeta_t += sum_i dA[t][i] KK[t][i]
//   dP = tril(dO U^T)
//   dQtil = dO S^T + dP Khat,          dKtil = -dR S^T + diag(beta) dA Khat
//   dKhat = dP^T Qtil + (diag(beta) dA)^T Ktil,       dKbar = U dS_C^T
//   dq = dQtil e^G,   dk = dKtil e^G + dKhat e^-G + dKbar e^{G_L - G}
//   dG = dKtil.Ktil + dQtil.Qtil - dKhat.Khat - dKbar.Kbar
//   dg_t = sum_{s >= t} dG_s + sum_s dKbar.Kbar|_s + e^{G_L} rowsum(S .* dS_C)
//
// Five rounds of products, each one commit: {Ktil S, dU}, {U, dR, dT_beta},
// {dKbar, dP, dT T^T, [dO; -dR] S^T}, {T^T Z}, {[dP; BdA] Khat, dKhat}.  A
// round's results are read from TMEM by the warps of quadrants 0 and 1 (rows
// 0-63; the M = 128 products' rows 64-127 multiply whatever follows an
// operand in shared memory and are not read), converted to bf16 tiles and
// fed to the next round.  Two products are stacked to fill all 128 rows:
// [dO; -dR] S^T and [dP; BdA] Khat accumulate into one TMEM tile whose rows
// 0-63 are dQtil and rows 64-127 dKtil.
//
// A chunk that decays below e^-80 within itself on some channel (the
// prefill's slow forms: Khat's factor would overflow) is left to the
// token-by-token kernel of kda_backward.cu, through a per-item flag.
#include <cuda.h>

#include "kda_chunk_prep.cuh"
#include "kda_internal.cuh"
#include "kda_sm100.cuh"

namespace kda {

bool make_bf16_map_3d(CUtensorMap *m, const void *base, int64_t T, int H, int inner, int box_inner,
                      CUtensorMapSwizzle sw);

namespace bwdtc {

using namespace sm100;

constexpr int C = 64;
constexpr int DK = 128;
constexpr int kThreads = 256;
constexpr uint32_t BAR = 1;   // named barrier of the CTA's 256 threads

// Shared memory (bytes; tiles bf16, K-major, 128-byte swizzle, 64 columns per
// K-atom).  Phase A (the prefill's preparation: gating, [A; P], the solve)
// and phase B (the products) share the region from AF on.
struct Sm {
    static constexpr uint32_t STK = 0;         // [Ktil rows 0-63 | Qtil rows 64-127], 2 x 16 KB
    static constexpr uint32_t KHAT = 32768;    // Khat [64 t][128 c], 2 x 8 KB
    static constexpr uint32_t TB = 49152;      // T_beta [64 t][64 i], then Z
    static constexpr uint32_t TB16 = 57344;    // T [64 t][64 i]
    static constexpr uint32_t KBAR = 65536;    // Kbar [64][128], then R, then PA = [dP; BdA] [128][64]
    static constexpr uint32_t PB = 81920;      // P [64 t][64 i], then dT
    // phase A
    static constexpr uint32_t AF = 90112;      // A fp32, rows of 65
    static constexpr uint32_t TF = 107520;     // T fp32, rows of 68
    static constexpr uint32_t GRAW = 124928;   // raw log_alpha [64][128] bf16
    static constexpr uint32_t XF = 141312;     // solve scratch (4608 bytes)
    // phase B
    // (dU and U serve as M = 128 A operands whose rows 64-127 read the 8 KB
    // after each K-atom: each is followed by another tile, not by the end)
    static constexpr uint32_t S0 = 90112;      // S [128 c][128 j], 2 x 16 KB; then the final exchange
    static constexpr uint32_t DOR = 122880;    // [dO rows 0-63 | -dR rows 64-127] [128][128], 2 x 16 KB
    static constexpr uint32_t DU = 155648;     // dU [64 t][128 j], 2 x 8 KB
    static constexpr uint32_t U = 172032;      // U [64 t][128 j], 2 x 8 KB
    static constexpr uint32_t DSC = 188416;    // dS_C [128 c][128 j], 2 x 16 KB
    static constexpr uint32_t XCH = S0;        // fp32 [64 t][128 c] (32 KB), 16-byte pieces swizzled
    static constexpr uint32_t BETA = 221184;   // 64 fp32
    static constexpr uint32_t EGL = 221440;    // 128 fp32: e^{G_L}
    static constexpr uint32_t CSUM = 221952;   // 4 x 128 fp32
    static constexpr uint32_t DB = 224000;     // 64 fp32: dbeta of the item
    static constexpr uint32_t DGL = 224256;    // 128 fp32: column sums of dKbar.Kbar
    static constexpr uint32_t ES = 224768;     // 128 fp32: rowsum(S .* dS_C)
    static constexpr uint32_t BARS = 225280;   // mbarriers: raw loads, dO, products
    static constexpr uint32_t MISC = 225344;   // tmem base, abort, slow flag
    static constexpr uint32_t SIZE = 225408;
    static constexpr uint32_t ALLOC = SIZE + 1024;
};
static_assert(Sm::ALLOC <= 232448, "shared memory");
static_assert(Sm::AF + 64 * prep::kAStride * 4 <= Sm::TF && Sm::TF + 64 * prep::kTStride * 4 <= Sm::GRAW &&
                  Sm::GRAW + 16384 <= Sm::XF && Sm::XF + 4608 <= Sm::DU,
              "phase A buffers");
static_assert(Sm::DU + 16384 == Sm::U && Sm::U + 16384 == Sm::DSC && Sm::DSC + 32768 <= Sm::BETA &&
                  Sm::XCH + 32768 <= Sm::GRAW,
              "phase B buffers");

// TMEM columns (512): [A; P] (KK in rows 0-63) until round 3; the stacked
// [dQtil; dKtil]; then per round the products listed.
constexpr uint32_t kColAP = 0;
constexpr uint32_t kColD1 = 64;     // rows 0-63 dQtil, 64-127 dKtil
constexpr uint32_t kColX = 192;     // Ktil S (round 0), U (1), dKbar (2 - end)
constexpr uint32_t kColY = 320;     // dU (0), dR (1), dP (2, 64 cols), dKhat (4 - end)
constexpr uint32_t kColZ = 384;     // Z (2, 64 cols)
constexpr uint32_t kColW = 448;     // dT_beta (1), T^T Z (3)

struct Args {
    const __nv_bfloat16 *q, *k, *v, *g, *beta, *d_o;
    const float *s_in, *ds_next;     // [record][128][128] fp32, record = chunk * H + head
    const int2 *chunk_tab;
    const uint32_t *total_chunks;
    float *dq, *dk, *dv, *dg, *dbeta;
    uint32_t *slow;                  // [record]: 1 where the item is left to the step kernel
    float *gscr;                     // [grid][64][128] fp32: the running sums of the CTA's item
    uint32_t *err_word;
    int H;
};

__device__ __forceinline__ uint4 pack8(const float *v) {
    uint4 pk;
    pk.x = pack_bf16x2(v[0], v[1]);
    pk.y = pack_bf16x2(v[2], v[3]);
    pk.z = pack_bf16x2(v[4], v[5]);
    pk.w = pack_bf16x2(v[6], v[7]);
    return pk;
}

// 32 bf16 of a row of a K-major tile (columns col .. col + 31 of one K-atom)
__device__ __forceinline__ void put32(uint8_t *atom, int row, int col, const float (&v)[32]) {
#pragma unroll
    for (int j = 0; j < 32; j += 8)
        *reinterpret_cast<uint4 *>(atom + sw128_off(row, col + j)) = pack8(v + j);
}

__device__ __forceinline__ void get32(const uint8_t *atom, int row, int col, float (&v)[32]) {
#pragma unroll
    for (int j = 0; j < 32; j += 8) {
        const uint4 w = *reinterpret_cast<const uint4 *>(atom + sw128_off(row, col + j));
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 h2 = *reinterpret_cast<const __nv_bfloat162 *>(&ww[e]);
            v[j + 2 * e] = __low2float(h2);
            v[j + 2 * e + 1] = __high2float(h2);
        }
    }
}

// 32 consecutive bf16 of global memory as fp32 (zeros when !valid)
__device__ __forceinline__ void gload32(const __nv_bfloat16 *src, bool valid, float (&v)[32]) {
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        if (valid) w = reinterpret_cast<const uint4 *>(src)[q4];
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 h2 = *reinterpret_cast<const __nv_bfloat162 *>(&ww[e]);
            v[8 * q4 + 2 * e] = __low2float(h2);
            v[8 * q4 + 2 * e + 1] = __high2float(h2);
        }
    }
}

// fp32 [64 t][128 c] exchange tile: 16-byte piece p of row t at piece p ^ (t mod 32)
__device__ __forceinline__ float4 *xch_at(uint8_t *sm, int t, int piece) {
    return reinterpret_cast<float4 *>(sm + Sm::XCH + t * 512 + ((piece ^ (t & 31)) << 4));
}

// Sums v[j] over the warp's 32 lanes for j = 0..31; lane l returns the sum of v[l].
__device__ __forceinline__ float column_sums(float (&v)[32], int lane) {
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
    return v[0];
}

__device__ __forceinline__ void issue_raw(uint8_t *sm, uint64_t *bar, const CUtensorMap &tm_k,
                                          const CUtensorMap &tm_q, const CUtensorMap &tm_g, const Args &p,
                                          uint32_t item) {
    const int h = (int)(item % (uint32_t)p.H);
    const int t = p.chunk_tab[item / (uint32_t)p.H].x;
    mbar_arrive_expect_tx(bar, 4 * 8192 + 16384);
    tma_load_3d(sm + Sm::STK, &tm_k, bar, 0, h, t);
    tma_load_3d(sm + Sm::STK + 16384, &tm_k, bar, 64, h, t);
    tma_load_3d(sm + Sm::STK + 8192, &tm_q, bar, 0, h, t);
    tma_load_3d(sm + Sm::STK + 16384 + 8192, &tm_q, bar, 64, h, t);
    tma_load_3d(sm + Sm::GRAW, &tm_g, bar, 0, h, t);
}

__global__ void __launch_bounds__(kThreads, 1)
kda_bwd_chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_do,
                        const Args p) {
    extern __shared__ uint8_t dyn_smem[];
    uint8_t *sm = dyn_smem + ((1024u - (smem_addr(dyn_smem) & 1023u)) & 1023u);
    const int pt = threadIdx.x, warp = pt >> 5, lane = pt & 31;
    const int quad = warp & 3, half = warp >> 2;
    const bool leader = pt == 0;
    uint64_t *BLD = reinterpret_cast<uint64_t *>(sm + Sm::BARS);
    uint64_t *BDO = BLD + 1, *BMMA = BLD + 2;
    uint32_t *misc = reinterpret_cast<uint32_t *>(sm + Sm::MISC);
    volatile uint32_t *abort_flag = misc + 1;
    float *beta = reinterpret_cast<float *>(sm + Sm::BETA);
    float *egl = reinterpret_cast<float *>(sm + Sm::EGL);
    float *db = reinterpret_cast<float *>(sm + Sm::DB);
    float *dgl = reinterpret_cast<float *>(sm + Sm::DGL);
    float *es = reinterpret_cast<float *>(sm + Sm::ES);
    if (leader) {
        mbar_init(BLD, 3);   // the leader's copies, one arrive per beta warp
        mbar_init(BDO, 1);
        mbar_init(BMMA, 1);
        misc[1] = 0u;
        fence_mbar_init();
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_g);
        tma_prefetch_desc(&tm_do);
    }
    if (warp == 0) {
        tmem_alloc(&misc[0], 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    const uint32_t total = *p.total_chunks * (uint32_t)p.H;
    float *gscr = p.gscr + (size_t)blockIdx.x * (C * DK);
    uint32_t n_mma = 0, n_do = 0;   // completed phases of BMMA, BDO
    auto mma_wait = [&]() {
        mbar_wait(BMMA, n_mma & 1u, abort_flag);
        ++n_mma;
        tc_fence_after();
    };
    // round end: this thread's tiles and TMEM reads before the next products
    auto round_barrier = [&]() {
        fence_async_smem();
        tc_fence_before();
        named_barrier(BAR, kThreads);
    };

    if (leader && blockIdx.x < total) issue_raw(sm, BLD, tm_k, tm_q, tm_g, p, blockIdx.x);
#pragma unroll 1
    for (uint32_t item = blockIdx.x, it = 0; item < total; item += gridDim.x, ++it) {
        const int h = (int)(item % (uint32_t)p.H);
        const uint32_t chunk = item / (uint32_t)p.H;
        const int2 ct = p.chunk_tab[chunk];
        const int64_t tok0 = ct.x;
        const int L = ct.y;
        const uint32_t next = item + gridDim.x;
        if (pt < C) {
            beta[pt] = pt < L ? __bfloat162float(p.beta[(size_t)(tok0 + pt) * p.H + h]) : 0.f;
            db[pt] = 0.f;
            __syncwarp();
            if (lane == 0) mbar_arrive(BLD);
        } else if (pt < C + 128) {
            dgl[pt - C] = 0.f;
        }
        prep::Bufs b = {};
        b.stk = sm + Sm::STK;
        b.khat = sm + Sm::KHAT;
        b.kbar = sm + Sm::KBAR;
        b.graw = sm + Sm::GRAW;
        b.af = reinterpret_cast<float *>(sm + Sm::AF);
        b.tf = reinterpret_cast<float *>(sm + Sm::TF);
        b.xf = reinterpret_cast<float *>(sm + Sm::XF);
        b.tb = sm + Sm::TB;
        b.pb = sm + Sm::PB;
        b.beta = beta;
        b.egl = egl;
        b.csum = reinterpret_cast<float *>(sm + Sm::CSUM);
        b.slow_flag = misc + 2;
        b.gout = gscr;
        mbar_wait(BLD, it & 1u, abort_flag);
        const int form = prep::gate<BAR, false, true>(b, pt, L);
        fence_async_smem();
        named_barrier(BAR, kThreads);
        if (form != prep::kProductForm) {   // left to the step kernel
            if (leader) {
                p.slow[item] = 1u;
                if (next < total) issue_raw(sm, BLD, tm_k, tm_q, tm_g, p, next);
            }
            continue;
        }

        // ---- phase A: [A; P] = [Ktil; Qtil] Khat^T, read-out, T = (I + A)^-1
        const uint32_t aSTK = smem_addr(sm + Sm::STK), aKH = smem_addr(sm + Sm::KHAT);
        const uint32_t aTB = smem_addr(sm + Sm::TB), aT16 = smem_addr(sm + Sm::TB16);
        const uint32_t aKB = smem_addr(sm + Sm::KBAR), aPB = smem_addr(sm + Sm::PB);
        const uint32_t aS0 = smem_addr(sm + Sm::S0), aDOR = smem_addr(sm + Sm::DOR);
        const uint32_t aDSC = smem_addr(sm + Sm::DSC), aDU = smem_addr(sm + Sm::DU);
        const uint32_t aU = smem_addr(sm + Sm::U);
        if (warp == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16_warp(tmem + kColAP, smem_desc(aSTK + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kLayoutSW128),
                              smem_desc(aKH + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024, kLayoutSW128), id,
                              ks > 0 ? 1u : 0u);
            mma_commit_warp(BMMA);
        }
        mma_wait();
        prep::read_ap(b, tmem + kColAP, quad, half, lane);
        tc_fence_before();
        named_barrier(BAR, kThreads);
        prep::solve<BAR>(b, pt);
        {   // T as bf16 (the solve's T_beta mapping), from T in fp32
            const float *TF = b.tf;
            const int t = pt >> 2, i0 = (pt & 3) * 16;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const float4 u0 = *reinterpret_cast<const float4 *>(&TF[prep::tfi(t, i0 + 8 * hh)]);
                const float4 u1 = *reinterpret_cast<const float4 *>(&TF[prep::tfi(t, i0 + 8 * hh + 4)]);
                const float w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
                *reinterpret_cast<uint4 *>(sm + Sm::TB16 + sw128_off(t, i0 + 8 * hh)) = pack8(w);
            }
        }
        named_barrier(BAR, kThreads);   // phase A's fp32 buffers are free

        // ---- phase B inputs: dO by TMA, S and dS_C converted to bf16
        if (leader) {
            mbar_arrive_expect_tx(BDO, 16384);
            tma_load_3d(sm + Sm::DOR, &tm_do, BDO, 0, h, (int)tok0);
            tma_load_3d(sm + Sm::DOR + 16384, &tm_do, BDO, 64, h, (int)tok0);
        }
        {
            const size_t rec = (size_t)chunk * p.H + h;
            const int c = pt >> 1, j0 = (pt & 1) * 64;
            const float4 *s4 = reinterpret_cast<const float4 *>(p.s_in + (rec * DK + c) * 128 + j0);
            const float4 *d4 = reinterpret_cast<const float4 *>(p.ds_next + (rec * DK + c) * 128 + j0);
            uint8_t *sa = sm + Sm::S0 + (pt & 1) * 16384, *da = sm + Sm::DSC + (pt & 1) * 16384;
            float dot = 0.f;
#pragma unroll
            for (int j = 0; j < 64; j += 8) {
                const float4 a0 = s4[j / 4], a1 = s4[j / 4 + 1];
                const float4 b0 = d4[j / 4], b1 = d4[j / 4 + 1];
                const float sv[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                const float dv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) dot = fmaf(sv[e], dv[e], dot);
                *reinterpret_cast<uint4 *>(sa + sw128_off(c, j)) = pack8(sv);
                *reinterpret_cast<uint4 *>(da + sw128_off(c, j)) = pack8(dv);
            }
            dot += __shfl_xor_sync(0xffffffffu, dot, 1);
            if ((pt & 1) == 0) es[c] = dot;
        }
        mbar_wait(BDO, n_do & 1u, abort_flag);
        ++n_do;
        if (L < C) {   // dO rows past the chunk end (the next tokens) read as zero
            for (int v = pt; v < (C - L) * 16; v += kThreads) {
                const int t = L + (v >> 4), piece = v & 15;
                *reinterpret_cast<uint4 *>(sm + Sm::DOR + (piece >> 3) * 16384 + sw128_off(t, (piece & 7) * 8)) =
                    make_uint4(0u, 0u, 0u, 0u);
            }
        }
        round_barrier();

        // ---- round 0: Ktil S (rows 0-63 of [Ktil; Qtil] S), dU = Kbar dS_C + P^T dO
        if (warp == 0) {
            tc_fence_after();
            const uint32_t idKN = idesc_bf16(128, 128, false, true);
            const uint32_t idMN = idesc_bf16(128, 128, true, true);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                mma_bf16_warp(tmem + kColX, smem_desc(aSTK + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kLayoutSW128),
                              smem_desc(aS0 + ks * 2048, 16384, 1024, kLayoutSW128), idKN, ks > 0 ? 1u : 0u);
                mma_bf16_warp(tmem + kColY, smem_desc(aKB + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024, kLayoutSW128),
                              smem_desc(aDSC + ks * 2048, 16384, 1024, kLayoutSW128), idKN, ks > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16_warp(tmem + kColY, smem_desc(aPB + ks * 2048, 8192, 1024, kLayoutSW128),
                              smem_desc(aDOR + ks * 2048, 16384, 1024, kLayoutSW128), idMN, 1u);
            mma_commit_warp(BMMA);
        }
        mma_wait();
        if (quad < 2) {
            const int t = 32 * quad + lane;
            const bool valid = t < L;
            const __nv_bfloat16 *vrow = p.v + ((size_t)(tok0 + t) * p.H + h) * 128;
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                const int j0 = 64 * half + 32 * part;
                float x[32], vv[32];
                tmem_ld32(tmem_addr(tmem + kColX, 32 * quad, j0), x);
                gload32(vrow + j0, valid, vv);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) x[j] = vv[j] - x[j];
                put32(sm + Sm::KBAR + half * 8192, t, 32 * part, x);   // R
                tmem_ld32(tmem_addr(tmem + kColY, 32 * quad, j0), x);
                tmem_wait_ld();
                put32(sm + Sm::DU + half * 8192, t, 32 * part, x);     // dU
            }
        }
        round_barrier();

        // ---- round 1: U = T_beta R, dR = T_beta^T dU, dT_beta = dU R^T
        if (warp == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {   // K = 64 (i, then t)
                mma_bf16_warp(tmem + kColX, smem_desc(aTB + ks * 32, 16, 1024, kLayoutSW128),
                              smem_desc(aKB + ks * 2048, 8192, 1024, kLayoutSW128),
                              idesc_bf16(128, 128, false, true), ks > 0 ? 1u : 0u);
                mma_bf16_warp(tmem + kColY, smem_desc(aTB + ks * 2048, 8192, 1024, kLayoutSW128),
                              smem_desc(aDU + ks * 2048, 8192, 1024, kLayoutSW128),
                              idesc_bf16(128, 128, true, true), ks > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)   // K = 128 (j)
                mma_bf16_warp(tmem + kColW, smem_desc(aDU + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024, kLayoutSW128),
                              smem_desc(aKB + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024, kLayoutSW128),
                              idesc_bf16(128, 64, false, false), ks > 0 ? 1u : 0u);
            mma_commit_warp(BMMA);
        }
        mma_wait();
        if (quad < 2) {
            const int t = 32 * quad + lane;
            const bool valid = t < L;
            float *dvrow = p.dv + ((size_t)(tok0 + t) * p.H + h) * 128;
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                const int j0 = 64 * half + 32 * part;
                float x[32];
                tmem_ld32(tmem_addr(tmem + kColX, 32 * quad, j0), x);
                tmem_wait_ld();
                put32(sm + Sm::U + half * 8192, t, 32 * part, x);        // U
                tmem_ld32(tmem_addr(tmem + kColY, 32 * quad, j0), x);
                tmem_wait_ld();
                if (valid) {
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<float4 *>(dvrow + j0 + j) = make_float4(x[j], x[j + 1], x[j + 2], x[j + 3]);
                }
#pragma unroll
                for (int j = 0; j < 32; ++j) x[j] = -x[j];
                put32(sm + Sm::DOR + half * 16384, 64 + t, 32 * part, x);   // -dR
            }
            {   // dT_beta: columns 32 half .. + 31
                const int i0 = 32 * half;
                float x[32], tv[32];
                tmem_ld32(tmem_addr(tmem + kColW, 32 * quad, i0), x);
                get32(sm + Sm::TB16, t, i0, tv);
                tmem_wait_ld();
                float cs[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) cs[j] = x[j] * tv[j];
                const float s = column_sums(cs, lane);   // over this warp's 32 rows t
                atomicAdd(&db[i0 + lane], s);
#pragma unroll
                for (int j = 0; j < 32; ++j) x[j] *= beta[i0 + j];
                put32(sm + Sm::PB, t, i0, x);   // dT
            }
        }
        round_barrier();

        // ---- round 2: dKbar = U dS_C^T, dP = dO U^T, Z = dT T^T, [dO; -dR] S^T
        if (warp == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {   // K = 128 (j)
                const uint64_t aUk = smem_desc(aU + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024, kLayoutSW128);
                const uint64_t aDk = smem_desc(aDOR + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kLayoutSW128);
                mma_bf16_warp(tmem + kColX, aUk,
                              smem_desc(aDSC + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kLayoutSW128),
                              idesc_bf16(128, 128, false, false), ks > 0 ? 1u : 0u);
                mma_bf16_warp(tmem + kColY, aDk, aUk, idesc_bf16(128, 64, false, false), ks > 0 ? 1u : 0u);
                mma_bf16_warp(tmem + kColD1, aDk,
                              smem_desc(aS0 + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kLayoutSW128),
                              idesc_bf16(128, 128, false, false), ks > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)   // K = 64 (k)
                mma_bf16_warp(tmem + kColZ, smem_desc(aPB + ks * 32, 16, 1024, kLayoutSW128),
                              smem_desc(aT16 + ks * 32, 16, 1024, kLayoutSW128), idesc_bf16(128, 64, false, false),
                              ks > 0 ? 1u : 0u);
            mma_commit_warp(BMMA);
        }
        mma_wait();
        if (quad < 2) {
            const int t = 32 * quad + lane;
            const int i0 = 32 * half;
            float x[32];
            tmem_ld32(tmem_addr(tmem + kColY, 32 * quad, i0), x);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) x[j] = (i0 + j <= t) ? x[j] : 0.f;
            put32(sm + Sm::KBAR, t, i0, x);   // dP, rows 0-63 of PA
            tmem_ld32(tmem_addr(tmem + kColZ, 32 * quad, i0), x);
            tmem_wait_ld();
            put32(sm + Sm::TB, t, i0, x);     // Z
        }
        round_barrier();

        // ---- round 3: T^T Z (dA = -strict_tril of it)
        if (warp == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)   // K = 64 (k)
                mma_bf16_warp(tmem + kColW, smem_desc(aT16 + ks * 2048, 8192, 1024, kLayoutSW128),
                              smem_desc(aTB + ks * 2048, 8192, 1024, kLayoutSW128), idesc_bf16(128, 64, true, true),
                              ks > 0 ? 1u : 0u);
            mma_commit_warp(BMMA);
        }
        mma_wait();
        if (quad < 2) {
            const int t = 32 * quad + lane;
            const int i0 = 32 * half;
            float x[32], kk[32];
            tmem_ld32(tmem_addr(tmem + kColW, 32 * quad, i0), x);
            tmem_ld32(tmem_addr(tmem + kColAP, 32 * quad, i0), kk);
            tmem_wait_ld();
            float s = 0.f;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                x[j] = (i0 + j < t) ? -x[j] : 0.f;   // dA
                s = fmaf(x[j], kk[j], s);
            }
            atomicAdd(&db[t], s);
            const float bt = beta[t];
#pragma unroll
            for (int j = 0; j < 32; ++j) x[j] *= bt;
            put32(sm + Sm::KBAR, 64 + t, i0, x);   // diag(beta) dA, rows 64-127 of PA
        }
        round_barrier();

        // ---- round 4: [dQtil; dKtil] += [dP; BdA] Khat, dKhat = dP^T Qtil + BdA^T Ktil
        if (warp == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)   // K = 64 (i)
                mma_bf16_warp(tmem + kColD1, smem_desc(aKB + ks * 32, 16, 1024, kLayoutSW128),
                              smem_desc(aKH + ks * 2048, 8192, 1024, kLayoutSW128), idesc_bf16(128, 128, false, true),
                              1u);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)   // K = 64 (t)
                mma_bf16_warp(tmem + kColY, smem_desc(aKB + ks * 2048, 8192, 1024, kLayoutSW128),
                              smem_desc(aSTK + 8192 + ks * 2048, 16384, 1024, kLayoutSW128),
                              idesc_bf16(128, 128, true, true), ks > 0 ? 1u : 0u);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16_warp(tmem + kColY, smem_desc(aKB + 8192 + ks * 2048, 8192, 1024, kLayoutSW128),
                              smem_desc(aSTK + ks * 2048, 16384, 1024, kLayoutSW128), idesc_bf16(128, 128, true, true),
                              1u);
            mma_commit_warp(BMMA);
        }
        mma_wait();
        // the next item's k, q, log_alpha go over tiles no product reads again
        if (leader && next < total) issue_raw(sm, BLD, tm_k, tm_q, tm_g, p, next);

        // ---- the gradients
        if (quad >= 2) {   // dKtil e^G (rows 64-127 of the stacked tile) into the exchange
            const int t = 32 * (quad - 2) + lane;
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                const int c0 = 64 * half + 32 * part;
                float x[32];
                tmem_ld32(tmem_addr(tmem + kColD1, 32 * quad, c0), x);
                tmem_wait_ld();
                const float4 *G4 = reinterpret_cast<const float4 *>(gscr + t * 128 + c0);
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const float4 G = G4[m];
                    *xch_at(sm, t, c0 / 4 + m) = make_float4(x[4 * m] * prep::exp2_f(G.x), x[4 * m + 1] * prep::exp2_f(G.y),
                                                             x[4 * m + 2] * prep::exp2_f(G.z), x[4 * m + 3] * prep::exp2_f(G.w));
                }
            }
        }
        tc_fence_before();
        named_barrier(BAR, kThreads);
        if (quad < 2) {
            tc_fence_after();
            const int t = 32 * quad + lane;
            const bool valid = t < L;
            const size_t row = (size_t)(tok0 + t) * p.H + h;
#pragma unroll 1
            for (int part = 0; part < 2; ++part) {
                const int c0 = 64 * half + 32 * part;
                float dQ[32], dKh[32], dKb[32], kr[32], qr[32];
                tmem_ld32(tmem_addr(tmem + kColD1, 32 * quad, c0), dQ);
                tmem_ld32(tmem_addr(tmem + kColY, 32 * quad, c0), dKh);
                tmem_ld32(tmem_addr(tmem + kColX, 32 * quad, c0), dKb);
                gload32(p.k + row * 128 + c0, valid, kr);
                gload32(p.q + row * 128 + c0, valid, qr);
                tmem_wait_ld();
                const float4 *G4 = reinterpret_cast<const float4 *>(gscr + t * 128 + c0);
                float xb[32];
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const float4 G = G4[m];
                    const float4 X = *xch_at(sm, t, c0 / 4 + m);
                    const float Gs[4] = {G.x, G.y, G.z, G.w}, Xs[4] = {X.x, X.y, X.z, X.w};
                    float dq4[4], dk4[4], dG4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = 4 * m + e;
                        const float eG = prep::exp2_f(Gs[e]), eiG = prep::exp2_f(-Gs[e]);
                        const float eb = egl[c0 + j] * eiG;
                        const float hk = dKh[j] * eiG, bk = dKb[j] * eb;
                        dq4[e] = dQ[j] * eG;
                        dk4[e] = Xs[e] + hk + bk;
                        xb[j] = kr[j] * bk;
                        dG4[e] = kr[j] * (Xs[e] - hk) - xb[j] + qr[j] * dq4[e];
                    }
                    if (valid) {
                        *reinterpret_cast<float4 *>(p.dq + row * 128 + c0 + 4 * m) =
                            make_float4(dq4[0], dq4[1], dq4[2], dq4[3]);
                        *reinterpret_cast<float4 *>(p.dk + row * 128 + c0 + 4 * m) =
                            make_float4(dk4[0], dk4[1], dk4[2], dk4[3]);
                    }
                    *xch_at(sm, t, c0 / 4 + m) = make_float4(dG4[0], dG4[1], dG4[2], dG4[3]);
                }
                atomicAdd(&dgl[c0 + lane], column_sums(xb, lane));
            }
        }
        named_barrier(BAR, kThreads);
        if (pt < 128) {   // dg: the running sum from the chunk end, plus the terms of G_L
            const int c = pt;
            const float tot = dgl[c] + egl[c] * es[c];
            float acc = 0.f;
            for (int t = L - 1; t >= 0; --t) {
                acc += reinterpret_cast<const float *>(xch_at(sm, t, c >> 2))[c & 3];
                p.dg[((size_t)(tok0 + t) * p.H + h) * 128 + c] = acc + tot;
            }
        } else if (pt - 128 < L) {
            const int t = pt - 128;
            p.dbeta[(size_t)(tok0 + t) * p.H + h] = db[t];
        }
        named_barrier(BAR, kThreads);
    }
    if (leader && *abort_flag) atomicOr(p.err_word, kDevErrTimeout);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(misc[0], 512);
    }
}

}  // namespace bwdtc

size_t backward_tc_scratch(int grid) { return (size_t)grid * bwdtc::C * bwdtc::DK * sizeof(float); }

cudaError_t launch_backward_tc(const void *q, const void *k, const void *v, const void *g, const void *beta,
                               const void *d_o, int64_t total_tokens, int H, const int2 *chunk_tab,
                               const uint32_t *total_chunks, const float *s_in, const float *ds_next, float *dq,
                               float *dk, float *dv, float *dg, float *dbeta, uint32_t *slow, float *gscr,
                               uint32_t *err_word, int grid, cudaStream_t stream) {
    using namespace bwdtc;
    CUtensorMap mk, mq, mg, mdo;
    if (!make_bf16_map_3d(&mk, k, total_tokens, H, DK, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_bf16_map_3d(&mq, q, total_tokens, H, DK, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_bf16_map_3d(&mg, g, total_tokens, H, DK, 128, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_bf16_map_3d(&mdo, d_o, total_tokens, H, 128, 64, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    cudaError_t e = set_max_dynamic_smem((const void *)kda_bwd_chunk_tc_kernel, (int)Sm::ALLOC);
    if (e != cudaSuccess) return e;
    Args a;
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.k = static_cast<const __nv_bfloat16 *>(k);
    a.v = static_cast<const __nv_bfloat16 *>(v);
    a.g = static_cast<const __nv_bfloat16 *>(g);
    a.beta = static_cast<const __nv_bfloat16 *>(beta);
    a.d_o = static_cast<const __nv_bfloat16 *>(d_o);
    a.s_in = s_in;
    a.ds_next = ds_next;
    a.chunk_tab = chunk_tab;
    a.total_chunks = total_chunks;
    a.dq = dq;
    a.dk = dk;
    a.dv = dv;
    a.dg = dg;
    a.dbeta = dbeta;
    a.slow = slow;
    a.gscr = gscr;
    a.err_word = err_word;
    a.H = H;
    kda_bwd_chunk_tc_kernel<<<grid, kThreads, Sm::ALLOC, stream>>>(mk, mq, mg, mdo, a);
    return cudaGetLastError();
}

}  // namespace kda
