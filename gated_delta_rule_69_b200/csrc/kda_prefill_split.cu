// KDA prefill as two kernels (bf16 I/O, d_k = d_v = 128, C = 64):
//
//   kda_prep_kernel  - persistent, chunk-parallel: for every (chunk, head) the
//                      chunk preparation of kda_chunk_prep.cuh (running sums,
//                      gated operands, [A; P] on the tensor cores, T = (I+A)^-1,
//                      W), then the chunk's transition operands
//                          MP = -Kbar^T W,  YT = Kbar^T T_beta,
//                          QP = Qtil - P W, ZB = P T_beta,  exp(G_L)
//                      on the tensor cores, written to the workspace as a
//                      73 KB record in the layout the chain's products read.
//   kda_chain_kernel - the serial state chain, one CTA per (sequence, head,
//                      slice of d_v; 32 columns or the whole 128): per chunk it
//                      bulk-copies the record (plus its v slice by TMA) into
//                      rings and, with the fp32 state S in TMEM, computes
//                          S <- Diag(exp(G_L)) S + MP S + YT V,  O = QP S + ZB V
//                      on the tensor cores.
//
// The state-independent preparation (the long-latency part of a chunk: the
// gating exponentials and the triangular solve) thus runs chunk-parallel
// over the whole GPU, once per (chunk, head), and leaves the serial chain
// (news digest page on Kimi Linear, section "Algorithme parallele par chunks":
// the previous chunk's final state is the next chunk's initial state) with
// one product group per chunk on its serial path.  The price is the record's
// round trip through L2 / global memory.
#include <cuda.h>

#include "kda_chunk_prep.cuh"
#include "kda_internal.cuh"
#include "kda_sm100.cuh"

namespace kda {
namespace split {

using namespace sm100;

constexpr int C = 64;
constexpr int DK = 128;
constexpr int DV = 128;

// ---- the per-(chunk, head) record: bf16 tensor-core operands in the
// K-major 128-byte-swizzled layout the chain kernel's products read.
//   MP = -Kbar^T W      [128 c_out][128 c_in]  (2 K-atoms x 16 KB)
//   YT = Kbar^T T_beta  [128 c][64 t]          (1 K-atom)
//   QP = Qtil - P W     [64 t][128 c]          (2 K-atoms x 8 KB)
//   ZB = P T_beta       [64 t][64 i]           (1 K-atom)
//   EGL = exp(G_L)      128 fp32
// so that, for a chunk with input state S and values V,
//   S_next = Diag(exp(G_L)) S + MP S + YT V,   O = QP S + ZB V.
struct Rec {
    static constexpr uint32_t MP = 0;
    static constexpr uint32_t YT = 32768;
    static constexpr uint32_t QP = 49152;
    static constexpr uint32_t ZB = 65536;
    static constexpr uint32_t EGL = 73728;
    static constexpr uint32_t BYTES = 74240;   // bytes carried
    static constexpr uint32_t STRIDE = 74752;  // record stride (1024-aligned)
};

// ---- prep kernel
// Two independent preparation pipelines per CTA (one CTA per SM), each of
// 8 warps; pipeline P owns warps 8P..8P+7, its own shared-memory half and
// its own 256 TMEM columns.
constexpr int kPipeThreads = 256;
constexpr int kPrepThreads = 2 * kPipeThreads;
struct PrepSmem {
    static constexpr uint32_t STK = 0;         // raw k | q -> [Ktil | Qtil] -> [-W | QP], 2 K-atoms x 16 KB
                                               // (rows 0-63 and 64-127 of each atom)
    static constexpr uint32_t KBAR = 32768;    // Kbar [64 t][128 c] (2 K-atoms x 8 KB), then YT
    static constexpr uint32_t TB = 49152;      // T diag(beta) [64 t][64 i], then ZB
    static constexpr uint32_t PB = 57344;      // P [64 t][64 i]
    static constexpr uint32_t EGL = 65536;     // 128 fp32
    static constexpr uint32_t KHAT = 66560;    // Khat, then A fp32 (16,640 bytes), then MP K-atom 0
    static constexpr uint32_t GRAW = 83968;    // raw log_alpha, then T fp32 (17,408 bytes), then MP K-atom 1
    static constexpr uint32_t XF = 101376;     // solve scratch (4608 bytes)
    static constexpr uint32_t BETA = 105984;   // 64 fp32
    static constexpr uint32_t CSUM = 106240;   // 4 x 128 fp32
    static constexpr uint32_t BARS = 108288;   // 6 mbarriers
    static constexpr uint32_t MISC = 108352;   // tmem base, abort, slow flag, next-item slots at 4, 5
    static constexpr uint32_t NRM = 108416;    // layer prologue: 128 fp32 inverse norms
    static constexpr uint32_t GSC = 108928;    // scalar gate: 64 fp32 raw log_alpha
    static constexpr uint32_t SIZE = 109184;
    static constexpr uint32_t PIPE = 109568;   // per-pipeline stride
    static constexpr uint32_t ALLOC = 2 * PIPE + 1024;
};
static_assert(PrepSmem::ALLOC <= 232448 && PrepSmem::SIZE <= PrepSmem::PIPE,
              "two preparation pipelines per CTA");
static_assert(PrepSmem::KHAT + 64 * prep::kAStride * 4 <= PrepSmem::GRAW &&
                  PrepSmem::GRAW + 64 * prep::kTStride * 4 <= PrepSmem::XF &&
                  PrepSmem::XF + 4608 <= PrepSmem::BETA,
              "solve scratch");
// per pipeline (256 columns): [A;P] at 0; then YT at 128, ZB at 192; then
// YT Ktil at 0 and ZB Ktil at 128 (all M = 128 products)
constexpr uint32_t kPrepTmemCols = 512;
constexpr uint32_t kRawBytes = 4 * 8192 + 16384;   // k, q (2 boxes each), log_alpha

// ---- chain kernel, one CTA per (sequence, head, 32-column slice of d_v).
// Warp 0 loads ring A, warp NCW + 2 ring B (each ring runs ahead on its own);
// warps 1 .. NCW hold the state (warp w: TMEM lanes of quadrant w mod 4,
// columns 32 ((w - 1) / 4) .. + 31 of the slice); warp NCW + 1 issues the
// products.  Ring A carries MP, YT, the v slice and exp(G_L); ring B QP, ZB.
// Three ring-A and two ring-B stages, two bf16 state copies.
constexpr uint32_t align1k(uint32_t x) { return (x + 1023u) & ~1023u; }

template <int DVT_>
struct ChainCfg {
    static constexpr int DVT = DVT_;
    static_assert(DVT_ == 32, "the row-major chain runs 32-column slices");
    static constexpr int NTILE = DV / DVT;
    static constexpr int NCW = 4 * (DVT / 32);
    static constexpr int THREADS = 32 * (NCW + 3);
    static constexpr int NSA = 3;
    static constexpr int NSB = 2;
    // Copies of the bf16 state: two let the chain warps write S_{n+1} while
    // chunk n's output products still read S_n.
    static constexpr int NSBC = 2;
    static constexpr uint32_t V_BYTES = (uint32_t)DVT * C * 2;
    static constexpr uint32_t A_MP = 0, A_YT = 32768, A_V = 49152;
    static constexpr uint32_t A_STRIDE = align1k(A_V + V_BYTES);
    static constexpr uint32_t B_QP = 0, B_ZB = 16384;
    static constexpr uint32_t B_STRIDE = 24576;
    static constexpr uint32_t SB_BYTES = (uint32_t)DK * DVT * 2;   // S bf16 [128 c][DVT j]
    static constexpr uint32_t RA = 0;
    static constexpr uint32_t RB = NSA * A_STRIDE;
    static constexpr uint32_t SB = RB + NSB * B_STRIDE;
    static constexpr uint32_t EGLR = SB + NSBC * SB_BYTES;  // NSA x exp(G_L), 128 fp32 each
    static constexpr uint32_t BARS = EGLR + NSA * 512;
    static constexpr uint32_t MISC = BARS + 256;
    static constexpr uint32_t SIZE = MISC + 64;
    static constexpr uint32_t ALLOC = SIZE + 1024;
    static constexpr uint32_t TMEM_COLS = 128;
    // X (the chunk's state products) x2, then O x2 (M = 64 layout)
    static constexpr uint32_t COL_X = 0, COL_O = 2 * DVT;
    static_assert(ALLOC <= 232448, "chain shared memory");
    static_assert(4 * DVT <= (int)TMEM_COLS, "chain TMEM");
};
static_assert(Rec::YT == Rec::MP + 32768 && Rec::ZB == Rec::QP + 16384,
              "MP and YT, QP and ZB travel as one copy each");

struct Params {
    const __nv_bfloat16 *k, *q, *beta;
    const __nv_bfloat16 *g;     // log_alpha [T, H] when scalar_gate
    int scalar_gate;
    // layer prologue / epilogue (layer != 0): the g map carries the gate
    // pre-activation, beta holds logits; the chain normalises and gates o
    int layer;
    // the layer prologue's inverse L2 norms of k and q, fp32 [T * H][2] (k, q),
    // for raw q and k (the preparation scales every operand by them); or null
    const float *nrm_in;
    const float *A_log;
    const __nv_bfloat16 *out_gate;
    const float *norm_weight;
    float qk_eps, norm_eps;
    const float *init_state;
    float *final_state;
    __nv_bfloat16 *o;
    const int32_t *cu;          // may be null: equal lengths
    const int32_t *perm;        // longest-first order (chain kernel) or null
    const int32_t *chunk_off;   // [N+1] first record index of each sequence
    const int2 *chunk_tab;      // [max_chunks] (first token, length) of each record's chunk
    const uint32_t *total_chunks;
    uint8_t *recs;              // records, STRIDE bytes each, index (chunk * H + h)
    uint32_t *rec_ready;        // [max_chunks * H] set to 1 once a record is complete; null
                                // when the chain kernel starts only after the prep grid
    uint32_t *work_next;        // prep items handed out after each pipeline's first one
    uint32_t *err_word;
    // backward-pass scans of the transposed chain: each chunk's state written
    // here as a bf16 tile [128 c][128 j] (two 16 KB K-atoms of 64 j, 128-byte
    // swizzle: the layout of a tensor-core operand), 32 KB per record
    // (record = chunk * H + head)
    uint8_t *states_out;
    int64_t total_tokens;
    int num_seqs, H;
};

__device__ __forceinline__ void seq_bounds(const Params &p, int seq, int64_t &bos, int64_t &eos) {
    if (p.cu) {
        bos = p.cu[seq];
        eos = p.cu[seq + 1];
        if (bos < 0 || eos < bos || eos > p.total_tokens) bos = eos = 0;  // flagged by the plan kernel
    } else {
        const int64_t len = p.total_tokens / p.num_seqs;
        bos = (int64_t)seq * len;
        eos = bos + len;
    }
}

// 1-D bulk copies between global and shared memory (16-byte aligned,
// multiple-of-16 sizes).  Loads complete on an mbarrier; stores are tracked
// as a bulk group of the issuing thread.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void bulk_store(void *dst, const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 ::"l"(dst), "r"(smem_addr(src)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

__device__ __forceinline__ void bulk_wait_read_all() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// all but the most recently committed bulk group have read their sources
__device__ __forceinline__ void bulk_wait_read_all_but_last() {
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}


// Record hand-off between the kernels: the writer completes its bulk stores,
// orders them before a release store of the flag; the reader acquires the
// flag and orders it before its own bulk (async-proxy) reads.
__device__ __forceinline__ void publish_flag(uint32_t *flag) {
    asm volatile("fence.proxy.async.global;" ::: "memory");
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(flag), "r"(1u) : "memory");
}

__device__ __forceinline__ bool acquire_flag(const uint32_t *flag, volatile uint32_t *abort) {
    const uint64_t t0 = global_timer_ns();
    uint32_t ns = 32;
    while (true) {
        uint32_t v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
        if (v) break;
        if (*abort) return false;
        if (global_timer_ns() - t0 > 2000000000ull) {
            *abort = 1u;
            return false;
        }
        __nanosleep(ns);
        if (ns < 1024) ns <<= 1;
    }
    asm volatile("fence.proxy.async.global;" ::: "memory");
    return true;
}

__device__ __forceinline__ void wait_drain(uint64_t *bar, uint32_t parity) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > 1000000000ull) return;
    }
}

// =============================================================== prep kernel

// ---- read-outs of the record's products (TMEM -> bf16, K-major 128-byte
// swizzle).  A warp of TMEM quadrant `quad` handles half `half` of the
// columns.  M = 64 products keep row r in lane (r mod 16) + 32 (r / 16).
__device__ __forceinline__ void store8(uint8_t *tile, uint32_t row, uint32_t col, const float *v) {
    uint4 pk;
    pk.x = pack_bf16x2(v[0], v[1]);
    pk.y = pack_bf16x2(v[2], v[3]);
    pk.z = pack_bf16x2(v[4], v[5]);
    pk.w = pack_bf16x2(v[6], v[7]);
    *reinterpret_cast<uint4 *>(tile + sw128_off(row, col)) = pk;
}

// MP = -(YT Ktil) [128 c_out][128 c_in] from the product YT Ktil in TMEM:
// K-atom `half` (at atom0 or atom1) holds c_in 64 half .. + 63.
__device__ __forceinline__ void write_mp(uint8_t *atom0, uint8_t *atom1, uint32_t tmem, int quad,
                                         int half, int lane) {
    uint8_t *atom = half ? atom1 : atom0;
    const int row = 32 * quad + lane;
#pragma unroll
    for (int part = 0; part < 2; ++part) {
        float v[32];
        tmem_ld32(tmem_addr(tmem, 32 * quad, 64 * half + 32 * part), v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = -v[j];
#pragma unroll
        for (int j = 0; j < 32; j += 8) store8(atom, row, 32 * part + j, v + j);
    }
}

// YT [128 c][64 t].
__device__ __forceinline__ void write_yt(uint8_t *yt, uint32_t tmem, int quad, int half, int lane) {
    float v[32];
    tmem_ld32(tmem_addr(tmem, 32 * quad, 32 * half), v);
    tmem_wait_ld();
    const int row = 32 * quad + lane;
#pragma unroll
    for (int j = 0; j < 32; j += 8) store8(yt, row, 32 * half + j, v + j);
}

// ZB [64 t][64 i]: rows 0-63 of an M = 128 product whose A operand starts
// at P (rows 64-127 multiply whatever follows P in shared memory and are not
// read), read by the warps of TMEM quadrants 0 and 1.
__device__ __forceinline__ void write_zb(uint8_t *zb, uint32_t tmem, int quad, int half, int lane) {
    if (quad >= 2) return;
    float v[32];
    tmem_ld32(tmem_addr(tmem, 32 * quad, 32 * half), v);
    tmem_wait_ld();
    const int t = 32 * quad + lane;
#pragma unroll
    for (int j = 0; j < 32; j += 8) store8(zb, t, 32 * half + j, v + j);
}

// QP = Qtil - ZB Ktil, in place over Qtil: rows 64-127 of the two 16 KB
// K-atoms of `stk`, K-atom `half` holding channels 64 half .. + 63.  ZB Ktil
// is rows 0-63 of an M = 128 product whose A operand starts at ZB, read by the
// warps of TMEM quadrants 0 and 1.
__device__ __forceinline__ void write_qp(uint8_t *stk, uint32_t tmem, int quad, int half, int lane) {
    if (quad >= 2) return;
    uint8_t *atom = stk + half * 16384;
    const int t = 32 * quad + lane;
#pragma unroll
    for (int part = 0; part < 2; ++part) {
        float v[32];
        tmem_ld32(tmem_addr(tmem, 32 * quad, 64 * half + 32 * part), v);
        tmem_wait_ld();
        {
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
                uint4 *q8 = reinterpret_cast<uint4 *>(atom + sw128_off(64 + t, 32 * part + j));
                const uint4 qv = *q8;
                const uint32_t w[4] = {qv.x, qv.y, qv.z, qv.w};
                float f[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const __nv_bfloat162 h2 = *reinterpret_cast<const __nv_bfloat162 *>(&w[e]);
                    f[2 * e] = __low2float(h2) - v[j + 2 * e];
                    f[2 * e + 1] = __high2float(h2) - v[j + 2 * e + 1];
                }
                store8(atom, 64 + t, 32 * part + j, f);
            }
        }
    }
}

// LAYER: 0 the plain operator; 1 the layer prologue inside (gate activation,
// beta sigmoid and the q / k norms from the raw rows); 2 the operator on raw q
// and k with their inverse norms given (p.nrm_in).
template <int P, int LAYER, bool SCALAR>
__device__ __forceinline__ void prep_pipeline(uint8_t *sm, uint32_t tmem, int tid, int warp, int lane,
                                              const CUtensorMap &tm_k, const CUtensorMap &tm_q,
                                              const CUtensorMap &tm_g, const Params &p,
                                              uint32_t total_items) {
    constexpr uint32_t BAR = 1 + P;          // this pipeline's 256 threads
    const int wp = warp - 8 * P;
    const int pt = tid - P * kPipeThreads;
    const bool leader = pt == 0;
    const int quad = warp & 3, half = wp >> 2;
    uint64_t *B = reinterpret_cast<uint64_t *>(sm + PrepSmem::BARS);   // raw, [A;P], YT/ZB, MP/QP,
                                                                      // (unused), secondary-chunking blocks
    uint32_t *misc = reinterpret_cast<uint32_t *>(sm + PrepSmem::MISC);
    volatile uint32_t *abort_flag = misc + 1;
    float *beta = reinterpret_cast<float *>(sm + PrepSmem::BETA);
    // The leader publishes a record one step late: it waits only for the
    // stores to have read shared memory before it loads the next item, and
    // for their writes to complete once the next item's first product has
    // been issued, by which time they have long landed.
    uint32_t *pending = nullptr;
    uint32_t sec_round = 0;   // phases of B[5] (secondary-chunking products) so far
    // Items: each pipeline starts with its own, then takes the next free one
    // from a global counter (SMs do not run at the same speed, so a fixed
    // share would leave the slowest as the tail).  The leader draws the
    // following item early in the current one and leaves it in a two-entry
    // slot, which every thread reads after the current item's last barrier.
    volatile uint32_t *next_slot = misc + 4;
    uint32_t item = 2 * blockIdx.x + P;
    uint32_t drawn = 0;   // the next item, drawn while the current one's loads are in flight
#pragma unroll 1
    for (int it = 0; item < total_items; ++it) {
        const int h = item % p.H;
        const uint32_t chunk = item / p.H;
        const int2 ct = p.chunk_tab[chunk];   // one load: the token range was planned
        const int64_t tok0 = ct.x;
        const int L = ct.y;
        uint8_t *rec = p.recs + ((size_t)chunk * p.H + h) * Rec::STRIDE;
        // Loads.  The leader reaches this point after every thread has
        // passed the previous item's last barrier and after the record
        // stores have read the buffers these loads overwrite (STK, GRAW);
        // the rest of the record may still be leaving shared memory, so the
        // leader's arrive, which lets the group write again, waits for that.
        if (leader) {
            mbar_expect_tx(&B[0], SCALAR ? kRawBytes - 16384 : kRawBytes);
            const int t = (int)tok0;
            tma_load_3d(sm + PrepSmem::STK, &tm_k, &B[0], 0, h, t);
            tma_load_3d(sm + PrepSmem::STK + 16384, &tm_k, &B[0], 64, h, t);
            tma_load_3d(sm + PrepSmem::STK + 8192, &tm_q, &B[0], 0, h, t);
            tma_load_3d(sm + PrepSmem::STK + 16384 + 8192, &tm_q, &B[0], 64, h, t);
            if (!SCALAR) tma_load_3d(sm + PrepSmem::GRAW, &tm_g, &B[0], 0, h, t);
            bulk_wait_read_all();
            mbar_arrive(&B[0]);
            // while the loads are in flight: draw the next item, and publish the
            // previous record once its stores have completed
            drawn = atomicAdd(p.work_next, 1u);   // consumed at the end of the item
            if (pending) {
                bulk_wait_all();
                publish_flag(pending);
                pending = nullptr;
            }
        }
        if (pt < C) {
            float bv = (pt < L) ? __bfloat162float(p.beta[(size_t)(tok0 + pt) * p.H + h]) : 0.f;
            if (LAYER == 1 && pt < L) bv = 1.f / (1.f + __expf(-bv));   // beta = sigmoid(logit)
            beta[pt] = bv;
            if (LAYER == 2) {   // the given inverse norms (none past the chunk end)
                float2 nv = make_float2(0.f, 0.f);
                if (pt < L) nv = *reinterpret_cast<const float2 *>(p.nrm_in + ((size_t)(tok0 + pt) * p.H + h) * 2);
                float *nrm = reinterpret_cast<float *>(sm + PrepSmem::NRM);
                nrm[pt] = nv.x;
                nrm[64 + pt] = nv.y;
            }
            if (SCALAR) {   // one log_alpha per token (zero past the chunk end)
                reinterpret_cast<float *>(sm + PrepSmem::GSC)[pt] =
                    pt < L ? __bfloat162float(p.g[(size_t)(tok0 + pt) * p.H + h]) : 0.f;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&B[0]);
        }

        prep::Bufs b;
        b.stk = sm + PrepSmem::STK;
        b.khat = sm + PrepSmem::KHAT;
        b.kbar = sm + PrepSmem::KBAR;
        b.graw = sm + PrepSmem::GRAW;
        b.af = reinterpret_cast<float *>(sm + PrepSmem::KHAT);
        b.tf = reinterpret_cast<float *>(sm + PrepSmem::GRAW);
        b.xf = reinterpret_cast<float *>(sm + PrepSmem::XF);
        b.tb = sm + PrepSmem::TB;
        b.pb = sm + PrepSmem::PB;
        b.beta = beta;
        b.egl = reinterpret_cast<float *>(sm + PrepSmem::EGL);
        b.csum = reinterpret_cast<float *>(sm + PrepSmem::CSUM);
        b.slow_flag = misc + 2;
        b.nrm = LAYER ? reinterpret_cast<float *>(sm + PrepSmem::NRM) : nullptr;
        b.neg_eA = LAYER == 1 ? -__expf(p.A_log[h]) : 0.f;
        b.qk_eps = p.qk_eps;
        b.gsc = SCALAR ? reinterpret_cast<const float *>(sm + PrepSmem::GSC) : nullptr;

        mbar_wait(&B[0], it & 1, abort_flag);
        const int form = SCALAR ? prep::gate_scalar<BAR>(b, pt, L) : prep::gate<BAR, LAYER>(b, pt, L);
        fence_async_smem();
        named_barrier(BAR, prep::kGroupThreads);
        if (wp == 0) {   // tensor-core products: issued by the group's first warp
            tc_fence_after();
            const uint32_t a0 = smem_addr(sm + PrepSmem::STK), b0 = smem_addr(sm + PrepSmem::KHAT);
            const uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)   // [Ktil; Qtil] Khat^T
                mma_bf16_warp(tmem, smem_desc(a0 + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kLayoutSW128),
                              smem_desc(b0 + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024, kLayoutSW128),
                              id, ks > 0 ? 1u : 0u);
            mma_commit_warp(&B[1]);
        }
        mbar_wait(&B[1], it & 1, abort_flag);
        tc_fence_after();
        if (form == prep::kProductForm) {
            prep::read_ap(b, tmem, quad, half, lane);
        } else {
            const size_t stride = (size_t)p.H * DK;
            const __nv_bfloat16 *kt0 = p.k + ((size_t)tok0 * p.H + h) * DK;
            const __nv_bfloat16 *qt0 = p.q + ((size_t)tok0 * p.H + h) * DK;
            if (form == prep::kSecondary) {
                prep::secondary<BAR>(b, pt, L, kt0, qt0, stride, sm + PrepSmem::KHAT, sm + PrepSmem::GRAW,
                                     sm + PrepSmem::XF, tmem, wp == 0, &B[5], sec_round, abort_flag);
                prep::read_ap(b, tmem, quad, half, lane);
            } else {
                prep::pairwise(b, pt, L, kt0, qt0, stride);
            }
        }
        tc_fence_before();
        named_barrier(BAR, prep::kGroupThreads);
        prep::solve<BAR>(b, pt);
        fence_async_smem();
        named_barrier(BAR, prep::kGroupThreads);
        const uint32_t sK = smem_addr(sm + PrepSmem::STK), sKb = smem_addr(sm + PrepSmem::KBAR);
        const uint32_t sT = smem_addr(sm + PrepSmem::TB), sP = smem_addr(sm + PrepSmem::PB);
        // W = T_beta Ktil is never formed: with YT = Kbar^T T_beta and
        // ZB = P T_beta, MP = -Kbar^T W = -YT Ktil and QP = Qtil - P W =
        // Qtil - ZB Ktil, so the record takes two groups of products.
        if (wp == 0) {
            tc_fence_after();
            const uint32_t idY = idesc_bf16(128, C, true, true);
            const uint32_t idZ = idesc_bf16(128, C, false, true);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {   // K = 64 tokens
                // YT = Kbar^T T_beta
                mma_bf16_warp(tmem + 128, smem_desc(sKb + ks * 2048, 8192, 1024, kLayoutSW128),
                              smem_desc(sT + ks * 2048, 8192, 1024, kLayoutSW128), idY, ks > 0 ? 1u : 0u);
                // ZB = P T_beta: rows 0-63 of an M = 128 product whose A starts at P
                mma_bf16_warp(tmem + 192, smem_desc(sP + ks * 32, 16, 1024, kLayoutSW128),
                              smem_desc(sT + ks * 2048, 8192, 1024, kLayoutSW128), idZ, ks > 0 ? 1u : 0u);
            }
            mma_commit_warp(&B[2]);
        }
        mbar_wait(&B[2], it & 1, abort_flag);
        tc_fence_after();
        // Kbar, T_beta are no longer read: YT and ZB go over them
        write_yt(sm + PrepSmem::KBAR, tmem + 128, quad, half, lane);
        write_zb(sm + PrepSmem::TB, tmem + 192, quad, half, lane);
        fence_async_smem();
        tc_fence_before();
        named_barrier(BAR, prep::kGroupThreads);
        if (wp == 0) {
            tc_fence_after();
            const uint32_t idK = idesc_bf16(128, DK, false, true);   // B = Ktil [t][c] (MN-major)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {   // K = 64 tokens
                const uint64_t bK = smem_desc(sK + ks * 2048, 16384, 1024, kLayoutSW128);
                // YT Ktil (= -MP)
                mma_bf16_warp(tmem, smem_desc(sKb + ks * 32, 16, 1024, kLayoutSW128), bK, idK,
                              ks > 0 ? 1u : 0u);
                // ZB Ktil (= Qtil - QP): rows 0-63 of an M = 128 product whose A starts at ZB
                mma_bf16_warp(tmem + 128, smem_desc(sT + ks * 32, 16, 1024, kLayoutSW128), bK, idK,
                              ks > 0 ? 1u : 0u);
            }
            mma_commit_warp(&B[3]);
        }
        mbar_wait(&B[3], it & 1, abort_flag);
        tc_fence_after();
        write_mp(sm + PrepSmem::KHAT, sm + PrepSmem::GRAW, tmem, quad, half, lane);
        write_qp(sm + PrepSmem::STK, tmem + 128, quad, half, lane);
        if (leader) next_slot[(it + 1) & 1] = 2 * gridDim.x + drawn;
        fence_async_smem();
        tc_fence_before();
        named_barrier(BAR, prep::kGroupThreads);
        const uint32_t next_item = next_slot[(it + 1) & 1];
        if (leader) {
            // first group: the sources the next item's loads overwrite
            bulk_store(rec + Rec::QP, sm + PrepSmem::STK + 8192, 8192);
            bulk_store(rec + Rec::QP + 8192, sm + PrepSmem::STK + 16384 + 8192, 8192);
            bulk_store(rec + Rec::MP + 16384, sm + PrepSmem::GRAW, 16384);
            bulk_commit();
            bulk_store(rec + Rec::MP, sm + PrepSmem::KHAT, 16384);
            bulk_store(rec + Rec::YT, sm + PrepSmem::KBAR, 16384);
            bulk_store(rec + Rec::ZB, sm + PrepSmem::TB, 8192);
            bulk_store(rec + Rec::EGL, sm + PrepSmem::EGL, 512);
            bulk_commit();
            bulk_wait_read_all_but_last();
            if (p.rec_ready) pending = p.rec_ready + (size_t)chunk * p.H + h;
        }
        item = next_item;
    }
    if (leader) {
        bulk_wait_all();
        if (pending) publish_flag(pending);
        if (*abort_flag) atomicOr(p.err_word, kDevErrTimeout);
    }
}

// LAYER (as prep_pipeline): 1 the layer prologue (gate activation, q / k
// normalisation, beta sigmoid) fused in, 2 raw q and k with given inverse
// norms; SCALAR: the Gated DeltaNet gate (one log_alpha per token); separate
// instantiations keep the plain kernel as it is.
template <int LAYER, bool SCALAR>
__global__ void __launch_bounds__(kPrepThreads, 1)
kda_prep_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                const __grid_constant__ CUtensorMap tm_g, const Params p) {
    extern __shared__ uint8_t dyn_smem[];
    uint8_t *sm0 = dyn_smem + ((1024u - (smem_addr(dyn_smem) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int P = warp / 8;
    uint8_t *sm = sm0 + P * PrepSmem::PIPE;
    uint32_t *misc0 = reinterpret_cast<uint32_t *>(sm0 + PrepSmem::MISC);
    if (tid == 0 || tid == kPipeThreads) {
        uint64_t *B = reinterpret_cast<uint64_t *>(sm + PrepSmem::BARS);
        mbar_init(&B[0], 3);   // the leader, and one arrive per beta warp
        for (int i = 1; i < 6; ++i) mbar_init(&B[i], 1);
        reinterpret_cast<uint32_t *>(sm + PrepSmem::MISC)[1] = 0u;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&misc0[0], kPrepTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_g);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // The set-up above overlaps the plan kernel (this grid is its
    // programmatic dependent); its output is read only past this wait.
    // Then a dependent chain kernel may start: it waits on per-record flags,
    // not on this grid's completion.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const uint32_t total_items = *p.total_chunks * (uint32_t)p.H;
    const uint32_t tmem = misc0[0] + 256u * P;
    if (2 * blockIdx.x < total_items) {
        if (P == 0) prep_pipeline<0, LAYER, SCALAR>(sm, tmem, tid, warp, lane, tm_k, tm_q, tm_g, p, total_items);
        else prep_pipeline<1, LAYER, SCALAR>(sm, tmem, tid, warp, lane, tm_k, tm_q, tm_g, p, total_items);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(misc0[0], kPrepTmemCols);
    }
}

// =============================================================== chain kernel

// One thread's 32 state columns (slice columns col0 .. col0 + 31 of row
// `row`) as bf16 into the B-operand copy of S: for a 32-column slice one
// 64-byte-swizzled tile [128 c][32 j]; for wider slices 128-byte-swizzled
// atoms [128 c][64 j], 16 KB apart.
template <int DVT>
__device__ __forceinline__ void store_sb_row(uint8_t *sb, int row, int col0, const float (&v)[32]) {
#pragma unroll
    for (int j = 0; j < 32; j += 8) {
        uint4 pk;
        pk.x = pack_bf16x2(v[j + 0], v[j + 1]);
        pk.y = pack_bf16x2(v[j + 2], v[j + 3]);
        pk.z = pack_bf16x2(v[j + 4], v[j + 5]);
        pk.w = pack_bf16x2(v[j + 6], v[j + 7]);
        if (DVT == 32) {
            *reinterpret_cast<uint4 *>(sb + sw64_off(row, j)) = pk;
        } else {
            const int col = col0 + j;
            *reinterpret_cast<uint4 *>(sb + (col >> 6) * 16384 + sw128_off(row, col & 63)) = pk;
        }
    }
}

// B-operand descriptor of k-step ks for the state copy (K = 128 rows of c)
// and the v slice (K = 64 rows of t).
template <int DVT>
__device__ __forceinline__ uint64_t desc_sb(uint32_t base, int ks) {
    return DVT == 32 ? smem_desc(base + ks * 1024, 16, 512, kLayoutSW64)
                     : smem_desc(base + ks * 2048, 16384, 1024, kLayoutSW128);
}

template <int DVT>
__device__ __forceinline__ uint64_t desc_v(uint32_t base, int ks) {
    return DVT == 32 ? smem_desc(base + ks * 1024, 16, 512, kLayoutSW64)
                     : smem_desc(base + ks * 2048, 8192, 1024, kLayoutSW128);
}

// O of chunk m, 32 columns (slice columns col0 ..) from TMEM (M = 64 layout:
// row t in lane (t mod 16) + 32 (t / 16)) to global memory; the whole warp
// reads, lanes 0-15 hold rows.
template <int DVT>
__device__ __forceinline__ void store_o(uint32_t tmem, int quad, int lane, int col0, int m,
                                        int64_t bos, int64_t len, int h, int j0, const Params &p,
                                        uint64_t *ofree) {
    using Cfg = ChainCfg<DVT>;
    float v[32];
    tmem_ld32(tmem_addr(tmem, 32 * quad, Cfg::COL_O + DVT * (m & 1) + col0), v);
    tmem_wait_ld();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(ofree);   // the O buffer may be written again
    const int t = 16 * quad + lane;
    if (lane < 16 && (int64_t)m * C + t < len) {
        uint4 *dst = reinterpret_cast<uint4 *>(p.o + ((size_t)(bos + (int64_t)m * C + t) * p.H + h) * DV +
                                               j0 + col0);
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

// Per chunk n, with S_n (fp32) in the chain warps' registers (each thread one
// row c and 32 columns of the slice):
//   chain warps: S_n -> bf16 SB[n mod 2] (shared memory, the B operand)
//   product warp, ahead (state-independent): X[n mod 2] = YT V, O[n mod 2] = ZB V
//                 after SB_n:  X[n mod 2] += MP SB_n  (the serial path),
//                              O[n mod 2] += QP SB_n
//   chain warps: S_{n+1} = Diag(exp(G_L)) S_n + X[n mod 2]
// The chain warps read the O of chunk n - 1 out while chunk n's state
// products run.  X[n mod 2] was read by the chain warps before their SREADY
// of chunk n - 1, O[n mod 2] once they arrive on OFREE after reading O_{n-2}.
template <int DVT>
__global__ void __launch_bounds__(ChainCfg<DVT>::THREADS, 1)
kda_chain_kernel(const __grid_constant__ CUtensorMap tm_v, const Params p) {
    using Cfg = ChainCfg<DVT>;
    constexpr int NSA = Cfg::NSA, NSB = Cfg::NSB, NCW = Cfg::NCW, NTILE = Cfg::NTILE;
    extern __shared__ uint8_t dyn_smem[];
    uint8_t *sm = dyn_smem + ((1024u - (smem_addr(dyn_smem) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tile = blockIdx.x % NTILE;
    const int h = (blockIdx.x / NTILE) % p.H;
    const int rank = blockIdx.x / (NTILE * p.H);
    const int seq = p.perm ? p.perm[rank] : rank;
    int64_t bos, eos;
    seq_bounds(p, seq, bos, eos);
    const int64_t len = eos - bos;
    const int nchunks = (int)((len + C - 1) / C);
    const int j0 = tile * DVT;
    const size_t rec0 = (size_t)p.chunk_off[seq];

    // mbarriers: FULLA[NSA], EMPTYA[NSA], FULLB[NSB], EMPTYB[NSB], SDONE, ODONE[2], FIN,
    // SREADY, OFREE[2]
    uint64_t *B = reinterpret_cast<uint64_t *>(sm + Cfg::BARS);
    uint64_t *FULLA = B, *EMPTYA = B + NSA, *FULLB = B + 2 * NSA, *EMPTYB = B + 2 * NSA + NSB;
    uint64_t *SDONE = B + 2 * NSA + 2 * NSB, *ODONE = SDONE + 1, *FIN = SDONE + 3, *SREADY = SDONE + 4;
    uint64_t *OFREE = SDONE + 5;
    constexpr int kBars = 2 * NSA + 2 * NSB + 7;
    static_assert(kBars * 8 <= 256, "barrier area");
    uint32_t *misc = reinterpret_cast<uint32_t *>(sm + Cfg::MISC);
    volatile uint32_t *abort_flag = misc + 1;
    if (tid == 0) {
        for (int i = 0; i < kBars; ++i) {
            // SREADY and OFREE take one arrive per chain warp
            const uint64_t *b = &B[i];
            const bool per_warp = b == SREADY || b == &OFREE[0] || b == &OFREE[1];
            mbar_init(&B[i], per_warp ? (uint32_t)NCW : 1u);
        }
        misc[1] = 0u;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&misc[0], Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];

    if (warp == 0) {
        // ---------------------------------------------- ring A: MP, YT, v slice, exp(G_L)
        if (lane == 0 && nchunks > 0) {
            tma_prefetch_desc(&tm_v);
            int issued_a = 0;
            for (int n = 0; n < nchunks; ++n) {
                const int sa = n % NSA;
                if (n >= NSA) mbar_wait(&EMPTYA[sa], ((n / NSA) - 1) & 1, abort_flag);
                if (*abort_flag) break;
                const size_t ri = (rec0 + n) * p.H + h;
                const uint8_t *rec = p.recs + ri * Rec::STRIDE;
                if (p.rec_ready && !acquire_flag(p.rec_ready + ri, abort_flag)) break;   // the record is complete
                uint8_t *slot_a = sm + Cfg::RA + sa * Cfg::A_STRIDE;
                const int t = (int)(bos + (int64_t)n * C);
                mbar_arrive_expect_tx(&FULLA[sa], 49152 + 512 + Cfg::V_BYTES);
                bulk_load(slot_a + Cfg::A_MP, rec + Rec::MP, 49152, &FULLA[sa]);   // MP, YT
                bulk_load(sm + Cfg::EGLR + sa * 512, rec + Rec::EGL, 512, &FULLA[sa]);
                tma_load_3d(slot_a + Cfg::A_V, &tm_v, &FULLA[sa], j0, h, t);
                issued_a = n + 1;
            }
            // the copies land before this CTA may exit
            for (int n = (issued_a > NSA ? issued_a - NSA : 0); n < issued_a; ++n)
                wait_drain(&FULLA[n % NSA], (n / NSA) & 1);
        }
    } else if (warp == NCW + 2) {
        // ---------------------------------------------- ring B: QP, ZB
        if (lane == 0 && nchunks > 0) {
            int issued_b = 0;
            for (int n = 0; n < nchunks; ++n) {
                const int sb = n % NSB;
                if (n >= NSB) mbar_wait(&EMPTYB[sb], ((n / NSB) - 1) & 1, abort_flag);
                if (*abort_flag) break;
                const size_t ri = (rec0 + n) * p.H + h;
                const uint8_t *rec = p.recs + ri * Rec::STRIDE;
                if (p.rec_ready && !acquire_flag(p.rec_ready + ri, abort_flag)) break;
                uint8_t *slot_b = sm + Cfg::RB + sb * Cfg::B_STRIDE;
                mbar_arrive_expect_tx(&FULLB[sb], 24576);
                bulk_load(slot_b + Cfg::B_QP, rec + Rec::QP, 24576, &FULLB[sb]);   // QP, ZB
                issued_b = n + 1;
            }
            for (int n = (issued_b > NSB ? issued_b - NSB : 0); n < issued_b; ++n)
                wait_drain(&FULLB[n % NSB], (n / NSB) & 1);
        }
    } else if (warp == NCW + 1) {
        // ---------------------------------------------- tensor-core products
        const uint32_t idS = idesc_bf16(128, DVT, false, true);
        const uint32_t idO = idesc_bf16(64, DVT, false, true);
        // the state-independent products of chunk m: X[m mod 2] = YT V, O[m mod 2] = ZB V
        auto pre = [&](int m) {
            const int sa = m % NSA, sb = m % NSB;
            uint8_t *slot_a = sm + Cfg::RA + sa * Cfg::A_STRIDE;
            const uint32_t aY = smem_addr(slot_a + Cfg::A_YT);
            const uint32_t bV = smem_addr(slot_a + Cfg::A_V);
            const uint32_t aZ = smem_addr(sm + Cfg::RB + sb * Cfg::B_STRIDE + Cfg::B_ZB);
            mbar_wait(&FULLA[sa], (m / NSA) & 1, abort_flag);
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)   // X = YT V
                mma_bf16_warp(tmem + Cfg::COL_X + DVT * (m & 1), smem_desc(aY + ks * 32, 16, 1024, kLayoutSW128),
                              desc_v<DVT>(bV, ks), idS, ks > 0 ? 1u : 0u);
            mbar_wait(&FULLB[sb], (m / NSB) & 1, abort_flag);
            if (m >= 2) mbar_wait(&OFREE[m & 1], ((m - 2) >> 1) & 1, abort_flag);
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)   // O = ZB V
                mma_bf16_warp(tmem + Cfg::COL_O + DVT * (m & 1), smem_desc(aZ + ks * 32, 16, 1024, kLayoutSW128),
                              desc_v<DVT>(bV, ks), idO, ks > 0 ? 1u : 0u);
        };
        if (nchunks > 0) pre(0);
        for (int n = 0; n < nchunks; ++n) {
            const int sa = n % NSA, sb = n % NSB;
            uint8_t *slot_a = sm + Cfg::RA + sa * Cfg::A_STRIDE;
            uint8_t *slot_b = sm + Cfg::RB + sb * Cfg::B_STRIDE;
            const uint32_t aM = smem_addr(slot_a + Cfg::A_MP);
            const uint32_t bS = smem_addr(sm + Cfg::SB + (n & 1) * Cfg::SB_BYTES);
            mbar_wait(SREADY, n & 1, abort_flag);
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)   // X += MP SB
                mma_bf16_warp(tmem + Cfg::COL_X + DVT * (n & 1),
                              smem_desc(aM + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kLayoutSW128),
                              desc_sb<DVT>(bS, ks), idS, 1u);
            mma_commit_warp(SDONE);
            const uint32_t aQ = smem_addr(slot_b + Cfg::B_QP);
            const uint32_t dO = tmem + Cfg::COL_O + DVT * (n & 1);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)   // O += QP SB
                mma_bf16_warp(dO, smem_desc(aQ + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024, kLayoutSW128),
                              desc_sb<DVT>(bS, ks), idO, 1u);
            mma_commit_warp(&ODONE[n & 1]);
            mma_commit_warp(&EMPTYA[sa]);
            mma_commit_warp(&EMPTYB[sb]);
            if (n + 1 < nchunks) pre(n + 1);
        }
        if (nchunks > 0) {   // every arrive of the commits above lands before the CTA exits
            mma_commit_warp(FIN);
            wait_drain(FIN, 0);
        }
    } else {
        // ---------------------------------------------- the state chain
        const int quad = warp & 3;
        const int col0 = 32 * ((warp - 1) >> 2);
        const int crow = 32 * quad + lane;
        const size_t soff = ((size_t)seq * p.H + h) * (size_t)(DK * DV) + (size_t)crow * DV + j0 + col0;
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
        auto store_o_m = [&](int m) {   // O of chunk m; the buffer is released once in registers
            mbar_wait(&ODONE[m & 1], (m >> 1) & 1, abort_flag);
            tc_fence_after();
            store_o<DVT>(tmem, quad, lane, col0, m, bos, len, h, j0, p, &OFREE[m & 1]);
        };
        for (int n = 0; n < nchunks; ++n) {
            const int sa = n % NSA;
            // SB[n mod 2] was last read by chunk n - 2's products, which
            // completed before SDONE of chunk n - 1
            store_sb_row<DVT>(sm + Cfg::SB + (n & 1) * Cfg::SB_BYTES, crow, col0, S);
            // this row's exp(G_L), read before the slot may be refilled
            mbar_wait(&FULLA[sa], (n / NSA) & 1, abort_flag);
            const float d = reinterpret_cast<const float *>(sm + Cfg::EGLR + sa * 512)[crow];
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(SREADY);
            if (n >= 1) store_o_m(n - 1);
            mbar_wait(SDONE, n & 1, abort_flag);
            tc_fence_after();
            float x[32];
            tmem_ld32(tmem_addr(tmem, 32 * quad, Cfg::COL_X + DVT * (n & 1) + col0), x);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) S[i] = fmaf(S[i], d, x[i]);
        }
        if (nchunks > 0) store_o_m(nchunks - 1);
        if (p.final_state) {
            float4 *dst = reinterpret_cast<float4 *>(p.final_state + soff);
#pragma unroll
            for (int i = 0; i < 8; ++i)
                dst[i] = make_float4(S[4 * i], S[4 * i + 1], S[4 * i + 2], S[4 * i + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::TMEM_COLS);
    }
    if (tid == 0 && *abort_flag) atomicOr(p.err_word, kDevErrTimeout);
}

// =============================================================== whole-d_v chain, transposed
//
// One CTA per (sequence, head) carrying the state transposed, S^T [j = d_v
// lanes][c = d_k columns]:
//     S_{n+1}^T = S_n^T Diag(exp(G_L)) + X_n,   X_n = SB_n^T MP_n^T + V_n^T YT_n^T
//     O_n^T     = SB_n^T QP_n^T + V_n^T ZB_n^T
// The fp32 state lives in the chain warps' registers (each thread one lane j
// and 32 columns c); per chunk they write its bf16 copy SB_n^T into TMEM as
// the A operand of the products, read the fresh product X_n back, and form
// S_{n+1} with one FMA per element: no fp32 state goes back to TMEM.  The
// record operands keep their tile layout (K-major, 128-byte swizzle); they
// only change side (B instead of A), and V (its two 64-column atoms) is the A
// operand in the MN-major form.
// A tcgen05 product costs about the same whatever its N up to 192 (~100
// cycles per M = 128, K = 16 instruction with A in shared memory, ~116 with
// A in TMEM, against ~134 at N = 256), so the products that share their A
// operand are issued as one: X and O^T lie side by side in TMEM (X in 128
// columns, O^T in the next 64) and the record's B operands side by side in
// shared memory (MP over QP, YT over ZB):
//     [X | O^T]  = V_n^T [YT_n; ZB_n]^T        (4 products, N = 192)
//     [X | O^T] += SB_n^T [MP_n; QP_n]^T       (8 products, N = 192)
// The state-independent group is issued ahead, while the chain warps still
// work on the previous state, so that once SB_n is in TMEM only the second
// group stands between it and S_{n+1}.  [X | O^T] is double-buffered in TMEM.
// The chain warps read O^T out together with X and, once SB_{n+1} is handed
// over, write it in bf16 to a shared-memory staging tile that a store warp
// copies to o with one tensor store per chunk (stores from the chain warps'
// registers straight to global memory, 16 of 64 bytes per warp and chunk,
// took most of a chunk's period).  The backward scan modes stage the state
// tiles they save the same way, and one bulk copy per chunk writes each out.
// Rings, each with its loader warp: R (MP, QP, YT, ZB of a record in the
// layout above), E (exp(G_L); its own deeper ring, since the chain warps read
// it only after the state products) and V (the v tile, read from HBM).
//   warp 0: rings R and E;  warp 18: the stores;  warp 19: ring V
//   warps 1..16: the state; warp w holds lanes j of quadrant w mod 4 and
//                columns c in 32 ((w - 1) / 4) .. + 31
//   warp 17: issues the products
struct ChainT {
    static constexpr int NCW = 16;
    static constexpr int THREADS = 32 * (NCW + 4);
    static constexpr int NSR = 2, NSV = 3, NSE = 3;
    // ring R stage: K-atom 0 of MP (128 rows c) over K-atom 0 of QP (64 rows t),
    // the same for K-atom 1, then YT (128 rows c) over ZB (64 rows t)
    static constexpr uint32_t R_MP = 0, R_QP = 16384, R_KATOM = 24576, R_YT = 49152, R_ZB = 65536;
    static constexpr uint32_t R_STRIDE = 73728;
    static constexpr uint32_t V_STRIDE = 16384;
    static constexpr uint32_t RR = 0;
    static constexpr uint32_t RV = NSR * R_STRIDE;
    static constexpr uint32_t STG = RV + NSV * V_STRIDE;   // 2 x 16 KB of o rows, or one 32 KB state tile
    static constexpr uint32_t EGLR = STG + 32768;          // NSE x exp(G_L), 128 fp32 each
    static constexpr uint32_t BARS = EGLR + NSE * 512;
    static constexpr uint32_t MISC = BARS + 256;
    static constexpr uint32_t SIZE = MISC + 64;
    static constexpr uint32_t ALLOC = SIZE + 1024;
    // TMEM columns: [X | O^T] x 2 (X fp32 in 128 columns, O^T fp32 in 64),
    // SB^T bf16 pairs x 2 (64 each)
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t COL_XO = 0, XO_STRIDE = 192, COL_O = 128, COL_SB = 384;
    static_assert(R_QP == 16384 && R_KATOM == R_QP + 8192 && R_ZB == R_YT + 16384,
                  "B operands of one product group must be contiguous rows");
    static_assert(ALLOC <= 232448, "chain shared memory");
};

// MODE (separate instantiations): kChainPlain; kChainTransition forms a
// segment's cumulative transition for context parallelism: the state starts
// as the identity, v counts as zero (the v ring and the YT V products are
// skipped), no output is formed, and the final state is the transition.
// The backward pass's two scans over the records (no output products):
//   kChainSaveS  - the forward chain, writing every chunk's entering state S_n;
//   kChainReverse - the chunks in reverse order with the transposed
//                  transition, G_n = Diag(exp(G_L)) G_{n+1} + MP^T G_{n+1}
//                  + QP^T dO_n (G = dL/dS; the tensor map carries dO, MP and
//                  QP are read MN-major), writing dL/dS at each chunk's end;
//                  init_state is dL/dS_T and final_state receives dL/dS_0.
enum : int { kChainPlain = 0, kChainTransition = 2, kChainSaveS = 3, kChainReverse = 4 };

// The chain of one (sequence, head) unit (rank `unit` in the longest-first
// order); the kernels below run one unit per CTA.
// tm_o (the output mode only): o as [64 tokens][128 channels] boxes of one head.
template <int MODE>
__device__ __forceinline__ void chain_t_unit(const CUtensorMap &tm_v, const CUtensorMap *tm_o, const Params &p,
                                             int unit) {
    constexpr bool TRANS = MODE == kChainTransition;
    constexpr bool SAVE = MODE == kChainSaveS;
    constexpr bool REV = MODE == kChainReverse;
    constexpr bool OUT = MODE == kChainPlain;          // output products and stores
    using Cfg = ChainT;
    constexpr int NSR = Cfg::NSR, NSV = Cfg::NSV, NSE = Cfg::NSE, NCW = Cfg::NCW;

    extern __shared__ uint8_t dyn_smem[];
    uint8_t *sm = dyn_smem + ((1024u - (smem_addr(dyn_smem) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = unit % p.H;
    const int rank = unit / p.H;
    const int seq = p.perm ? p.perm[rank] : rank;
    int64_t bos, eos;
    seq_bounds(p, seq, bos, eos);
    const int64_t len = eos - bos;
    const int nchunks = (int)((len + C - 1) / C);
    const size_t rec0 = (size_t)p.chunk_off[seq];
    const bool stage_states = (SAVE || REV) && p.states_out != nullptr;

    // mbarriers: FULLR[NSR], EMPTYR[NSR], FULLV[NSV], EMPTYV[NSV], FULLE[NSE],
    // EMPTYE[NSE], SDONE, FIN, SREADY, STGF[2], STGE[2]
    uint64_t *B = reinterpret_cast<uint64_t *>(sm + Cfg::BARS);
    uint64_t *FULLR = B, *EMPTYR = B + NSR, *FULLV = B + 2 * NSR, *EMPTYV = FULLV + NSV;
    uint64_t *FULLE = EMPTYV + NSV, *EMPTYE = FULLE + NSE;
    uint64_t *SDONE = EMPTYE + NSE, *FIN = SDONE + 1, *SREADY = SDONE + 2;
    uint64_t *STGF = SDONE + 3, *STGE = SDONE + 5;
    constexpr int kBars = 2 * NSR + 2 * NSV + 2 * NSE + 7;
    static_assert(kBars * 8 <= 256, "barrier area");
    uint32_t *misc = reinterpret_cast<uint32_t *>(sm + Cfg::MISC);
    volatile uint32_t *abort_flag = misc + 1;
    if (tid == 0) {
        for (int i = 0; i < kBars; ++i) {
            // SREADY, EMPTYE and STGF take one arrive per chain warp
            const uint64_t *b = &B[i];
            const bool per_warp = b == SREADY || b == &STGF[0] || b == &STGF[1] ||
                                  (b >= EMPTYE && b < EMPTYE + NSE);
            mbar_init(&B[i], per_warp ? (uint32_t)NCW : 1u);
        }
        misc[1] = 0u;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&misc[0], Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];

    if (warp == 0) {
        // ---------------------------------------------- rings R (MP, QP, YT, ZB) and E (exp(G_L))
        if (lane == 0 && nchunks > 0) {
            int issued_r = 0, issued_e = 0;
            for (int n = 0; n < nchunks; ++n) {
                const int sr = n % NSR, se = n % NSE;
                if (n >= NSR) mbar_wait(&EMPTYR[sr], ((n / NSR) - 1) & 1, abort_flag);
                if (n >= NSE) mbar_wait(&EMPTYE[se], ((n / NSE) - 1) & 1, abort_flag);
                if (*abort_flag) break;
                const int nn = REV ? nchunks - 1 - n : n;
                const size_t ri = (rec0 + nn) * p.H + h;
                const uint8_t *rec = p.recs + ri * Rec::STRIDE;
                if (p.rec_ready && !acquire_flag(p.rec_ready + ri, abort_flag)) break;   // the record is complete
                uint8_t *slot = sm + Cfg::RR + sr * Cfg::R_STRIDE;
                // MP always; QP for the output (and, read MN-major, the reverse scan);
                // YT wherever v enters; ZB for the output
                constexpr uint32_t kRBytes = 32768 + ((OUT || REV) ? 16384 : 0) + ((OUT || SAVE) ? 16384 : 0) +
                                             (OUT ? 8192 : 0);
                mbar_arrive_expect_tx(&FULLR[sr], kRBytes);
                bulk_load(slot + Cfg::R_MP, rec + Rec::MP, 16384, &FULLR[sr]);
                bulk_load(slot + Cfg::R_MP + Cfg::R_KATOM, rec + Rec::MP + 16384, 16384, &FULLR[sr]);
                if (OUT || REV) {
                    bulk_load(slot + Cfg::R_QP, rec + Rec::QP, 8192, &FULLR[sr]);
                    bulk_load(slot + Cfg::R_QP + Cfg::R_KATOM, rec + Rec::QP + 8192, 8192, &FULLR[sr]);
                }
                if (OUT || SAVE) bulk_load(slot + Cfg::R_YT, rec + Rec::YT, 16384, &FULLR[sr]);
                if (OUT) bulk_load(slot + Cfg::R_ZB, rec + Rec::ZB, 8192, &FULLR[sr]);
                issued_r = n + 1;
                mbar_arrive_expect_tx(&FULLE[se], 512);
                bulk_load(sm + Cfg::EGLR + se * 512, rec + Rec::EGL, 512, &FULLE[se]);
                issued_e = n + 1;
            }
            // the copies land before this CTA may exit
            for (int n = (issued_r > NSR ? issued_r - NSR : 0); n < issued_r; ++n)
                wait_drain(&FULLR[n % NSR], (n / NSR) & 1);
            for (int n = (issued_e > NSE ? issued_e - NSE : 0); n < issued_e; ++n)
                wait_drain(&FULLE[n % NSE], (n / NSE) & 1);
        }
    } else if (warp == NCW + 3) {
        // ---------------------------------------------- ring V: the v (or dO) tile (from HBM)
        if (!TRANS && lane == 0 && nchunks > 0) {
            tma_prefetch_desc(&tm_v);
            int issued_v = 0;
            for (int n = 0; n < nchunks; ++n) {
                const int sv = n % NSV;
                if (n >= NSV) mbar_wait(&EMPTYV[sv], ((n / NSV) - 1) & 1, abort_flag);
                if (*abort_flag) break;
                uint8_t *slot_v = sm + Cfg::RV + sv * Cfg::V_STRIDE;
                const int t = (int)(bos + (int64_t)(REV ? nchunks - 1 - n : n) * C);
                mbar_arrive_expect_tx(&FULLV[sv], 16384);
                tma_load_3d(slot_v, &tm_v, &FULLV[sv], 0, h, t);
                tma_load_3d(slot_v + 8192, &tm_v, &FULLV[sv], 64, h, t);
                issued_v = n + 1;
            }
            for (int n = (issued_v > NSV ? issued_v - NSV : 0); n < issued_v; ++n)
                wait_drain(&FULLV[n % NSV], (n / NSV) & 1);
        }
    } else if (warp == NCW + 2) {
        // ---------------------------------------------- stores from the staging tiles
        if (OUT && nchunks > 0) {
            // chunk m's o rows: buffer m mod 2, row r (token m C + r) at r * 256
            // bytes.  A whole chunk goes out as one tensor store; a sequence's
            // partial last chunk row by row in 16-byte pieces (16 lanes per row),
            // since the box's further rows belong to the next sequence.
            if (lane == 0) tma_prefetch_desc(tm_o);
            for (int m = 0; m < nchunks; ++m) {
                const int b = m & 1;
                const bool ok = mbar_wait(&STGF[b], (m >> 1) & 1, abort_flag);
                // one decision for the whole warp: the loop below synchronises it
                if (__any_sync(0xffffffffu, !ok || *abort_flag != 0u)) break;
                const uint8_t *src = sm + Cfg::STG + b * 16384;
                const int rows = (int)min((int64_t)C, len - (int64_t)m * C);
                if (rows == C) {
                    if (lane == 0) {
                        tma_store_3d(tm_o, src, 0, h, (int)(bos + (int64_t)m * C));
                        bulk_commit();
                        bulk_wait_read_all();
                    }
                } else {
#pragma unroll 4
                    for (int it = 0; it < 32; ++it) {
                        const int r = 2 * it + (lane >> 4), piece = lane & 15;
                        if (r < rows) {
                            const uint4 v = *reinterpret_cast<const uint4 *>(src + r * 256 + piece * 16);
                            *reinterpret_cast<uint4 *>(p.o + ((size_t)(bos + (int64_t)m * C + r) * p.H + h) * DV +
                                                       piece * 8) = v;
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&STGE[b]);
            }
            if (lane == 0) bulk_wait_all();
        } else if (stage_states && lane == 0 && nchunks > 0) {
            // the state tile (two 16 KB halves over j) of each chunk
            for (int n = 0; n < nchunks; ++n) {
                mbar_wait(&STGF[0], n & 1, abort_flag);
                if (*abort_flag) break;
                const int nn = REV ? nchunks - 1 - n : n;
                bulk_store(p.states_out + ((rec0 + nn) * p.H + h) * (size_t)32768, sm + Cfg::STG, 32768);
                bulk_commit();
                bulk_wait_read_all();
                mbar_arrive(&STGE[0]);
            }
            bulk_wait_all();
        }
    } else if (warp == NCW + 1) {
        // ---------------------------------------------- tensor-core products
        // N = 192 where the output products ride along, else 128; the reverse
        // scan's B operands (MP and QP themselves) are read MN-major
        constexpr int NP = OUT ? 192 : 128;
        const uint32_t idS = idesc_bf16(128, NP, false, REV);   // A = SB^T (TMEM), B = [MP; QP]^T
        const uint32_t idP = idesc_bf16(128, NP, true, REV);    // A = V^T (MN-major), B = [YT; ZB]^T
        // The state-independent group of chunk m into [X | O^T][m mod 2], which
        // the chain warps read out (X and O^T) before their SREADY of chunk m - 1,
        // which this warp has passed.
        auto pre = [&](int m) {
            if (TRANS) return;
            const int sr = m % NSR, sv = m % NSV;
            const uint32_t slot = smem_addr(sm + Cfg::RR + sr * Cfg::R_STRIDE);
            const uint32_t aV = smem_addr(sm + Cfg::RV + sv * Cfg::V_STRIDE);
            const uint32_t d = tmem + Cfg::COL_XO + Cfg::XO_STRIDE * (uint32_t)(m & 1);
            mbar_wait(&FULLR[sr], (m / NSR) & 1, abort_flag);
            mbar_wait(&FULLV[sv], (m / NSV) & 1, abort_flag);
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)   // V^T [YT; ZB]^T, or dO^T QP  (K = t)
                mma_bf16_warp(d, smem_desc(aV + ks * 2048, 8192, 1024, kLayoutSW128),
                              REV ? smem_desc(slot + Cfg::R_QP + ks * 2048, Cfg::R_KATOM, 1024, kLayoutSW128)
                                  : smem_desc(slot + Cfg::R_YT + ks * 32, 16, 1024, kLayoutSW128),
                              idP, ks > 0 ? 1u : 0u);
            mma_commit_warp(&EMPTYV[sv]);
        };
        if (nchunks > 0) pre(0);
        for (int n = 0; n < nchunks; ++n) {
            const int sr = n % NSR;
            const uint32_t slot = smem_addr(sm + Cfg::RR + sr * Cfg::R_STRIDE);
            const uint32_t aSB = tmem + Cfg::COL_SB + 64u * (uint32_t)(n & 1);
            const uint32_t d = tmem + Cfg::COL_XO + Cfg::XO_STRIDE * (uint32_t)(n & 1);
            if (TRANS) mbar_wait(&FULLR[sr], (n / NSR) & 1, abort_flag);
            mbar_wait(SREADY, n & 1, abort_flag);
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)   // SB^T [MP; QP]^T, or GB^T MP  (K = c')
                mma_bf16_ts_warp(d, aSB + 8 * ks,
                                 REV ? smem_desc(slot + Cfg::R_MP + ks * 2048, Cfg::R_KATOM, 1024, kLayoutSW128)
                                     : smem_desc(slot + Cfg::R_MP + (ks >> 2) * Cfg::R_KATOM + (ks & 3) * 32, 16,
                                                 1024, kLayoutSW128),
                                 idS, (TRANS && ks == 0) ? 0u : 1u);
            mma_commit_warp(SDONE);
            mma_commit_warp(&EMPTYR[sr]);
            if (n + 1 < nchunks) pre(n + 1);
        }
        if (nchunks > 0) {   // every arrive of the commits above lands before the CTA exits
            mma_commit_warp(FIN);
            wait_drain(FIN, 0);
        }
    } else {
        // ---------------------------------------------- the state chain
        const int quad = warp & 3;
        const int g = (warp - 1) >> 2;
        const int j = 32 * quad + lane;
        const size_t sbase = ((size_t)seq * p.H + h) * (size_t)(DK * DV) + (size_t)(32 * g) * DV + j;
        float S[32];
        if (TRANS) {   // the identity: S[c][j] = (c == j)
#pragma unroll
            for (int i = 0; i < 32; ++i) S[i] = (32 * g + i == j) ? 1.f : 0.f;
        } else if (p.init_state) {
#pragma unroll
            for (int i = 0; i < 32; ++i) S[i] = p.init_state[sbase + (size_t)i * DV];
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) S[i] = 0.f;
        }
        // O^T of chunk m (this warp's 16 t columns, lane j), read out with X_m,
        // into staging buffer m mod 2 as o rows [t][j]; the buffer's previous
        // rows (chunk m - 2) have been copied out once STGE says so
        float ov[16];
        auto stage_o = [&](int m) {
            const int b = m & 1;
            if (m >= 2) mbar_wait(&STGE[b], ((m - 2) >> 1) & 1, abort_flag);
            __nv_bfloat16 *st = reinterpret_cast<__nv_bfloat16 *>(sm + Cfg::STG + b * 16384) + (16 * g) * DV + j;
#pragma unroll
            for (int i = 0; i < 16; ++i) st[i * DV] = __float2bfloat16(ov[i]);
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&STGF[b]);
        };
        for (int n = 0; n < nchunks; ++n) {
            // SB_n^T: column COL_SB + 64 (n mod 2) + c / 2 holds (c, c + 1).  Its
            // previous contents, SB_{n-2}, were last read by chunk n - 2's
            // products, which completed before SDONE of chunk n - 1.
            uint32_t w16[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) w16[i] = pack_bf16x2(S[2 * i], S[2 * i + 1]);
            tmem_st16u(tmem_addr(tmem, 32 * quad, Cfg::COL_SB + 64 * (n & 1) + 16 * g), w16);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(SREADY);
            if (stage_states) {   // the state entering (forward) or leaving (reverse) this chunk
                if (n >= 1) mbar_wait(&STGE[0], (n - 1) & 1, abort_flag);
                uint8_t *tile = sm + Cfg::STG + (j >> 6) * 16384;
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    *reinterpret_cast<__nv_bfloat16 *>(tile + sw128_off(32 * g + i, j & 63)) = __float2bfloat16(S[i]);
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&STGF[0]);
            }
            if (OUT && n >= 1) stage_o(n - 1);
            // S_{n+1} = S_n Diag(exp(G_L)) + X_n, in two halves of 16 columns
            const int se = n % NSE;
            mbar_wait(&FULLE[se], (n / NSE) & 1, abort_flag);
            mbar_wait(SDONE, n & 1, abort_flag);
            tc_fence_after();
            const float4 *egl = reinterpret_cast<const float4 *>(sm + Cfg::EGLR + se * 512) + 8 * g;
            const uint32_t xo = Cfg::COL_XO + Cfg::XO_STRIDE * (n & 1);
            float x0[16], x1[16];   // X's two halves (and O^T) in one round trip
            tmem_ld16(tmem_addr(tmem, 32 * quad, xo + 32 * g), x0);
            tmem_ld16(tmem_addr(tmem, 32 * quad, xo + 32 * g + 16), x1);
            if (OUT) tmem_ld16(tmem_addr(tmem, 32 * quad, xo + Cfg::COL_O + 16 * g), ov);
            tmem_wait_ld();
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const float *x = hh ? x1 : x0;
#pragma unroll
                for (int e4 = 0; e4 < 4; ++e4) {
                    const float4 d = egl[4 * hh + e4];
                    float *s = S + 16 * hh + 4 * e4;
                    s[0] = fmaf(s[0], d.x, x[4 * e4 + 0]);
                    s[1] = fmaf(s[1], d.y, x[4 * e4 + 1]);
                    s[2] = fmaf(s[2], d.z, x[4 * e4 + 2]);
                    s[3] = fmaf(s[3], d.w, x[4 * e4 + 3]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&EMPTYE[se]);
        }
        if (OUT && nchunks > 0) stage_o(nchunks - 1);
        if (p.final_state) {
#pragma unroll
            for (int i = 0; i < 32; ++i) p.final_state[sbase + (size_t)i * DV] = S[i];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::TMEM_COLS);
    }
    if (tid == 0 && *abort_flag) atomicOr(p.err_word, kDevErrTimeout);
}

template <int MODE>
__global__ void __launch_bounds__(ChainT::THREADS, 1)
kda_chain_t_kernel(const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                   const Params p) {
    chain_t_unit<MODE>(tm_v, &tm_o, p, (int)blockIdx.x);
}

// The backward pass's two scans in one grid: CTAs [0, units) run the forward
// scan (each chunk's entering state), CTAs [units, 2 units) the reverse one
// (dL/dS at each chunk's end); they share only the records, which both read.
__global__ void __launch_bounds__(ChainT::THREADS, 1)
kda_backward_scans_kernel(const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                          const Params pf, const Params pr, int units) {
    if ((int)blockIdx.x < units) chain_t_unit<kChainSaveS>(tm_v, nullptr, pf, (int)blockIdx.x);
    else chain_t_unit<kChainReverse>(tm_do, nullptr, pr, (int)blockIdx.x - units);
}

// A segment's two local chains for context parallelism in one grid: CTAs
// [0, units) run the chain from a zero state with v (the state the segment
// generates), CTAs [units, 2 units) from the identity with v counting as zero
// (its transition); both over the same records, neither writing o.
__global__ void __launch_bounds__(ChainT::THREADS, 1)
kda_cp_local_chains_kernel(const __grid_constant__ CUtensorMap tm_v, const Params pl, const Params pt,
                           int units) {
    if ((int)blockIdx.x < units) chain_t_unit<kChainSaveS>(tm_v, nullptr, pl, (int)blockIdx.x);
    else chain_t_unit<kChainTransition>(tm_v, nullptr, pt, (int)blockIdx.x - units);
}

// =============================================================== layer prologue
// The layer's activations as the operator's inputs: log_alpha = -e^{A_log[h]}
// softplus(z) and beta = sigmoid(logit) in bf16, and the inverse L2 norms
// rsqrt(sum x^2 + eps) of every k and q row in fp32 ([row][k, q]); the
// preparation reads the raw q and k and scales every operand by the norms, so
// the normalised rows are never written out.  A half-warp per (token, head) row
// of 128 channels (16-byte pieces, eight channels per lane).  A pass of its own
// ahead of the operator: inside the chunk preparation the same arithmetic sat
// on that kernel's latency-bound path, while as a stream over the activations
// it is bound by HBM.
constexpr int kProThreads = 256;

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &w, float (&x)[8]) {
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 h2 = *reinterpret_cast<const __nv_bfloat162 *>(&ww[e]);
        x[2 * e] = __low2float(h2);
        x[2 * e + 1] = __high2float(h2);
    }
}

__device__ __forceinline__ uint4 f32x8_to_bf16(const float (&x)[8], float s) {
    uint4 w;
    w.x = pack_bf16x2(x[0] * s, x[1] * s);
    w.y = pack_bf16x2(x[2] * s, x[3] * s);
    w.z = pack_bf16x2(x[4] * s, x[5] * s);
    w.w = pack_bf16x2(x[6] * s, x[7] * s);
    return w;
}

__global__ void __launch_bounds__(kProThreads)
kda_layer_prologue_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                          const __nv_bfloat16 *__restrict__ z, const __nv_bfloat16 *__restrict__ blogit,
                          const float *__restrict__ A_log, float eps, int H, int64_t rows,
                          float *__restrict__ nrm, __nv_bfloat16 *__restrict__ la,
                          __nv_bfloat16 *__restrict__ bt) {
    const int lane = threadIdx.x & 31, sub = lane & 15;
    // a warp's two rows (half-warps); the shuffles take all 32 lanes, so a row
    // past the end is masked, not skipped
    const int64_t row = ((int64_t)blockIdx.x * (kProThreads / 32) + (threadIdx.x >> 5)) * 2 + (lane >> 4);
    const bool valid = row < rows;
    const size_t at = (size_t)row * 16 + sub;
    uint4 qv = make_uint4(0u, 0u, 0u, 0u), kv = qv, zv = qv;
    if (valid) {
        qv = reinterpret_cast<const uint4 *>(q)[at];
        kv = reinterpret_cast<const uint4 *>(k)[at];
        zv = reinterpret_cast<const uint4 *>(z)[at];
    }
    float xq[8], xk[8], xz[8];
    bf16x8_to_f32(qv, xq);
    bf16x8_to_f32(kv, xk);
    bf16x8_to_f32(zv, xz);
    float sq = 0.f, sk = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        sq = fmaf(xq[e], xq[e], sq);
        sk = fmaf(xk[e], xk[e], sk);
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) {   // within the half-warp
        sq += __shfl_xor_sync(0xffffffffu, sq, off);
        sk += __shfl_xor_sync(0xffffffffu, sk, off);
    }
    if (!valid) return;
    const float c = -__expf(A_log[row % H]);
#pragma unroll
    for (int e = 0; e < 8; ++e)   // softplus as the in-kernel prologue takes it
        xz[e] = c * (xz[e] > 15.f ? xz[e] : __logf(1.f + __expf(xz[e])));
    reinterpret_cast<uint4 *>(la)[at] = f32x8_to_bf16(xz, 1.f);
    if (sub == 0) {
        reinterpret_cast<float2 *>(nrm)[row] = make_float2(rsqrtf(sk + eps), rsqrtf(sq + eps));
        bt[row] = __float2bfloat16(1.f / (1.f + __expf(-__bfloat162float(blogit[row]))));
    }
}

// =============================================================== layer epilogue
// o <- o / sqrt(mean_j o_j^2 + eps) * w_j * sigmoid(g_j) per (token, head) row,
// in place after the chain: a half-warp per row of 128 (eight channels per
// lane, 16-byte pieces).  A pass of its own: inside the chain's loop the same
// work sat on the serial state path (about 1.5 us per chunk); here it is a
// stream over o and the gate.
constexpr int kEpiThreads = 256;

__global__ void __launch_bounds__(kEpiThreads)
kda_layer_epilogue_kernel(__nv_bfloat16 *__restrict__ o, const __nv_bfloat16 *__restrict__ gate,
                          const float *__restrict__ w, float eps, int64_t rows) {
    const int lane = threadIdx.x & 31, sub = lane & 15;
    const int64_t row = ((int64_t)blockIdx.x * (kEpiThreads / 32) + (threadIdx.x >> 5)) * 2 + (lane >> 4);
    const bool valid = row < rows;   // masked, not skipped: the shuffles take all 32 lanes
    const size_t at = (size_t)row * (DV / 8) + sub;
    uint4 ov = make_uint4(0u, 0u, 0u, 0u), gv4 = ov;
    if (valid) {
        ov = reinterpret_cast<const uint4 *>(o)[at];
        if (gate) gv4 = reinterpret_cast<const uint4 *>(gate)[at];
    }
    float x[8], gv[8];
    bf16x8_to_f32(ov, x);
    bf16x8_to_f32(gv4, gv);
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if (!valid) return;
    const float r = rsqrtf(ss * (1.f / DV) + eps);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        x[e] *= r * (w ? w[8 * sub + e] : 1.f);
        if (gate) x[e] *= 1.f / (1.f + __expf(-gv[e]));
    }
    reinterpret_cast<uint4 *>(o)[at] = f32x8_to_bf16(x, 1.f);
}

// =============================================================== plan kernel
// One CTA: checks cu_seqlens (error word), counts each sequence's chunks,
// writes the record offset of every sequence (exclusive prefix sum), the
// first token and length of every record's chunk, the record count, and the longest-first
// sequence order used by the chain kernel.
constexpr int kPlanThreads = 1024;
constexpr int kMaxSortedSeqs = 4096;

__device__ __forceinline__ int64_t seq_len_checked(const int32_t *cu, int i, int n, int64_t total) {
    if (!cu) return total / n;
    const int64_t a = cu[i], b = cu[i + 1];
    return (a < 0 || b < a || b > total) ? 0 : b - a;
}

__global__ void __launch_bounds__(kPlanThreads)
kda_split_plan_kernel(const int32_t *cu, int n, int64_t total, int32_t *perm, int32_t *chunk_off,
                      int2 *chunk_tab, uint32_t *total_chunks, uint32_t *err,
                      uint32_t *rec_ready, size_t n_flags, uint32_t *work_next) {
    // The prep grid may start its set-up now; it reads nothing of this
    // grid's output before this grid has completed.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    for (size_t i = threadIdx.x; i < n_flags; i += kPlanThreads) rec_ready[i] = 0u;
    if (threadIdx.x == 0) *work_next = 0u;
    __shared__ int32_t warp_sums[kPlanThreads / 32];
    __shared__ int32_t carry_s;
    // up to kMaxSortedSeqs sequences, cu_seqlens and the chunk offsets are
    // worked on in shared memory (one read of cu, no global round trips)
    __shared__ int32_t s_cu[kMaxSortedSeqs + 1], s_off[kMaxSortedSeqs + 1];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const bool small = n <= kMaxSortedSeqs;
    if (cu && small)
        for (int i = tid; i <= n; i += kPlanThreads) s_cu[i] = cu[i];
    __syncthreads();
    const int32_t *cuv = (cu && small) ? s_cu : cu;
    int32_t *offv = small ? s_off : chunk_off;
    int bad = 0;
    if (cu) {
        for (int i = tid; i < n; i += kPlanThreads) {
            const int64_t a = cuv[i], b = cuv[i + 1];
            if (a < 0 || b < a || b > total) bad = 1;
        }
        if (tid == 0 && (cuv[0] != 0 || cuv[n] != total)) bad = 1;
    }
    bad = __syncthreads_or(bad);
    if (tid == 0) {
        *err = bad ? kDevErrCuSeqlens : kDevErrNone;
        carry_s = 0;
    }
    __syncthreads();
    // exclusive scan of the chunk counts, 1024 sequences at a time
    for (int base = 0; base < n; base += kPlanThreads) {
        const int i = base + tid;
        const int cnt = (i < n) ? (int)((seq_len_checked(cuv, i, n, total) + C - 1) / C) : 0;
        int incl = cnt;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        if (lane == 31) warp_sums[wid] = incl;
        __syncthreads();
        if (wid == 0) {
            int w = warp_sums[lane];
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, w, off);
                if (lane >= off) w += y;
            }
            warp_sums[lane] = w;   // inclusive over warps
        }
        __syncthreads();
        const int carry = carry_s;
        const int excl = carry + (wid > 0 ? warp_sums[wid - 1] : 0) + incl - cnt;
        if (i < n) offv[i] = excl;
        __syncthreads();
        if (tid == kPlanThreads - 1) carry_s = excl + cnt;
        __syncthreads();
    }
    const int nchunks = carry_s;
    if (tid == 0) {
        offv[n] = nchunks;
        *total_chunks = (uint32_t)nchunks;
    }
    __syncthreads();
    if (small)
        for (int i = tid; i <= n; i += kPlanThreads) chunk_off[i] = s_off[i];
    for (int c = tid; c < nchunks; c += kPlanThreads) {
        int lo = 0, hi = n;   // last sequence i with chunk_off[i] <= c
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (offv[mid] <= c) lo = mid;
            else hi = mid;
        }
        const int64_t bos = cu ? (int64_t)cuv[lo] : (int64_t)lo * (total / n);
        const int64_t t0 = bos + (int64_t)(c - offv[lo]) * C;
        const int64_t len = seq_len_checked(cuv, lo, n, total);
        chunk_tab[c] = make_int2((int)t0, (int)min((int64_t)C, bos + len - t0));
    }
    if (!perm) return;
    for (int i = tid; i < n; i += kPlanThreads) {
        if (n > kMaxSortedSeqs) {
            perm[i] = i;
            continue;
        }
        const int64_t li = seq_len_checked(cuv, i, n, total);
        int r = 0;
        for (int j = 0; j < n; ++j) {
            const int64_t lj = seq_len_checked(cuv, j, n, total);
            r += (lj > li) || (lj == li && j < i);
        }
        perm[r] = i;
    }
}

}  // namespace split

// ---- host side -------------------------------------------------------------------

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's encoder, looked up once per process (a function-local static
// is initialised once even when several threads arrive together).
EncodeTiledFn encode_fn_split() {
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

bool make_map_split(CUtensorMap *m, const void *base, int64_t T, int H, int inner, int box_inner,
                    CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encode_fn_split();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)H, (cuuint64_t)T};
    const cuuint64_t strides[2] = {(cuuint64_t)inner * 2, (cuuint64_t)inner * 2 * H};
    const cuuint32_t box[3] = {(cuuint32_t)box_inner, 1, (cuuint32_t)split::C};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct SplitLayout {
    size_t perm, chunk_off, chunk_tab, flags, recs, total;
    size_t max_chunks;
};

SplitLayout split_layout(int num_seqs, int64_t total_tokens, int H) {
    SplitLayout l;
    l.max_chunks = (size_t)(total_tokens / split::C) + (size_t)num_seqs;
    l.perm = kWorkspaceHeader;
    l.chunk_off = l.perm + round_up((size_t)num_seqs * 4, 256);
    l.chunk_tab = l.chunk_off + round_up((size_t)(num_seqs + 1) * 4, 256);
    l.flags = round_up(l.chunk_tab + l.max_chunks * 8, 256);
    l.recs = round_up(l.flags + l.max_chunks * (size_t)H * 4, 1024);
    l.total = l.recs + l.max_chunks * (size_t)H * split::Rec::STRIDE;
    return l;
}

// The chain kernel for one slice width: grid = sequences x heads x slices.
// With `overlap` it is launched as a programmatic dependent of the prep grid.
template <int DVT>
cudaError_t launch_chain(const void *v, int64_t total_tokens, int H, const split::Params &prm,
                         unsigned units, bool overlap, cudaStream_t stream) {
    using namespace split;
    using Cfg = ChainCfg<DVT>;
    CUtensorMap mv;
    if (!make_map_split(&mv, v, total_tokens, H, DV, DVT == 32 ? 32 : 64,
                        DVT == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    {
        const cudaError_t e = set_max_dynamic_smem((const void *)kda_chain_kernel<DVT>, (int)Cfg::ALLOC);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(units * Cfg::NTILE);
    cfg.blockDim = dim3(Cfg::THREADS);
    cfg.dynamicSmemBytes = Cfg::ALLOC;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = overlap ? 1 : 0;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kda_chain_kernel<DVT>, mv, prm);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// The transposed whole-d_v chain: grid = sequences x heads.
cudaError_t launch_chain_t(const void *v, int64_t total_tokens, int H, const split::Params &prm,
                           unsigned units, bool overlap, cudaStream_t stream,
                           int mode = split::kChainPlain) {
    using namespace split;
    CUtensorMap mv, mo;
    if (!make_map_split(&mv, v, total_tokens, H, DV, 64, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (mode != kChainPlain) mo = mv;   // not read
    else if (!make_map_split(&mo, prm.o, total_tokens, H, DV, DV, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    {
        const void *fn = mode == kChainTransition ? (const void *)kda_chain_t_kernel<kChainTransition>
                         : mode == kChainSaveS    ? (const void *)kda_chain_t_kernel<kChainSaveS>
                         : mode == kChainReverse  ? (const void *)kda_chain_t_kernel<kChainReverse>
                                                  : (const void *)kda_chain_t_kernel<kChainPlain>;
        const cudaError_t e = set_max_dynamic_smem(fn, (int)ChainT::ALLOC);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(units);
    cfg.blockDim = dim3(ChainT::THREADS);
    cfg.dynamicSmemBytes = ChainT::ALLOC;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = overlap ? 1 : 0;
    const cudaError_t e =
        mode == kChainTransition ? cudaLaunchKernelEx(&cfg, kda_chain_t_kernel<kChainTransition>, mv, mo, prm)
        : mode == kChainSaveS    ? cudaLaunchKernelEx(&cfg, kda_chain_t_kernel<kChainSaveS>, mv, mo, prm)
        : mode == kChainReverse  ? cudaLaunchKernelEx(&cfg, kda_chain_t_kernel<kChainReverse>, mv, mo, prm)
                                 : cudaLaunchKernelEx(&cfg, kda_chain_t_kernel<kChainPlain>, mv, mo, prm);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// Chain slice width and overlap, from a cost model in SM cycles:
//   prep ~ items x c_p / (SMs it gets), c_p ~ 12 K cycles per (chunk, head)
//     per SM (two pipelines per SM, ~24 K cycles per item each);
//   chain ~ chunks per sequence x period when its CTAs fit on the GPU at
//     once, else (CTA-chunks x period / SMs); period ~ 1.6 K cycles for a
//     32-column slice and ~2.7 K for the whole d_v (a burst of N = 128
//     products costs little more per instruction than N = 32, so the wide
//     CTA does four times the work per chunk in under twice the time);
//   overlap (prep on the SMs the chain leaves free, chain consuming
//     records as they appear) costs the larger of the two, otherwise their
//     sum.
// Few (sequence, head) units and short chains favour narrow slices with
// overlap; many units or long chains the whole-d_v CTA.
struct ChainPlan {
    int dvt;
    bool overlap;
};

ChainPlan choose_chain(unsigned units, uint64_t items, int64_t total_tokens, int num_seqs,
                       unsigned sm_count, bool whole_dv_only) {
    const double c_p = 12e3, sm = (double)sm_count;
    const double chunks = (double)((total_tokens / num_seqs + split::C - 1) / split::C);
    ChainPlan best = {128, false};
    double best_cost = -1.0;
    const int widths[2] = {32, 128};
    for (int wi = whole_dv_only ? 1 : 0; wi < 2; ++wi) {
        const int dvt = widths[wi];
        const double per = dvt == 32 ? 1.6e3 : 2.7e3;
        const double ctas = (double)units * (split::DV / dvt);
        const double chain = ctas <= sm ? chunks * per : ctas * chunks * per / sm;
        for (int ov = 0; ov < 2; ++ov) {
            if (ov && ctas >= sm) continue;
            const double cost = ov ? fmax((double)items * c_p / (sm - ctas), chain)
                                   : (double)items * c_p / sm + chain;
            if (best_cost < 0.0 || cost < best_cost) {
                best_cost = cost;
                best.dvt = dvt;
                best.overlap = ov != 0;
            }
        }
    }
    return best;
}

}  // namespace

// A [T, H, inner] bf16 tensor as [64 tokens][box_inner] boxes (one head).
bool make_bf16_map_3d(CUtensorMap *m, const void *base, int64_t T, int H, int inner, int box_inner,
                      CUtensorMapSwizzle sw) {
    return make_map_split(m, base, T, H, inner, box_inner, sw);
}

// The layer path with its prologue as a pass of its own: the split
// workspace, then the prologue's outputs (log_alpha [T, H, 128] and beta
// [T, H] in bf16, the inverse norms [T, H, 2] in fp32), 256-byte aligned.
struct LayerLayout {
    size_t nrm, la, bt, total;
};

LayerLayout layer_layout(int num_seqs, int64_t total_tokens, int H) {
    LayerLayout l;
    const size_t tile = (size_t)total_tokens * H * 128 * sizeof(__nv_bfloat16);
    l.nrm = round_up(split_layout(num_seqs, total_tokens, H).total, 256);
    l.la = l.nrm + round_up((size_t)total_tokens * H * 2 * sizeof(float), 256);
    l.bt = l.la + round_up(tile, 256);
    l.total = l.bt + round_up((size_t)total_tokens * H * sizeof(__nv_bfloat16), 256);
    return l;
}

size_t layer_prefill_workspace(int num_seqs, int64_t total_tokens, int H) {
    return layer_layout(num_seqs, total_tokens, H).total;
}

cudaError_t launch_layer_prefill_split(const void *q, const void *k, const void *v, const LayerArgs &la,
                                       const float *init_state, const int32_t *cu, int num_seqs,
                                       int64_t total_tokens, int H, void *o, float *final_state,
                                       void *workspace, cudaStream_t stream) {
    using namespace split;
    const LayerLayout l = layer_layout(num_seqs, total_tokens, H);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    auto *nrm = reinterpret_cast<float *>(ws + l.nrm);
    auto *lg = reinterpret_cast<__nv_bfloat16 *>(ws + l.la);
    auto *bt = reinterpret_cast<__nv_bfloat16 *>(ws + l.bt);
    const int64_t rows = total_tokens * H;
    if (rows > 0) {
        const int64_t per = kProThreads / 16;   // rows per CTA
        kda_layer_prologue_kernel<<<(unsigned)((rows + per - 1) / per), kProThreads, 0, stream>>>(
            static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k),
            static_cast<const __nv_bfloat16 *>(la.gate_z), static_cast<const __nv_bfloat16 *>(la.beta_logit),
            la.A_log, la.qk_eps, H, rows, nrm, lg, bt);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    cudaError_t e = launch_prefill_split(q, k, v, lg, bt, init_state, cu, num_seqs, total_tokens, H, o,
                                         final_state, workspace, false, nullptr, stream, kCpNone, nullptr, nrm);
    if (e != cudaSuccess || rows == 0) return e;
    kda_layer_epilogue_kernel<<<(unsigned)((rows + kEpiThreads / 16 - 1) / (kEpiThreads / 16)), kEpiThreads, 0,
                                stream>>>(static_cast<__nv_bfloat16 *>(o),
                                          static_cast<const __nv_bfloat16 *>(la.out_gate), la.norm_weight,
                                          la.norm_eps, rows);
    return cudaGetLastError();
}

size_t prefill_split_workspace(int num_seqs, int64_t total_tokens, int H) {
    return split_layout(num_seqs, total_tokens, H).total;
}

SplitTables split_tables(const void *workspace, int num_seqs, int64_t total_tokens, int H) {
    const SplitLayout l = split_layout(num_seqs, total_tokens, H);
    const uint8_t *ws = static_cast<const uint8_t *>(workspace);
    SplitTables t;
    t.chunk_off = reinterpret_cast<const int32_t *>(ws + l.chunk_off);
    t.chunk_tab = reinterpret_cast<const int2 *>(ws + l.chunk_tab);
    t.total_chunks = reinterpret_cast<const uint32_t *>(ws + 4);
    t.recs = ws + l.recs;
    t.rec_stride = split::Rec::STRIDE;
    t.max_chunks = l.max_chunks;
    t.off_mp = split::Rec::MP;
    t.off_yt = split::Rec::YT;
    t.off_qp = split::Rec::QP;
    t.off_egl = split::Rec::EGL;
    return t;
}

cudaError_t launch_backward_scans(const void *v, const void *d_o, const float *init_state,
                                  const float *d_final_state, const int32_t *cu, int num_seqs,
                                  int64_t total_tokens, int H, void *workspace, void *s_in,
                                  void *ds_next, float *d_init_state, cudaStream_t stream) {
    using namespace split;
    const SplitLayout l = split_layout(num_seqs, total_tokens, H);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    Params prm = {};
    prm.cu = cu;
    prm.perm = cu ? reinterpret_cast<int32_t *>(ws + l.perm) : nullptr;
    prm.chunk_off = reinterpret_cast<int32_t *>(ws + l.chunk_off);
    prm.chunk_tab = reinterpret_cast<int2 *>(ws + l.chunk_tab);
    prm.total_chunks = reinterpret_cast<uint32_t *>(ws + 4);
    prm.recs = ws + l.recs;
    prm.rec_ready = nullptr;   // the preparation has completed
    prm.work_next = reinterpret_cast<uint32_t *>(ws + 8);
    prm.err_word = reinterpret_cast<uint32_t *>(ws);
    prm.total_tokens = total_tokens;
    prm.num_seqs = num_seqs;
    prm.H = H;
    const unsigned units = (unsigned)((size_t)num_seqs * H);
    // each chunk's entering state: the forward chain over the records
    Params pf = prm;
    pf.init_state = init_state;
    pf.final_state = nullptr;
    pf.states_out = static_cast<uint8_t *>(s_in);
    // dL/dS at each chunk's end: the reverse chain over the same records
    Params pr = prm;
    pr.init_state = d_final_state;
    pr.final_state = d_init_state;
    pr.states_out = static_cast<uint8_t *>(ds_next);
    // both at once, in one grid
    CUtensorMap mv, mdo;
    if (!make_map_split(&mv, v, total_tokens, H, DV, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_split(&mdo, d_o, total_tokens, H, DV, 64, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    cudaError_t e = set_max_dynamic_smem((const void *)kda_backward_scans_kernel, (int)ChainT::ALLOC);
    if (e != cudaSuccess) return e;
    if (units == 0) return cudaSuccess;
    kda_backward_scans_kernel<<<2 * units, ChainT::THREADS, ChainT::ALLOC, stream>>>(mv, mdo, pf, pr, (int)units);
    return cudaGetLastError();
}

cudaError_t launch_prefill_split(const void *q, const void *k, const void *v, const void *g,
                                 const void *beta, const float *init_state, const int32_t *cu,
                                 int num_seqs, int64_t total_tokens, int H, void *o,
                                 float *final_state, void *workspace, bool scalar_gate,
                                 const LayerArgs *layer, cudaStream_t stream, int cp_mode,
                                 float *cp_transition, const float *nrm_in) {
    using namespace split;
    const SplitLayout l = split_layout(num_seqs, total_tokens, H);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint32_t *err = reinterpret_cast<uint32_t *>(ws);
    uint32_t *total_chunks = reinterpret_cast<uint32_t *>(ws + 4);
    uint32_t *work_next = reinterpret_cast<uint32_t *>(ws + 8);
    int32_t *perm = cu ? reinterpret_cast<int32_t *>(ws + l.perm) : nullptr;
    int32_t *chunk_off = reinterpret_cast<int32_t *>(ws + l.chunk_off);
    int2 *chunk_tab = reinterpret_cast<int2 *>(ws + l.chunk_tab);
    if (cp_mode == kCpFinish) {
        // the records, chunk tables and sequence order are those a kCpLocal
        // call left in this workspace: only the chain runs, from init_state
        Params prm = {};
        prm.init_state = init_state;
        prm.final_state = final_state;
        prm.o = static_cast<__nv_bfloat16 *>(o);
        prm.cu = cu;
        prm.perm = perm;
        prm.chunk_off = chunk_off;
        prm.chunk_tab = chunk_tab;
        prm.total_chunks = total_chunks;
        prm.recs = ws + l.recs;
        prm.rec_ready = nullptr;
        prm.work_next = work_next;
        prm.err_word = err;
        prm.total_tokens = total_tokens;
        prm.num_seqs = num_seqs;
        prm.H = H;
        return launch_chain_t(v, total_tokens, H, prm, (unsigned)((size_t)num_seqs * H), false, stream);
    }

    CUtensorMap mk, mq, mg;
    if (!make_map_split(&mk, k, total_tokens, H, DK, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_split(&mq, q, total_tokens, H, DK, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        // with a scalar gate the map is never used (log_alpha comes in by plain loads)
        !make_map_split(&mg, scalar_gate ? k : g, total_tokens, H, DK, 128, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    // Prep runs as a persistent grid (one CTA per SM).  With overlap the prep
    // grid leaves the chain's SMs free and the chain kernel is launched as a
    // programmatic dependent of it, so that it starts at once and consumes
    // records as they are published; otherwise the two kernels run one after
    // the other and the records need no flags.
    const int sm_count = device_sm_count();
    const unsigned units = (unsigned)((size_t)num_seqs * H);
    // a segment's transition is d_k x d_k: whole-d_v chain CTAs only
    const ChainPlan plan = choose_chain(units, (uint64_t)(total_tokens / C + num_seqs) * H, total_tokens,
                                        num_seqs, (unsigned)sm_count, cp_mode == kCpLocal);
    // a segment's two local chains run side by side (twice the chain CTAs)
    const unsigned chain_blocks = units * (unsigned)(DV / plan.dvt) * (cp_mode == kCpLocal ? 2u : 1u);
    const bool overlap = (cp_mode == kCpLocal ? chain_blocks < (unsigned)sm_count : plan.overlap) &&
                         cp_mode != kPrepOnly;
    uint32_t *rec_ready = overlap ? reinterpret_cast<uint32_t *>(ws + l.flags) : nullptr;
    kda_split_plan_kernel<<<1, kPlanThreads, 0, stream>>>(cu, num_seqs, total_tokens, perm,
                                                          chunk_off, chunk_tab, total_chunks, err,
                                                          rec_ready, overlap ? l.max_chunks * (size_t)H : 0,
                                                          work_next);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = set_max_dynamic_smem((const void *)kda_prep_kernel<0, false>, (int)PrepSmem::ALLOC);
    if (e != cudaSuccess) return e;
    e = set_max_dynamic_smem((const void *)kda_prep_kernel<1, false>, (int)PrepSmem::ALLOC);
    if (e != cudaSuccess) return e;
    e = set_max_dynamic_smem((const void *)kda_prep_kernel<2, false>, (int)PrepSmem::ALLOC);
    if (e != cudaSuccess) return e;
    e = set_max_dynamic_smem((const void *)kda_prep_kernel<0, true>, (int)PrepSmem::ALLOC);
    if (e != cudaSuccess) return e;
    Params prm;
    prm.k = static_cast<const __nv_bfloat16 *>(k);
    prm.q = static_cast<const __nv_bfloat16 *>(q);
    prm.beta = static_cast<const __nv_bfloat16 *>(beta);
    prm.g = static_cast<const __nv_bfloat16 *>(g);
    prm.scalar_gate = scalar_gate ? 1 : 0;
    prm.layer = layer ? 1 : 0;
    prm.nrm_in = nrm_in;
    prm.A_log = layer ? layer->A_log : nullptr;
    prm.out_gate = layer ? static_cast<const __nv_bfloat16 *>(layer->out_gate) : nullptr;
    prm.norm_weight = layer ? layer->norm_weight : nullptr;
    prm.qk_eps = layer ? layer->qk_eps : 0.f;
    prm.norm_eps = layer ? layer->norm_eps : 0.f;
    prm.init_state = init_state;
    prm.final_state = final_state;
    prm.o = static_cast<__nv_bfloat16 *>(o);
    prm.cu = cu;
    prm.perm = perm;
    prm.chunk_off = chunk_off;
    prm.chunk_tab = chunk_tab;
    prm.total_chunks = total_chunks;
    prm.recs = ws + l.recs;
    prm.rec_ready = rec_ready;
    prm.work_next = work_next;
    prm.err_word = err;
    prm.total_tokens = total_tokens;
    prm.num_seqs = num_seqs;
    prm.H = H;
    const size_t max_items = l.max_chunks * (size_t)H;
    size_t prep_blocks = (size_t)(overlap ? sm_count - chain_blocks : sm_count);
    if (2 * prep_blocks > max_items) prep_blocks = (max_items + 1) / 2;
    {   // a programmatic dependent of the plan kernel: its set-up overlaps it
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)prep_blocks);
        cfg.blockDim = dim3(kPrepThreads);
        cfg.dynamicSmemBytes = PrepSmem::ALLOC;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = layer         ? cudaLaunchKernelEx(&cfg, kda_prep_kernel<1, false>, mk, mq, mg, prm)
            : nrm_in      ? cudaLaunchKernelEx(&cfg, kda_prep_kernel<2, false>, mk, mq, mg, prm)
            : scalar_gate ? cudaLaunchKernelEx(&cfg, kda_prep_kernel<0, true>, mk, mq, mg, prm)
                          : cudaLaunchKernelEx(&cfg, kda_prep_kernel<0, false>, mk, mq, mg, prm);
        if (e != cudaSuccess) return e;
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (cp_mode == kPrepOnly) return cudaSuccess;
    if (cp_mode == kCpLocal) {
        // the locally generated state (from zero) and, over the same records, the
        // segment's transition (from the identity, v counting as zero), in one
        // grid, consuming the records as the preparation publishes them
        Params pl = prm;
        pl.init_state = nullptr;
        pl.states_out = nullptr;
        Params pt = prm;
        pt.init_state = nullptr;
        pt.final_state = cp_transition;
        CUtensorMap mv;
        if (!make_map_split(&mv, v, total_tokens, H, DV, 64, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
        e = set_max_dynamic_smem((const void *)kda_cp_local_chains_kernel, (int)ChainT::ALLOC);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * units);
        cfg.blockDim = dim3(ChainT::THREADS);
        cfg.dynamicSmemBytes = ChainT::ALLOC;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = overlap ? 1 : 0;
        e = cudaLaunchKernelEx(&cfg, kda_cp_local_chains_kernel, mv, pl, pt, (int)units);
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    }
    e = plan.dvt == 32 ? launch_chain<32>(v, total_tokens, H, prm, units, overlap, stream)
                       : launch_chain_t(v, total_tokens, H, prm, units, overlap, stream);
    if (e != cudaSuccess || !layer) return e;
    const int64_t rows = total_tokens * H;
    kda_layer_epilogue_kernel<<<(unsigned)((rows + kEpiThreads / 16 - 1) / (kEpiThreads / 16)),
                                kEpiThreads, 0, stream>>>(
        static_cast<__nv_bfloat16 *>(o), static_cast<const __nv_bfloat16 *>(layer->out_gate),
        layer->norm_weight, layer->norm_eps, rows);
    return cudaGetLastError();
}

}  // namespace kda
