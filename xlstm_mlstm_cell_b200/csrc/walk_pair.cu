// walk_pair.cu -- the in-segment walk of the tensor-core forward pass at chunk 128, run by CTA pairs.
//
// The walk of fwd_tc.cu gives every 128 value columns of a head one CTA, and each of those CTAs
// computes the chunk's S = Q K^T, turns it into P and passes over Q and K on its own, the same work
// once per value tile.  Here two CTAs of a cluster (a tcgen05 CTA pair) share one chunk: the pair
// covers 256 value columns (128 per CTA, each holding its part of the state C^T in its own TMEM),
// and the work that does not depend on the value columns is split between the two CTAs instead of
// repeated:
//   * S = Q K^T is one pair MMA (M = 128: CTA r provides the 64 query rows 64r.. and the 64 keys
//     64r..; each CTA receives S of its 64 query rows over all 128 keys);
//   * each CTA turns its 64 rows of S into P (the causal decay matrix D of the xLSTM Guide's "The
//     Dual Formulation", restricted to the chunk) and scales its 64 rows of q (Q');
//   * H^T = C^T Q'^T + V^T P^T is one pair MMA (M = 256 value columns, N = the chunk's 128 tokens,
//     B columns from both CTAs), the inter-chunk term in tf32 straight from the fp32 state in TMEM;
//   * the state update C^T += V^T K' is one pair MMA whose B (K' = diag(W) K) is split by halves
//     of DK: each CTA scales its half of K and sums its half of the normalizer n.
// The two CTAs exchange, through distributed shared memory, their halves of n (for q . n) and the
// denominators of their 64 rows (the output epilogue of each CTA writes all 128 tokens of its value
// columns).  The per-token quantities are those of fwd_tc.cu's walk:
//   h_t = o_t * r_t H_t / max(|rowsum(P')_t r_t + sc_t q_t . n|, exp(-m_t)),
//   sc_t = exp(a_t + m_c - m_t) / sqrt(d) = r_t 2^e_t,  Q' = diag(2^e) Q (exact),  P' = diag(1/r) P,
// with the state in TMEM kept in the lazily rescaled frame of fwd_tc.cu.
//
// Roles of a CTA: a TMA producer warp; the MMA warp (in the leader CTA, the even rank, one thread
// issues every MMA of the pair; in the other CTA one thread relays its arrivals to the leader's
// barriers, so that the compute warps never wait on a cross-CTA release); sixteen compute warps that
// take the chunk's CUDA-core phases in turn, all sixteen on each: the Q pass first, so that the
// long tf32 part of the output MMA runs while they turn S into P'; the K pass while the rest of the
// output MMA runs; the denominators and the next chunk's gate factors; then the output epilogue,
// while the next chunk's S and this chunk's state update run.  Per-warp arrivals hand P', Q' and K' to the MMAs.
// The output gate tile is loaded by TMA into the half of the Q' buffer that the output MMA has
// finished reading, h replaces it in place and leaves by a TMA store.  Operand tiles that only
// MMAs read are loaded with TMA completions counted on the leader's barriers; every MMA completion
// is signalled to the barriers of both CTAs.  Every wait is bounded (the status word reports a
// timeout), and the pair meets at a cluster barrier before either CTA frees its TMEM or exits.
#include "common.cuh"
#include "mlstm_internal.h"
#include "tc_common.cuh"
#include "tc_fwd.h"
#include "tc_pair.cuh"

#include <cudaTypedefs.h>

namespace mlstm {
namespace tcfwd {

using namespace tc;

namespace pair {

constexpr int L = 128;        // chunk length
constexpr int HL = 64;        // query rows (and keys of the S operand) per CTA
constexpr int DVT = 128;      // value columns per CTA
constexpr float THRESH = 20.f;
constexpr float LOG2E = 1.4426950408889634f;
constexpr int THREADS = 64 + 16 * 32;   // producer warp, MMA warp, 16 compute warps
constexpr int GA = 512;                 // threads of the compute warps (warps 2..17)

// Optional timeline trace (build with -DMLSTM_WALK_TRACE): clock64 stamps of the roles of the CTA
// pair of value tiles 0 and 1, head 0, per segment and chunk (stamps of one CTA share its SM's
// clock; the two CTAs' clocks are not comparable).  Off in normal builds.
#ifdef MLSTM_WALK_TRACE
constexpr int PT_SLOTS = 32, PT_CHUNKS = 128, PT_SEGS = 64;
__device__ long long g_pair_trace[2 * PT_SEGS * PT_CHUNKS * PT_SLOTS];
#define PAIR_TRACE(slot, ci)                                                                                 \
    do {                                                                                                     \
        if (tile < 2 && bh == 0 && seg < PT_SEGS && (ci) < PT_CHUNKS)                                        \
            g_pair_trace[(((size_t)tile * PT_SEGS + seg) * PT_CHUNKS + (ci)) * PT_SLOTS + (slot)] = clock64(); \
    } while (0)
#else
#define PAIR_TRACE(slot, ci) do { } while (0)
#endif

template <int DK>
struct Smem {
    // operand tiles (128-byte swizzled blocks of 64 bf16 or 32 fp32 columns)
    static constexpr uint32_t QS = 0;                          // q, this CTA's 64 query rows [64][DK]
    static constexpr uint32_t QS_BYTES = HL * DK * 2;
    static constexpr uint32_t KS = QS + QS_BYTES;              // k, this CTA's 64 keys [64][DK]
    static constexpr uint32_t KS_BYTES = HL * DK * 2;
    static constexpr uint32_t KD = KS + KS_BYTES;              // k, all 128 keys, this CTA's half of DK
    static constexpr uint32_t KD_BYTES = L * (DK / 2) * 2;
    static constexpr uint32_t VS = KD + KD_BYTES;              // v, 128 keys x this CTA's 128 value columns
    static constexpr uint32_t VS_BYTES = L * DVT * 2;
    static constexpr uint32_t PS = VS + VS_BYTES;              // P', this CTA's 64 query rows x 128 keys
    static constexpr uint32_t PS_BYTES = HL * L * 2;
    static constexpr uint32_t Q32 = PS + PS_BYTES;             // Q' in fp32 (the tf32 operand) [64][DK]
    static constexpr uint32_t Q32_BYTES = HL * DK * 4;
    // the output tile (128 tokens x this CTA's 128 value columns, bf16, two 64-column swizzled
    // blocks): the output gate is loaded into it and h is stored from it, in the upper half of the
    // Q' buffer, which is free from the end of the output MMA until the next chunk's Q pass
    static constexpr uint32_t OS = Q32 + Q32_BYTES / 2;
    static constexpr uint32_t OS_BYTES = L * DVT * 2;
    static_assert(OS_BYTES <= Q32_BYTES / 2 && OS % 1024 == 0, "output tile");
    static constexpr uint32_t F = Q32 + Q32_BYTES;
    // floats: arow, mrow, icol, ccol, wcol, srow, qexp, rrow [L]; rs [8][HL]; dpart [8][HL];
    // bcol [8]; nX [2][DK]; inv [2][L]
    static constexpr uint32_t NF = 8 * L + 16 * HL + 8 + 2 * DK + 2 * L;
    static constexpr uint32_t BAR = F + ((NF * 4 + 7u) & ~7u);
    static constexpr uint32_t NBAR = 32;   // at least the barrier slots below
    static constexpr uint32_t TOTAL = BAR + NBAR * 8 + 16 + 1024;
    // TMEM columns: the state C^T (DK), H^T (128 tokens), two S buffers of 64 columns
    static constexpr uint32_t C_COL = 0, H_COL = DK, S_COL = DK + L;
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(S_COL + 128 <= TMEM_COLS, "TMEM columns");
    static_assert(TOTAL <= 232448, "shared memory");
};

// barrier slots
enum : int {
    B_QFULL = 0, B_KSFULL, B_VFULL,        // leader: TMA bytes of both CTAs
    B_KDFULL, B_OFULL,                     // local TMA
    B_QEMPTY,                              // the S MMA's commit and every compute warp's Q pass
    B_SFULL0, B_SFULL1, B_HFULL, B_CUPD, B_OSFREE,   // MMA completions (both CTAs)
    B_EPQ, B_EPP, B_KREADY, B_SFREE0, B_SFREE1,      // one arrival per compute warp (+ the relay's)
    B_HSFREE,                              // leader: one arrival from each CTA; other CTA: local
    B_NREADY0, B_NREADY1, B_INVREADY0, B_INVREADY1,  // bytes sent by the other CTA
    B_DRAIN
};
constexpr int NWARP = GA / 32;             // compute warps
static_assert(B_DRAIN < (int)Smem<256>::NBAR, "barrier slots");

// Named barrier that also ORs a predicate over the threads that meet there: every thread gets the
// same answer.
__device__ __forceinline__ bool named_sync_or(uint32_t id, uint32_t count, bool pred)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}

// One thread of a warp group waits on the barrier, then the group meets at its named barrier: the
// other warps wait there without taking issue slots from the warps that compute.  Returns false for
// every thread of the group alike once the CTA aborted (a bounded wait gave up), so that the group
// leaves its loop together.
__device__ __forceinline__ bool group_wait(uint64_t *bar, uint32_t parity, const WaitCtx &w, bool waiter,
                                           bool cluster_scope, uint32_t bar_id, uint32_t nthreads)
{
    if (waiter) {
        if (cluster_scope) mbar_wait_cluster(bar, parity, w);
        else mbar_wait(bar, parity, w);
    }
    return !named_sync_or(bar_id, nthreads, *reinterpret_cast<volatile uint32_t *>(w.abort) != 0u);
}

template <int DK>
__global__ void __launch_bounds__(THREADS, 1)
walk_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_ks,
                 const __grid_constant__ CUtensorMap tm_kd, const __grid_constant__ CUtensorMap tm_v,
                 const __grid_constant__ CUtensorMap tm_o, const __grid_constant__ CUtensorMap tm_h, Params p)
{
    using SM = Smem<DK>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *Qs = smem + SM::QS;
    uint8_t *Ks = smem + SM::KS;
    uint8_t *Kd = smem + SM::KD;
    uint8_t *Vs = smem + SM::VS;
    uint8_t *Ps = smem + SM::PS;
    uint8_t *Q32 = smem + SM::Q32;
    uint8_t *Os = smem + SM::OS;
    float *F = reinterpret_cast<float *>(smem + SM::F);
    float *arow = F, *mrow = F + L, *icol = F + 2 * L, *ccol = F + 3 * L, *wcol = F + 4 * L;
    float *srow = F + 5 * L, *qexp = F + 6 * L, *rrow = F + 7 * L;
    float *rs = F + 8 * L;                 // [8][HL] partial row sums of P' (one per 16-key block)
    float *dpart = rs + 8 * HL;            // [8][HL] partial q . n
    float *bcol = dpart + 8 * HL;          // [8] block maxima of icol (16-key blocks)
    float *nX = bcol + 8;                  // [2][DK] the normalizer (frame of the TMEM state)
    float *inv = nX + 2 * DK;              // [2][L] r_t / denominator of every token of the chunk
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + SM::NBAR);
    uint32_t *abort_flag = tmem_slot + 1;

    const uint32_t rank = cluster_ctarank();   // 0: the leader, which issues the pair's MMAs
    const bool leader = rank == 0;
    const uint32_t peer = rank ^ 1u;
    const int tile = blockIdx.x, seg = blockIdx.y, bh = blockIdx.z;
    const int j0 = tile * DVT;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c_begin = seg * p.R;
    const int nck = min(p.R, p.NC - c_begin);
    WaitCtx wc{abort_flag, p.status};

    if (threadIdx.x == 0) {
        // the leader's barriers also count the other CTA's (relayed) arrival
        const uint32_t wv = leader ? NWARP + 1 : NWARP, two = leader ? 2u : 1u;
        for (int b = 0; b <= B_DRAIN; ++b) {
            uint32_t c = 1;
            if (b == B_QEMPTY) c = 1 + NWARP;   // the S MMA's commit and the Q pass of every warp
            if (b == B_EPQ || b == B_EPP || b == B_KREADY || b == B_SFREE0 || b == B_SFREE1) c = wv;
            if (b == B_HSFREE) c = two;
            mbar_init(&bars[b], c);
        }
        *abort_flag = 0u;
        fence_barrier_init();
        tma_prefetch(&tm_q);
        tma_prefetch(&tm_ks);
        tma_prefetch(&tm_kd);
        tma_prefetch(&tm_v);
        if (p.o) tma_prefetch(&tm_o);
        tma_prefetch(&tm_h);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, SM::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    // both CTAs have initialized their barriers and allocated TMEM before either addresses the other
    cluster_arrive_release();
    cluster_wait_acquire();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // the producer loads only q, k, v and the MMA warp reads shared memory and TMEM: they start while
    // the preceding kernel may still run; the compute warps read its outputs and wait for them
    if (warp >= 2) griddep_wait();
    griddep_launch_dependents();

    if (warp == 0) {
        if (lane == 0) {   // TMA producer of this CTA
            const uint32_t lq = map_to_rank(&bars[B_QFULL], 0), lks = map_to_rank(&bars[B_KSFULL], 0);
            const uint32_t lv = map_to_rank(&bars[B_VFULL], 0);
            int nkd = 0;
            bool whole = true;
            // the output gate of chunk c into the output tile, once that chunk's output MMA has read
            // the half of the Q' buffer that holds it
            auto load_o = [&](int c) -> bool {
                if (!mbar_wait(&bars[B_OSFREE], (uint32_t)c & 1u, wc)) return false;
                PAIR_TRACE(12, c);
                mbar_arrive_expect_tx(&bars[B_OFULL], SM::OS_BYTES);
                for (int b = 0; b < DVT / 64; ++b)
                    tma_load_3d(Os + b * L * 128, &tm_o, j0 + b * 64, (c_begin + c) * L, bh, &bars[B_OFULL]);
                return true;
            };
            for (int i = 0; i < nck; ++i) {
                const int t0 = (c_begin + i) * L;
                const uint32_t pp = (uint32_t)(i - 1) & 1u;
                whole = false;
                // k rows of S first (free once S of the previous chunk is done), then q (free once the
                // Q pass of the previous chunk has read it)
                if (i > 0 && !mbar_wait(&bars[B_SFULL0 + ((i - 1) & 1)], (uint32_t)((i - 1) >> 1) & 1u, wc)) break;
                if (leader) mbar_arrive_expect_tx(&bars[B_KSFULL], 2 * SM::KS_BYTES);
                for (int b = 0; b < DK / 64; ++b)
                    tma_load_3d_pair(Ks + b * HL * 128, &tm_ks, b * 64, t0 + HL * (int)rank, bh, lks);
                if (i > 0 && !mbar_wait_cluster(&bars[B_QEMPTY], pp, wc)) break;
                PAIR_TRACE(20, i);
                if (leader) mbar_arrive_expect_tx(&bars[B_QFULL], 2 * SM::QS_BYTES);
                for (int b = 0; b < DK / 64; ++b)
                    tma_load_3d_pair(Qs + b * HL * 128, &tm_q, b * 64, t0 + HL * (int)rank, bh, lq);
                if (i > 0 && p.o && !load_o(i - 1)) break;
                // k and v tiles of the state update: free once the previous update is done
                if (i > 0 && !mbar_wait(&bars[B_CUPD], pp, wc)) break;
                mbar_arrive_expect_tx(&bars[B_KDFULL], SM::KD_BYTES);
                for (int b = 0; b < DK / 128; ++b)
                    tma_load_3d(Kd + b * L * 128, &tm_kd, (int)rank * (DK / 2) + b * 64, t0, bh, &bars[B_KDFULL]);
                ++nkd;
                PAIR_TRACE(21, i);
                if (leader) mbar_arrive_expect_tx(&bars[B_VFULL], 2 * SM::VS_BYTES);
                for (int b = 0; b < DVT / 64; ++b)
                    tma_load_3d_pair(Vs + b * L * 128, &tm_v, j0 + b * 64, t0, bh, lv);
                // the next chunk's tiles (and this chunk's output gate) into L2 now: their loads can
                // only start once the buffers are free, and then hit L2
                if (p.o)
                    for (int b = 0; b < DVT / 64; ++b) tma_prefetch_l2_3d(&tm_o, j0 + b * 64, t0, bh);
                if (i + 1 < nck) {
                    const int t1 = t0 + L;
                    for (int b = 0; b < DK / 64; ++b) {
                        tma_prefetch_l2_3d(&tm_q, b * 64, t1 + HL * (int)rank, bh);
                        tma_prefetch_l2_3d(&tm_ks, b * 64, t1 + HL * (int)rank, bh);
                    }
                    for (int b = 0; b < DK / 128; ++b)
                        tma_prefetch_l2_3d(&tm_kd, (int)rank * (DK / 2) + b * 64, t1, bh);
                    for (int b = 0; b < DVT / 64; ++b) tma_prefetch_l2_3d(&tm_v, j0 + b * 64, t1, bh);
                }
                whole = true;
            }
            if (whole && nck > 0 && p.o) load_o(nck - 1);
            if (nkd > 0) mbar_wait_drain(&bars[B_KDFULL], (uint32_t)(nkd - 1) & 1u);
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {   // MMA issuer of the pair
            constexpr uint32_t ID_S = idesc_bf16(2 * HL, L, 0, 0);     // S = Q K^T (M = 128 over the pair)
            constexpr uint32_t ID_HC = idesc_tf32(2 * DVT, L);          // H^T = C^T Q'^T (tf32, A in TMEM)
            constexpr uint32_t ID_HP = idesc_bf16(2 * DVT, L, 1, 0);    // H^T += V^T P'^T
            constexpr uint32_t ID_C = idesc_bf16(2 * DVT, DK, 1, 1);    // C^T += V^T K'
            // descriptors of the operand tiles, advanced by byte offsets in the loops (the issuing
            // thread shares its scheduler with busy compute warps: every instruction here counts)
            const uint64_t dQ = smem_desc(smem_u32(Qs), 16, 1024), dK = smem_desc(smem_u32(Ks), 16, 1024);
            const uint64_t dQ32 = smem_desc(smem_u32(Q32), 16, 1024), dP = smem_desc(smem_u32(Ps), 16, 1024);
            const uint64_t dV = smem_desc(smem_u32(Vs), L * 128, 1024), dKD = smem_desc(smem_u32(Kd), L * 128, 1024);
            // both CTAs' copies of the barriers that MMA completions arrive on
            struct Pair2 { uint32_t r0, r1; };
            auto both = [&](int bar) { return Pair2{map_to_rank(&bars[bar], 0), map_to_rank(&bars[bar], 1)}; };
            const Pair2 cSF0 = both(B_SFULL0), cSF1 = both(B_SFULL1), cQE = both(B_QEMPTY), cOS = both(B_OSFREE);
            const Pair2 cHF = both(B_HFULL), cCU = both(B_CUPD), cDR = both(B_DRAIN);
            auto commit2 = [&](const Pair2 &c) {
                mma_commit_to(c.r0);
                mma_commit_to(c.r1);
            };
            const uint32_t tS = tmem + SM::S_COL, tH = tmem + SM::H_COL, tC = tmem + SM::C_COL;
            auto issue_s = [&](int ci) -> bool {
                if (!mbar_wait(&bars[B_QFULL], (uint32_t)ci & 1u, wc)) return false;
                if (!mbar_wait(&bars[B_KSFULL], (uint32_t)ci & 1u, wc)) return false;
                // S buffer ci & 1 was read by both CTAs' S -> P of chunk ci - 2
                if (ci >= 2 && !mbar_wait(&bars[B_SFREE0 + (ci & 1)], (uint32_t)((ci >> 1) - 1) & 1u, wc))
                    return false;
                PAIR_TRACE(29, ci);
                tc_fence_after();
                const uint32_t sa = tS + (uint32_t)(ci & 1) * 64u;
#pragma unroll
                for (int k = 0; k < DK / 16; ++k) {
                    const uint32_t off = ((k >> 2) * HL * 128 + (k & 3) * 32) >> 4;
                    mma_pair_ss(sa, dQ + off, dK + off, ID_S, k > 0 ? 1u : 0u);
                }
                commit2((ci & 1) ? cSF1 : cSF0);   // (the producer's k rows of S are free then too)
                commit2(cQE);
                PAIR_TRACE(2, ci);
                return true;
            };
            bool run = nck > 0 && issue_s(0);
            for (int i = 0; i < nck && run; ++i) {
                const uint32_t ph = (uint32_t)i & 1u;
                // both CTAs: Q' is ready, the previous outputs are read
                if (!mbar_wait(&bars[B_EPQ], ph, wc)) break;
                if (i > 0 && !mbar_wait(&bars[B_HSFREE], ph ^ 1u, wc)) break;
                PAIR_TRACE(3, i);
                tc_fence_after();
                // H^T = C^T Q'^T, 8 tf32 (32 bytes of a 128-byte row) per step; the upper half of DK
                // first, whose Q' half then takes the output gate tile
#pragma unroll
                for (int kk = 0; kk < DK / 8; ++kk) {
                    const int k = (kk + DK / 16) % (DK / 8);
                    const uint32_t off = ((k >> 2) * HL * 128 + (k & 3) * 32) >> 4;
                    mma_pair_ts_tf32(tH, tC + k * 8, dQ32 + off, ID_HC, kk > 0 ? 1u : 0u);
                    if (kk == DK / 16 - 1) commit2(cOS);
                }
                PAIR_TRACE(28, i);
                // both CTAs: P' is ready
                if (!mbar_wait(&bars[B_EPP], ph, wc)) break;
                if (!mbar_wait(&bars[B_VFULL], ph, wc)) break;
                PAIR_TRACE(4, i);
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < L / 16; ++k) {   // H^T += V^T P'^T
                    const uint32_t poff = ((k >> 2) * HL * 128 + (k & 3) * 32) >> 4;
                    mma_pair_ss(tH, dV + ((k * 2048) >> 4), dP + poff, ID_HP, 1u);
                }
                commit2(cHF);
                PAIR_TRACE(5, i);
                if (i < nck - 1) {
                    // the next chunk's S first (its tiles arrived long ago): it is what the compute
                    // warps wait for next, the state update is needed only by the next output MMA
                    if (!issue_s(i + 1)) break;
                    if (!mbar_wait(&bars[B_KREADY], ph, wc)) break;
                    PAIR_TRACE(6, i);
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < L / 16; ++k)
                        mma_pair_ss(tC, dV + ((k * 2048) >> 4), dKD + ((k * 2048) >> 4), ID_C, 1u);
                    commit2(cCU);   // (the producer's V and K' tiles are free then too)
                    PAIR_TRACE(31, i);
                }
            }
            commit2(cDR);
        }
        if (!leader && lane == 0) {
            // relay of the compute warps' arrivals to the leader, in the order the compute warps make
            // them (one thread, so that no relay waits behind another's suspended wait)
            const uint32_t l_epq = map_to_rank(&bars[B_EPQ], 0), l_epp = map_to_rank(&bars[B_EPP], 0);
            const uint32_t l_kready = map_to_rank(&bars[B_KREADY], 0), l_hs = map_to_rank(&bars[B_HSFREE], 0);
            for (int i = 0; i < nck; ++i) {
                const uint32_t ph = (uint32_t)i & 1u;
                if (!mbar_wait(&bars[B_EPQ], ph, wc)) break;
                mbar_arrive_cluster(l_epq);
                if (!mbar_wait(&bars[B_EPP], ph, wc)) break;
                mbar_arrive_cluster(map_to_rank(&bars[B_SFREE0 + (i & 1)], 0));
                mbar_arrive_cluster(l_epp);
                if (i < nck - 1) {
                    if (!mbar_wait(&bars[B_KREADY], ph, wc)) break;
                    mbar_arrive_cluster(l_kready);
                }
                if (!mbar_wait(&bars[B_HSFREE], ph, wc)) break;
                mbar_arrive_cluster(l_hs);
            }
        }
        if (lane == 0) mbar_wait_cluster_drain(&bars[B_DRAIN], 0);   // every MMA of the pair has completed
    } else {
        // ------------------------------------------------ compute warps 2..17: four per TMEM lane quadrant
        //     One chunk at a time: S -> P', the Q pass, the K pass during the output MMA, the
        //     denominators, the next chunk's gate factors while the output MMA finishes, the output
        //     epilogue while the state update and the next S run.
        const int ct = threadIdx.x - 64;          // 0..511
        const int q = warp & 3;                   // TMEM lane quadrant
        const int cw = warp - 2;                  // 0..15
        const int hq = cw >> 2;                   // which quarter of the columns (or tokens)
        const float scale = rsqrtf((float)DK);
        const float *Ab = p.A + (size_t)bh * p.S;
        const float *Mb = p.Mtok + (size_t)bh * p.S;
        const float *igb = p.ig + (size_t)bh * p.S;
        const float *MCb = p.MC + (size_t)bh * (p.NC + 1);
        const float *Gb = p.G + (size_t)bh * p.NC;

        // the segment's start state -> TMEM (C^T of this CTA's value columns) and nX[0] (all of n)
        {
            const float *src = p.DC + ((size_t)bh * p.NSEG + seg) * (size_t)DK * p.DV;
            const int j = q * 32 + lane;
            for (int c0 = hq * (DK / 4); c0 < (hq + 1) * (DK / 4); c0 += 16) {
                uint32_t r[16];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float4 v4 = *reinterpret_cast<const float4 *>(src + ((size_t)((c0 >> 2) + u) * p.DV + j0 + j) * 4);
                    r[4 * u] = __float_as_uint(v4.x);
                    r[4 * u + 1] = __float_as_uint(v4.y);
                    r[4 * u + 2] = __float_as_uint(v4.z);
                    r[4 * u + 3] = __float_as_uint(v4.w);
                }
                tmem_st16(tmem_addr(tmem, q * 32, SM::C_COL + c0), r);
            }
            tmem_wait_st();
            for (int d = ct; d < DK; d += GA) nX[d] = p.DN[((size_t)bh * p.NSEG + seg) * DK + d];
        }

        // Gate factors of chunk i (into the shared arrays) and the chunk's scalars; `rho` is the frame
        // of the TMEM state at the chunk's start.  The inputs are loaded one chunk ahead.
        float rho = MCb[c_begin];
        float pa = 0.f, pm = 0.f, pi = 0.f;
        float pmc = MCb[c_begin], pmn = MCb[c_begin + 1], pg = Gb[c_begin];
        if (ct < L && c_begin * L + ct < p.S) {
            const int t = c_begin * L + ct;
            pa = Ab[t];
            pm = Mb[t];
            pi = igb[t];
        }
        float alpha = 0.f, beta = 1.f, rho_next = rho;
        bool rescale = false;
        auto gate_step = [&](int i) {
            const int c = c_begin + i;
            const int t0 = c * L;
            const int len = min(L, p.S - t0);
            const float mc = pmc, mn = pmn, g = pg;
            const float ca = pa, cm = pm, ci = pi;
            if (i + 1 < nck) {
                pmc = MCb[c + 1];
                pmn = MCb[c + 2];
                pg = Gb[c + 1];
                const int t = t0 + L + ct;
                if (ct < L && t < p.S) {
                    pa = Ab[t];
                    pm = Mb[t];
                    pi = igb[t];
                }
            }
            const bool last = (i == nck - 1);
            rescale = !last && (mn - (rho + g) > THRESH);
            const float rho_new = rescale ? (mn - g) : rho;
            alpha = expf(rho - mc);
            beta = expf(rho - rho_new);
            rho_next = rho_new + g;
            const float ahc = alpha;   // scale of the TMEM state as the tf32 product reads it (frame rho)
            if (ct < L) {
                if (ct < len) {
                    const float mt = ca + fmaxf(mc, cm);
                    arow[ct] = (ca - mt) * LOG2E;
                    mrow[ct] = mt;
                    icol[ct] = (ci - ca) * LOG2E;
                    const float sc = expf(ca + mc - mt) * scale;
                    srow[ct] = sc;
                    const float sct = sc * ahc;
                    int ex = 0;
                    const float fr = frexpf(sct, &ex);
                    qexp[ct] = sct > 0.f ? (float)(ex - 1) : -1000.f;
                    rrow[ct] = sct > 0.f ? 2.f * fr : 1.f;
                    wcol[ct] = last ? 0.f : expf(ci - ca - rho_new);
                } else {
                    arow[ct] = 0.f;
                    mrow[ct] = 0.f;
                    icol[ct] = -INFINITY;
                    srow[ct] = 0.f;
                    qexp[ct] = -1000.f;
                    rrow[ct] = 1.f;
                    wcol[ct] = 0.f;
                }
                // column factors for the 16-key blocks below the diagonal: 2^(icol - block max)
                const float ic = ct < len ? (ci - ca) * LOG2E : -INFINITY;
                float bm = ic;
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
                ccol[ct] = bm == -INFINITY ? 0.f : exp2f(ic - bm);
                if ((ct & 15) == 0) bcol[ct >> 4] = bm;
            }
        };
        if (nck > 0) gate_step(0);

        const __nv_bfloat16 *og = p.o;
        for (int i = 0; i < nck; ++i) {
            const int t0 = (c_begin + i) * L;
            const uint32_t ph = (uint32_t)i & 1u;
            const int b = i & 1;
            const bool last = (i == nck - 1);
            if (ct == 0) {
                PAIR_TRACE(8, i);
                // arm the barriers of what the other CTA sends during this chunk; their previous phases
                // completed before this CTA's outputs of chunk i - 1 were written, and the other CTA
                // cannot send into the next phase before this CTA's state update of chunk i
                if (!last) mbar_arrive_expect_tx(&bars[B_NREADY0 + ((i + 1) & 1)], (DK / 2) * 4);
                mbar_arrive_expect_tx(&bars[B_INVREADY0 + b], HL * 4);
            }
            // (b) S of this chunk is done (so q has landed) and the other CTA's half of n has arrived;
            //     the previous chunk's h store has read the upper half of the Q' buffer.  The group's
            //     barrier also orders the gate arrays written at the end of the previous chunk.
            if (ct == 0) {
                mbar_wait(&bars[B_SFULL0 + b], (uint32_t)(i >> 1) & 1u, wc);
            }
            if (!group_wait(&bars[B_NREADY0 + b], (uint32_t)((i >> 1) - 1 + b) & 1u, wc, ct == 0 && i > 0, true, 1, GA))
                break;
            if (ct == 0) PAIR_TRACE(10, i);
            tc_fence_after();

            // (c) Q pass over this CTA's 64 rows: q . n from the unscaled bf16 q (fp32) and Q' = 2^e q in
            //     fp32.  A thread takes the 16-byte chunks part + 8 u of its row: the lower half of DK
            //     first, then (once the previous chunk's h store has read it) the upper half.
            {
                constexpr int CPT = DK / 64;             // chunks of q per thread (8 threads per row)
                const int row = ct & (HL - 1), part = ct >> 6;
                const int qe = (int)qexp[HL * (int)rank + row];
                const float s2 = qe >= -126 ? __int_as_float((qe + 127) << 23) : 0.f;
                const uint64_t ss = f2_pack(s2, s2);
                const float *nb = nX + b * DK;
                uint64_t dot2 = 0ull;
                uint4 uq[CPT];
#pragma unroll
                for (int u = 0; u < CPT; ++u) uq[u] = *reinterpret_cast<const uint4 *>(Qs + sw128_chunk(row, part + 8 * u, HL));
                auto put = [&](int u) {
                    const int jc = part + 8 * u;
                    *reinterpret_cast<ulonglong2 *>(Q32 + sw128_chunk(row, 2 * jc, HL)) =
                        make_ulonglong2(f2_mul(f2_from_bf16x2(uq[u].x), ss), f2_mul(f2_from_bf16x2(uq[u].y), ss));
                    *reinterpret_cast<ulonglong2 *>(Q32 + sw128_chunk(row, 2 * jc + 1, HL)) =
                        make_ulonglong2(f2_mul(f2_from_bf16x2(uq[u].z), ss), f2_mul(f2_from_bf16x2(uq[u].w), ss));
                };
#pragma unroll
                for (int u = 0; u < CPT; ++u) {
                    const int jc = part + 8 * u;
                    const ulonglong2 na = *reinterpret_cast<const ulonglong2 *>(nb + jc * 8);
                    const ulonglong2 nn = *reinterpret_cast<const ulonglong2 *>(nb + jc * 8 + 4);
                    dot2 = f2_fma(f2_from_bf16x2(uq[u].x), na.x, dot2);
                    dot2 = f2_fma(f2_from_bf16x2(uq[u].y), na.y, dot2);
                    dot2 = f2_fma(f2_from_bf16x2(uq[u].z), nn.x, dot2);
                    dot2 = f2_fma(f2_from_bf16x2(uq[u].w), nn.y, dot2);
                    if (u < CPT / 2) put(u);
                }
                const float2 dd = f2_unpack(dot2);
                dpart[part * HL + row] = dd.x + dd.y;
                if (ct == 0) bulk_wait_read0();   // the previous chunk's h store has read the upper half
                named_sync(1, GA);
#pragma unroll
                for (int u = CPT / 2; u < CPT; ++u) put(u);
            }
            fence_proxy_async();
            tc_fence_before();   // (the segment's start state in TMEM)
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars[B_QEMPTY]);   // this warp has read q
                mbar_arrive(&bars[B_EPQ]);      // this warp's Q' is ready
            }
            if (ct == 0) PAIR_TRACE(13, i);

            // (d) S -> P' for this CTA's 64 query rows.  TMEM lane 32 q + lane holds query row
            //     m = 32 (q & 1) + lane over the keys [64 (q >> 1), +64) in the S buffer's 64 columns;
            //     warp quarter hq takes the 16-key block hq of those columns
            {
                const int len = min(L, p.S - t0);
                const int m = 32 * (q & 1) + lane;
                const int tau = HL * (int)rank + m;
                const int kh = q >> 1;
                const int kb = 4 * kh + hq;                  // 16-key block 0..7
                const int s0 = 16 * kb;                      // its first key
                const int rb = tau >> 4;
                const int rb_warp = (HL * (int)rank + 32 * (q & 1) + 31) >> 4;   // largest row block of the warp
                float v[16];
                if (kb <= rb_warp) {
                    uint32_t r[16];
                    tmem_ld16(tmem_addr(tmem + SM::S_COL + (uint32_t)b * 64u, q * 32, hq * 16), r);
                    tmem_wait_ld();
                    const float at = arow[tau];
                    if (kb < rb) {                           // row factor x column factor
                        const float rf = tau < len ? exp2f(at + bcol[kb]) * scale : 0.f;
#pragma unroll
                        for (int z = 0; z < 16; ++z) v[z] = __uint_as_float(r[z]) * (ccol[s0 + z] * rf);
                    } else if (kb == rb) {                   // diagonal block: per element, causal mask
#pragma unroll
                        for (int z = 0; z < 16; ++z) {
                            float d = exp2f(at + icol[s0 + z]);
                            if (s0 + z > tau) d = 0.f;
                            v[z] = __uint_as_float(r[z]) * d * scale;
                        }
                    } else {
#pragma unroll
                        for (int z = 0; z < 16; ++z) v[z] = 0.f;
                    }
                } else {
#pragma unroll
                    for (int z = 0; z < 16; ++z) v[z] = 0.f;
                }
                float sum = 0.f;
#pragma unroll
                for (int z = 0; z < 16; z += 4) sum += (v[z] + v[z + 1]) + (v[z + 2] + v[z + 3]);
                rs[kb * HL + m] = sum;
                const float ri = 1.f / rrow[tau];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const float *w8 = v + 8 * hh;
                    *reinterpret_cast<uint4 *>(Ps + sw128_chunk(m, 2 * kb + hh, HL)) =
                        make_uint4(pack_bf16(w8[0] * ri, w8[1] * ri), pack_bf16(w8[2] * ri, w8[3] * ri),
                                   pack_bf16(w8[4] * ri, w8[5] * ri), pack_bf16(w8[6] * ri, w8[7] * ri));
                }
            }
            fence_proxy_async();
            tc_fence_before();   // (the S reads)
            __syncwarp();
            if (lane == 0) {
                if (leader) mbar_arrive(&bars[B_SFREE0 + b]);   // (the other CTA's relay does both)
                mbar_arrive(&bars[B_EPP]);                      // this warp's P' is ready
            }
            if (ct == 0) PAIR_TRACE(11, i);

            // (e) while the output MMA runs: K pass over this CTA's half of DK.  n sums W k from the
            //     unscaled bf16 k (fp32) and K' = W k in bf16 in place; warp cw owns the 16-byte column
            //     cw of every key row (lane = key), so its n sums reduce inside the warp.  The group's
            //     barrier also orders the partial sums of (c) and (d) for the denominators.
            if (!group_wait(&bars[B_KDFULL], ph, wc, ct == 0 && !last, false, 1, GA)) break;
            if (!last) {
                if (ct == 0) PAIR_TRACE(14, i);
                uint64_t nacc2[4];
#pragma unroll
                for (int z = 0; z < 4; ++z) nacc2[z] = 0ull;
                uint4 uk[L / 32];
#pragma unroll
                for (int rg = 0; rg < L / 32; ++rg) uk[rg] = *reinterpret_cast<const uint4 *>(Kd + sw128_chunk(rg * 32 + lane, cw, L));
#pragma unroll
                for (int rg = 0; rg < L / 32; ++rg) {
                    const int row = rg * 32 + lane;
                    const float w = wcol[row];
                    const uint64_t ww = f2_pack(w, w);
                    const uint64_t k0 = f2_from_bf16x2(uk[rg].x), k1 = f2_from_bf16x2(uk[rg].y),
                                   k2 = f2_from_bf16x2(uk[rg].z), k3 = f2_from_bf16x2(uk[rg].w);
                    nacc2[0] = f2_fma(ww, k0, nacc2[0]);
                    nacc2[1] = f2_fma(ww, k1, nacc2[1]);
                    nacc2[2] = f2_fma(ww, k2, nacc2[2]);
                    nacc2[3] = f2_fma(ww, k3, nacc2[3]);
                    *reinterpret_cast<uint4 *>(Kd + sw128_chunk(row, cw, L)) =
                        make_uint4(f2_to_bf16x2(f2_mul(k0, ww)), f2_to_bf16x2(f2_mul(k1, ww)),
                                   f2_to_bf16x2(f2_mul(k2, ww)), f2_to_bf16x2(f2_mul(k3, ww)));
                }
                fence_proxy_async();
                __syncwarp();
                // A frame move rescales this warp's part of the state once the output MMA, which reads
                // the state in the chunk's starting frame, has completed, and before the update adds
                // the chunk's tokens in the new frame.  (One fp32 frame cannot serve both ends of a
                // chunk whose log decay is in the hundreds: exp(rho_new - m_c) overflows while
                // exp(rho - rho_new) underflows.)
                if (rescale) {
                    uint32_t done = 1u;
                    if (lane == 0) done = mbar_wait(&bars[B_HFULL], ph, wc) ? 1u : 0u;
                    if (__shfl_sync(0xffffffffu, done, 0)) {   // (aborted: (g) leaves the loop)
                        tc_fence_after();
#pragma unroll 1
                        for (int c0 = hq * (DK / 4); c0 < (hq + 1) * (DK / 4); c0 += 16) {
                            uint32_t r[16];
                            tmem_ld16(tmem_addr(tmem, q * 32, SM::C_COL + c0), r);
                            tmem_wait_ld();
#pragma unroll
                            for (int u = 0; u < 16; ++u) r[u] = __float_as_uint(__uint_as_float(r[u]) * beta);
                            tmem_st16(tmem_addr(tmem, q * 32, SM::C_COL + c0), r);
                        }
                        tmem_wait_st();
                        tc_fence_before();
                    }
                }
                if (lane == 0) mbar_arrive(&bars[B_KREADY]);   // this warp's K' is ready
                float nacc[8];
#pragma unroll
                for (int z = 0; z < 4; ++z) {
                    const float2 v = f2_unpack(nacc2[z]);
                    nacc[2 * z] = v.x;
                    nacc[2 * z + 1] = v.y;
                }
                // transposed reduction over the 32 lanes: lane l ends with the sum of value l / 4
                int nv = 8;
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) {
                    if (nv > 1) {
                        const bool up = (lane & o) != 0;
                        const int h = nv / 2;
#pragma unroll
                        for (int z = 0; z < 4; ++z) {
                            if (z < h) {
                                const float send = up ? nacc[z] : nacc[z + h];
                                const float keep = up ? nacc[z + h] : nacc[z];
                                nacc[z] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                            }
                        }
                        nv = h;
                    } else {
                        nacc[0] += __shfl_xor_sync(0xffffffffu, nacc[0], o);
                    }
                }
                if ((lane & 3) == 0) {   // this CTA's half of n for the next chunk, here and in the other CTA
                    const int d = (int)rank * (DK / 2) + cw * 8 + (lane >> 2);
                    const float nn = nX[b * DK + d] * beta + nacc[0];
                    float *dst = nX + ((i + 1) & 1) * DK + d;
                    *dst = nn;
                    st_async_f32(map_to_rank(dst, peer), nn, map_to_rank(&bars[B_NREADY0 + ((i + 1) & 1)], peer));
                }
                if (ct == 0) PAIR_TRACE(15, i);
            }
            // (f) r / denominator of this CTA's 64 tokens, here and in the other CTA
            if (ct < HL) {
                const int tau = HL * (int)rank + ct;
                float qn = 0.f, rsum = 0.f;
#pragma unroll
                for (int k8 = 0; k8 < 8; ++k8) {
                    qn += dpart[k8 * HL + ct];
                    rsum += rs[k8 * HL + ct];
                }
                const float den = rsum + qn * alpha * srow[tau];
                const float iv = rrow[tau] / fmaxf(fabsf(den), expf(-mrow[tau]));
                float *dst = inv + b * L + tau;
                *dst = iv;
                st_async_f32(map_to_rank(dst, peer), iv, map_to_rank(&bars[B_INVREADY0 + b], peer));
            }
            if (ct == 0) PAIR_TRACE(9, i);
            named_sync(1, GA);   // the gate arrays of this chunk have been read
            if (ct == 0) PAIR_TRACE(16, i);
            rho = rho_next;
            if (i + 1 < nck) gate_step(i + 1);
            if (ct == 0) PAIR_TRACE(27, i);

            // (g) output epilogue: H^T of this CTA's 128 value columns (TMEM lane = value column j)
            //     times r / denominator and the output gate, for warp quarter hq's 32 tokens.  The
            //     output gate tile arrives by TMA and h replaces it in place; a lane pair (j even, j + 1)
            //     swaps one value per token pair so that each lane handles the two columns of one
            //     token as one 4-byte word (a warp's words of one token are 64 contiguous bytes of a
            //     swizzled row), and one thread stores the tile by TMA.
            if (ct == 0) {
                mbar_wait(&bars[B_HFULL], ph, wc);
                PAIR_TRACE(17, i);
                if (og) mbar_wait(&bars[B_OFULL], ph, wc);
            }
            if (!group_wait(&bars[B_INVREADY0 + b], (uint32_t)(i >> 1) & 1u, wc, ct == 0, true, 1, GA)) break;
            if (ct == 0) PAIR_TRACE(18, i);
            tc_fence_after();
            {
                uint32_t r[32];
                tmem_ld32(tmem_addr(tmem, q * 32, SM::H_COL + hq * 32), r);
                const int j = q * 32 + lane;
                const int odd = lane & 1;
                // Token pairs (k, k + 4), k = 8 a + c (c < 4): the even lane takes token k, the odd
                // lane token k + 4, each for columns (j & ~1, j | 1); the rows k and k + 4 of an 8-row
                // group fall in opposite halves of the banks under the 128-byte swizzle, so the 16
                // lanes of each row do not conflict.  The word of (token 32 hq + 8 a + e, e < 8,
                // columns j & ~1, +1) is at blk + 1024 a + 128 e + 16 ((j / 8 mod 8) ^ e).
                uint8_t *blk = Os + (j >> 6) * (L * 128) + (hq * 4) * 1024 + (j & 6) * 2;
                const uint32_t jch = (uint32_t)(j & 63) >> 3;
                uint32_t offc[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t e = (uint32_t)(c + 4 * odd);
                    offc[c] = e * 128u + ((jch ^ e) << 4);
                }
                const float4 *iv4 = reinterpret_cast<const float4 *>(inv + b * L + 32 * hq);
                tmem_wait_ld();
                if (ct == 0) PAIR_TRACE(24, i);
#pragma unroll
                for (int a8 = 0; a8 < 4; ++a8) {
                    const float4 ive = iv4[2 * a8], ivo = iv4[2 * a8 + 1];   // tokens 8 a + 0..3, + 4..7
                    const float4 ivx = odd ? ivo : ive;
                    const float ivs[4] = {ivx.x, ivx.y, ivx.z, ivx.w};
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int k = 8 * a8 + c;
                        const float send = __uint_as_float(odd ? r[k] : r[k + 4]);
                        const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
                        const float lo = odd ? recv : __uint_as_float(r[k]);       // column j & ~1
                        const float hi = odd ? __uint_as_float(r[k + 4]) : recv;   // column j | 1
                        uint32_t *w = reinterpret_cast<uint32_t *>(blk + a8 * 1024 + offc[c]);
                        uint64_t hv = f2_mul(f2_pack(lo, hi), f2_pack(ivs[c], ivs[c]));
                        if (og) hv = f2_mul(f2_from_bf16x2(*w), hv);
                        *w = f2_to_bf16x2(hv);
                    }
                }
                if (ct == 0) PAIR_TRACE(26, i);
            }
            fence_proxy_async();
            tc_fence_before();
            named_sync(1, GA);
            if (ct == 0) {
                PAIR_TRACE(19, i);
                mbar_arrive(&bars[B_HSFREE]);   // this CTA's H^T has been read
                // rows past the end of the sequence are not written
                for (int bb = 0; bb < DVT / 64; ++bb) tma_store_3d(&tm_h, Os + bb * L * 128, j0 + bb * 64, t0, bh);
                bulk_commit();
            }
        }
        if (ct == 0) bulk_wait0();   // the stores of h have completed
    }
    tc_fence_before();
    __syncthreads();
    if (*reinterpret_cast<volatile uint32_t *>(abort_flag)) {
        // a wait gave up: give copies this CTA may still have in flight time to land before the pair
        // releases its memory (bounded)
        const unsigned long long t0 = global_timer();
        while (global_timer() - t0 < 100000ull) { }
    }
    // neither CTA frees its TMEM or leaves while the other may still address its memory
    cluster_arrive_release();
    cluster_wait_acquire();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, SM::TMEM_COLS);
    }
}

}  // namespace pair

#ifdef MLSTM_WALK_TRACE
extern "C" int mlstm_pair_trace_copy(void *dst, size_t bytes)
{
    return (int)cudaMemcpyFromSymbol(dst, pair::g_pair_trace, bytes);
}
#endif

bool walk_pair_supported(int DK, int DV, int L)
{
    return L == pair::L && DK == 256 && DV % (2 * pair::DVT) == 0;
}

cudaError_t launch_walk_pair(const Params &p, const void *q, const void *k, const void *v, cudaStream_t stream)
{
    using namespace pair;
    if (!walk_pair_supported(p.DK, p.DV, p.L)) return cudaErrorInvalidValue;
    CUtensorMap mq, mks, mkd, mv, mo, mh;
    if (!make_map(&mq, q, p.DK, p.S, p.BH, HL) || !make_map(&mks, k, p.DK, p.S, p.BH, HL) ||
        !make_map(&mkd, k, p.DK, p.S, p.BH, L) || !make_map(&mv, v, p.DV, p.S, p.BH, L) ||
        !make_map(&mh, p.h, p.DV, p.S, p.BH, L) || !make_map(&mo, p.o ? (const void *)p.o : (const void *)p.h, p.DV, p.S, p.BH, L))
        return cudaErrorInvalidValue;
    using SM = Smem<256>;
    cudaError_t e = ensure_dynamic_smem((const void *)walk_pair_kernel<256>, SM::TOTAL);
    if (e != cudaSuccess) return e;
    return launch_kernel(walk_pair_kernel<256>, dim3(p.DV / DVT, p.NSEG, p.BH), dim3(THREADS), SM::TOTAL, stream, 2,
                         mq, mks, mkd, mv, mo, mh, p);
}

}  // namespace tcfwd
}  // namespace mlstm
