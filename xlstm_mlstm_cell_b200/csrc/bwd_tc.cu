// bwd_tc.cu -- the chunkwise backward pass's products on the 5th-generation tensor cores (tcgen05,
// bf16 operands, fp32 accumulators in TMEM), for bf16 inputs: dq, dk, dv and the read-out
// numerator (grad_tc_kernel), the chunk's scores and dS (chunk_tc_kernel), and the two walks over
// the chunks per state tile, the forward carry (carry_tc_kernel) and the state gradients
// (gstate_tc_kernel).
//
// Per chunk c (L tokens) and head, the gradients of the read-out (the training form of the xLSTM
// Guide's "The Dual Formulation: How mLSTM Enables Parallel GPU Training", taken chunkwise as in
// "Exploit Chunkwise Hardware Kernels for Production Training") are each a chunk-local product
// plus an inter-chunk product with the chunk's state or state gradient:
//   dq^T = scale (K^T dS^T + sc (C_c g^T + n_c dden^T)),
//   dk^T = scale Q^T dS + w (G_end V^T + dn_end 1^T),
//   dv^T = g^T A + w (G_end^T K^T),
// with sc_t = exp(m_c - max(m_c, p_t)), w_s = exp(g_c - a_s + i~_s - m_{c+1}), scale = 1/sqrt(DK)
// and the per-token factors applied column-wise (columns = tokens) in the epilogue.  A tile is
// 128 output columns (d or j: the MMA's M, one per TMEM lane) for all L tokens of one chunk (the
// MMA's N), computed as two accumulators in TMEM, the chunk-local one (K = L tokens) and the
// inter-chunk one (K = DV or DK).  The CTAs are persistent and keep a tile's two accumulators twice
// in TMEM, so that one tile's epilogue runs while the next tile's loads and MMAs do.  Every operand
// is a [rows][64] bf16 tile loaded by TMA with the 128-byte swizzle
// and read by the MMA as K-major (the reduction index runs along the row) or MN-major (along the
// column), as it lies in memory: no operand is transposed.  The fp32 intermediates (dS, A, g and
// the per-chunk states) reach this kernel as bf16 copies written by the kernels that compute them.
//
// Roles: warp 0 one TMA thread, warp 1 the MMA thread (and the TMEM allocation), warps 2..5 the
// epilogue (TMEM lane quadrant = warp % 4).  Every wait is bounded; a timeout sets the call's
// status word.
#include "bwd_tc.h"
#include "common.cuh"
#include "tc_common.cuh"
#include "tc_fwd.h"

#include <cudaTypedefs.h>

#include <algorithm>

namespace mlstm {
namespace bwdtc {

using namespace tc;

constexpr int TM = 128;                // output columns per CTA (M)
constexpr int STAGES = 4;              // pipeline stages of 64 reduction elements
constexpr int THREADS = 192;
constexpr uint32_t SA = TM * 128;      // A tile of a stage: 128 rows of 64 bf16, or 64 rows x 2 blocks

template <int L>
struct Smem {
    static constexpr uint32_t SB = L * 128;                   // B tile of a stage: L tokens x 64
    static constexpr uint32_t STAGE = SA + SB;
    static constexpr uint32_t F = STAGES * STAGE;             // floats: tokw [L], ddv [L], red [4][L]
    static constexpr uint32_t BAR = F + 6 * L * 4;
    static constexpr uint32_t NBAR = 2 * STAGES + 4;          // full, empty, accf [2], tfree [2]
    static constexpr uint32_t TOTAL = BAR + NBAR * 8 + 16 + 1024;
    // the two accumulators of a tile, twice: the MMAs of the next tile run while the epilogue reads one
    static constexpr uint32_t TMEM_COLS = 4 * L;
    static constexpr int CTAS_PER_SM = L == 64 ? 2 : 1;       // (TMEM: 512 columns per SM)
};

struct KParams {
    int S, NC, DK, DV, NTK, NJT, BH;
    const float *A, *P, *MC, *G, *ig, *DD, *NS, *GN;
    const __nv_bfloat16 *pq;               // q (KIND 0) or k (KIND 1): the partial row sums
    __nv_bfloat16 *out;
    float *part;                           // q . dq^inter (KIND 0: the inter-chunk term alone) or k . dk
    float *part2;                          // k . dk^inter (KIND 1)
    // KIND 3 (the read-out numerator)
    const __nv_bfloat16 *dh, *o;
    const float *NRM;
    float *DOTP;
    __nv_bfloat16 *g16w, *dog, *sg16;
    uint32_t *status;
};

// OR of a predicate over the `count` threads that meet at named barrier `id`: every thread gets the
// same answer.
__device__ __forceinline__ bool group_any(uint32_t id, uint32_t count, bool pred)
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

// Sums v[u] (u < 16) over the 32 lanes of the warp for every u at once: each step hands half of the
// remaining values to the lane partner and keeps the other half.  Lane l ends with the sum of value
// sum16_index(l) (both lanes of a pair hold it).
__device__ __forceinline__ float warp_sum16(float (&v)[16], int lane)
{
#pragma unroll
    for (int o = 16, nv = 16; o >= 2; o >>= 1, nv >>= 1) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int z = 0; z < nv / 2; ++z) {
            const float send = up ? v[z] : v[z + nv / 2], keep = up ? v[z + nv / 2] : v[z];
            v[z] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
}
__device__ __forceinline__ int sum16_index(int lane)
{
    return ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1);
}

// The read-out numerator's epilogue for 16 tokens g * 16 .. of a thread's value column:
// num = A V + sc scale q C_c (r1, r2: the two accumulators' columns), hh = num / N, do = dh hh,
// g = o dh / N; the warp's row sums of g . hh go to red[t].
__device__ __forceinline__ void epilogue_num(const KParams &p, const uint32_t (&r1)[16], const uint32_t (&r2)[16],
                                             const float *tokw, const float *nrm, float *red, int grp, int len,
                                             size_t g0, int col, float scale, int lane, __nv_bfloat16 *sg_hi,
                                             __nv_bfloat16 *g_hi)
{
    float dhv[16], ov[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
        const int t = grp * 16 + u;
        const size_t off = (g0 + t) * p.DV + col;
        dhv[u] = t < len ? __bfloat162float(p.dh[off]) : 0.f;
        ov[u] = (t < len && p.o) ? __bfloat162float(p.o[off]) : 1.f;
    }
    tmem_wait_ld();
    float pr[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
        const int t = grp * 16 + u;
        const size_t off = (g0 + t) * p.DV + col;
        const float num = __uint_as_float(r1[u]) + tokw[t] * scale * __uint_as_float(r2[u]);
        const float rN = nrm[t];   // 1 / N
        const float hh = num * rN;
        const float g = ov[u] * dhv[u] * rN;
        pr[u] = 0.f;
        if (t < len) {
            if (p.dog) p.dog[off] = __float2bfloat16_rn(dhv[u] * hh);
            // g and sc_t g_t as two bf16 parts each, [BH][2][S][DV]: the operands of dS, dq, dv and
            // of the state gradient
            const size_t o2 = (size_t)t * p.DV + col;
            bf16_parts(g, g_hi[o2], g_hi[o2 + (size_t)p.S * p.DV]);
            bf16_parts(tokw[t] * g, sg_hi[o2], sg_hi[o2 + (size_t)p.S * p.DV]);
            pr[u] = g * hh;
        }
    }
    const float sum = warp_sum16(pr, lane);
    if ((lane & 1) == 0) red[grp * 16 + sum16_index(lane)] = sum;
}

// KIND 0: dq, 1: dk, 2: dv, 3: the read-out numerator num^T = V^T A^T + sc scale C_c^T Q^T.
// Operands of the chunk-local product (A1, B1) and of the inter-chunk product (A2, B2), by tensor map:
//   KIND 0: A1 = k [s][d] (MN-major), B1 = dS [t][s] (K-major), A2 = C_c [d][j] (K), B2 = g [t][j] (K)
//   KIND 1: A1 = q [t][d] (MN),       B1 = dS [t][s] (MN),      A2 = G_end [d][j] (K), B2 = v [s][j] (K)
//   KIND 2: A1 = g [t][j] (MN),       B1 = A [t][s] (MN),       A2 = G_end [d][j] (MN), B2 = k [s][d] (K)
//   KIND 3: A1 = v [s][j] (MN),       B1 = A [t][s] (K),        A2 = C_c [d][j] (MN),   B2 = q [t][d] (K)
template <int KIND, int L>
__global__ void __launch_bounds__(THREADS, Smem<L>::CTAS_PER_SM)
grad_tc_kernel(const __grid_constant__ CUtensorMap tm_a1, const __grid_constant__ CUtensorMap tm_b1,
               const __grid_constant__ CUtensorMap tm_a2, const __grid_constant__ CUtensorMap tm_b2, KParams p)
{
    using SM = Smem<L>;
    constexpr int A1_MN = 1, B1_MN = (KIND == 0 || KIND == 3) ? 0 : 1, A2_MN = (KIND == 2 || KIND == 3) ? 1 : 0;
    constexpr int B2_MN = 0;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    float *tokw = reinterpret_cast<float *>(smem + SM::F);   // sc_t (KIND 0) or w_s
    float *ddv = tokw + L;                                    // dden_t (KIND 0), 1 / N_t (KIND 3)
    float *red = ddv + L;                                     // [4][L] per-warp row sums (KIND 3)
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::BAR);
    uint64_t *full = bars, *empty = bars + STAGES, *accf = bars + 2 * STAGES, *tfree = accf + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + SM::NBAR);
    uint32_t *abort_flag = tmem_slot + 1;

    // persistent: this CTA takes tiles blockIdx.x, + gridDim.x, ...; a tile is (head, chunk, 128 output
    // columns), the output-column tiles of a chunk consecutive (they share the chunk's B operands)
    const int MT = (KIND >= 2 ? p.DV : p.DK) / TM;
    const long long ntiles = (long long)p.BH * p.NC * MT;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // KIND 3 takes its fp32 operands (A and C_c) as two bf16 parts, the value and the rounding
    // residue, and sums both products in the accumulator
    constexpr int NPART = KIND == 3 ? 2 : 1;
    const int nloc = L / 64, ninter = (KIND >= 2 ? p.DK : p.DV) / 64;
    const int nl = NPART * nloc, nb = nl + NPART * ninter;
    WaitCtx wc{abort_flag, p.status};
    struct Tile { int bh, c, m0; };
    auto tile_of = [&](long long t) {
        Tile r;
        r.m0 = (int)(t % MT) * TM;
        const long long bc = t / MT;
        r.c = (int)(bc % p.NC);
        r.bh = (int)(bc / p.NC);
        return r;
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accf[b], 1);
            mbar_init(&tfree[b], 4);   // one arrival per epilogue warp
        }
        *abort_flag = 0u;
        fence_barrier_init();
        tma_prefetch(&tm_a1);
        tma_prefetch(&tm_b1);
        tma_prefetch(&tm_a2);
        tma_prefetch(&tm_b2);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, SM::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    griddep_wait();   // every operand is written by the kernels before this one
    griddep_launch_dependents();

    if (warp == 0) {
        if (lane == 0) {   // TMA producer: one ring of stages across this CTA's tiles
            long long kg = 0;
            bool ok = true;
            for (long long tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
                const Tile T = tile_of(tile);
                const int bh = T.bh, t0 = T.c * L, m0 = T.m0;
                const int zc = bh * p.NC + T.c;   // (head, chunk) of the per-chunk arrays
                for (int kb = 0; kb < nb; ++kb, ++kg) {
                    const int st = (int)(kg % STAGES);
                    if (kg >= STAGES && !mbar_wait(&empty[st], (uint32_t)((kg / STAGES) - 1) & 1u, wc)) { ok = false; break; }
                    mbar_arrive_expect_tx(&full[st], SM::STAGE);
                    uint8_t *a = smem + st * SM::STAGE, *b = a + SA;
                    const bool loc = kb < nl;
                    const int idx = loc ? kb : kb - nl, nper = loc ? nloc : ninter;
                    const int part = idx / nper, k0 = 64 * (idx % nper);   // bf16 part, first reduction index
                    if (loc) {
#pragma unroll
                        for (int mb = 0; mb < 2; ++mb)   // A1 rows: the stage's 64 tokens, 2 x 64 output columns
                            tma_load_3d(a + mb * 8192, &tm_a1, m0 + 64 * mb, t0 + k0, KIND == 2 ? 2 * bh : bh, &full[st]);
                        // the chunk's first row in the score arrays: A holds two parts per chunk
                        const int rb = KIND >= 2 ? 2 * t0 + part * L : t0;
#pragma unroll
                        for (int n = 0; n < L / 64; ++n) {
                            if (!B1_MN)      // dS or A rows t (N), columns s (K)
                                tma_load_3d(b + n * 8192, &tm_b1, k0, rb + 64 * n, bh, &full[st]);
                            else             // dS or A rows t (K), columns s (N)
                                tma_load_3d(b + n * 8192, &tm_b1, 64 * n, rb + k0, bh, &full[st]);
                        }
                    } else {
                        // C_c holds two parts per chunk, G_end one
                        const int za = (KIND == 0 || KIND == 3) ? 2 * zc + part : zc;
#pragma unroll
                        for (int mb = 0; mb < 2; ++mb) {
                            if (A2_MN)       // G_end or C_c rows d (K), columns j (M)
                                tma_load_3d(a + mb * 8192, &tm_a2, m0 + 64 * mb, k0, za, &full[st]);
                            else             // C_c or G_end rows d (M), columns j (K)
                                tma_load_3d(a + mb * 8192, &tm_a2, k0, m0 + 64 * mb, za, &full[st]);
                        }
#pragma unroll
                        for (int n = 0; n < L / 64; ++n)   // g, v, k or q rows (N), columns (K)
                            tma_load_3d(b + n * 8192, &tm_b2, k0, t0 + 64 * n, KIND == 0 ? 2 * bh : bh, &full[st]);
                    }
                }
            }
            // the last stages' copies have landed before the CTA may leave
            for (int s = 0; s < STAGES && s < kg; ++s) {
                const long long last = kg - 1 - s;
                mbar_wait_drain(&full[last % STAGES], (uint32_t)(last / STAGES) & 1u);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {   // MMA issuer: tile it into TMEM buffer it & 1 once the epilogue has read it
            constexpr uint32_t ID1 = idesc_bf16(TM, L, A1_MN, B1_MN), ID2 = idesc_bf16(TM, L, A2_MN, B2_MN);
            long long kg = 0;
            int it = 0;
            bool ok = true;
            for (long long tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++it) {
                const int buf = it & 1;
                if (it >= 2 && !mbar_wait(&tfree[buf], (uint32_t)((it >> 1) - 1) & 1u, wc)) break;
                tc_fence_after();
                for (int kb = 0; kb < nb; ++kb, ++kg) {
                    const int st = (int)(kg % STAGES);
                    if (!mbar_wait(&full[st], (uint32_t)(kg / STAGES) & 1u, wc)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a = smem_u32(smem + st * SM::STAGE), b = a + SA;
                    const bool loc = kb < nl;
                    const int first = loc ? kb : kb - nl;   // blocks of this accumulator before this one
                    const int amn = loc ? A1_MN : A2_MN, bmn = loc ? B1_MN : B2_MN;
                    const uint32_t d = tmem + (uint32_t)(buf * 2 * L) + (loc ? 0u : (uint32_t)L);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {   // 16 reduction elements per MMA
                        // K-major: 32 bytes further along the 128-byte rows; MN-major: 16 rows further
                        const uint64_t ad = amn ? smem_desc(a + kk * 2048, 8192, 1024) : smem_desc(a, 16, 1024) + (uint64_t)(kk * 2);
                        const uint64_t bd = bmn ? smem_desc(b + kk * 2048, 8192, 1024) : smem_desc(b, 16, 1024) + (uint64_t)(kk * 2);
                        mma_ss(d, ad, bd, loc ? ID1 : ID2, (first > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(&empty[st]);
                }
                if (ok) mma_commit(&accf[buf]);
            }
        }
    } else {
        // ------------------------------------------------ epilogue: warps 2..5
        const int et = threadIdx.x - 64;           // 0..127
        const int q4 = warp & 3;                   // TMEM lane quadrant
        const float scale = rsqrtf((float)p.DK);
        const int NCOL = KIND >= 2 ? p.DV : p.DK;
        int it = 0;
        for (long long tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
            const Tile T = tile_of(tile);
            const int bh = T.bh, c = T.c, m0 = T.m0, buf = it & 1;
            const int t0 = c * L, len = min(L, p.S - t0);
            const int col = m0 + q4 * 32 + lane;       // this thread's output column
            const size_t g0 = (size_t)bh * p.S + t0;   // first token of the chunk
            named_sync(1, 128);   // the previous tile's readers of tokw, ddv and red are done
            if (et < L) {
                const int t = et;
                const bool okt = t < len;
                if (KIND == 0 || KIND == 3) {
                    const float mc = p.MC[(size_t)bh * (p.NC + 1) + c];
                    tokw[t] = okt ? expf(mc - fmaxf(mc, p.P[g0 + t])) : 0.f;
                    if (KIND == 0) ddv[t] = okt ? p.DD[g0 + t] : 0.f;
                    else ddv[t] = okt ? 1.f / p.NRM[g0 + t] : 1.f;
                } else {
                    const float gm = p.G[(size_t)bh * p.NC + c] - p.MC[(size_t)bh * (p.NC + 1) + c + 1];
                    tokw[t] = okt ? expf(p.ig[g0 + t] - p.A[g0 + t] + gm) : 0.f;
                    ddv[t] = 0.f;
                }
            }
            float colv = 0.f;   // n_c (KIND 0) or dn_end (KIND 1) of this column
            if (KIND == 0) colv = p.NS[((size_t)bh * p.NC + c) * p.DK + col];
            if (KIND == 1) colv = p.GN[((size_t)bh * p.NC + c) * p.DK + col];
            // the rows the epilogue reads (dh and o, or q or k: L tokens x 128 columns) into L2 while
            // the tile's MMAs run, a 128-byte line per thread and array
            if (KIND != 2) {
                for (int e = et; e < 2 * L; e += 128) {
                    const int t = e >> 1;
                    if (t < len) {
                        const size_t off = (g0 + t) * (size_t)(KIND == 3 ? p.DV : p.DK) + m0 + (e & 1) * 64;
                        if (KIND == 3) {
                            asm volatile("prefetch.global.L2 [%0];" ::"l"(p.dh + off));
                            if (p.o) asm volatile("prefetch.global.L2 [%0];" ::"l"(p.o + off));
                        } else {
                            asm volatile("prefetch.global.L2 [%0];" ::"l"(p.pq + off));
                        }
                    }
                }
            }
            named_sync(1, 128);   // tokw, ddv
            // one thread waits for the accumulators; the four warps take its answer together (the TMEM
            // loads below are warp-collective)
            bool failed = false;
            if (et == 0) failed = !mbar_wait(&accf[buf], (uint32_t)(it >> 1) & 1u, wc);
            failed = group_any(2, 128, failed);
            if (failed) break;
            tc_fence_after();
            const uint32_t tb = (uint32_t)(buf * 2 * L);
#pragma unroll 1
            for (int g = 0; g < L / 16; ++g) {
                uint32_t r1[16], r2[16];
                tmem_ld16(tmem_addr(tmem, q4 * 32, tb + g * 16), r1);
                tmem_ld16(tmem_addr(tmem, q4 * 32, tb + L + g * 16), r2);
                float pv[16];
                if (KIND == 3) {
                    epilogue_num(p, r1, r2, tokw, ddv, red + q4 * L, g, len, g0, col, scale, lane,
                                 p.sg16 + ((size_t)2 * bh * p.S + t0) * p.DV,
                                 p.g16w + ((size_t)2 * bh * p.S + t0) * p.DV);
                    continue;
                }
                if (KIND < 2) {
#pragma unroll
                    for (int u = 0; u < 16; ++u) {
                        const int t = g * 16 + u;
                        pv[u] = t < len ? __bfloat162float(p.pq[(g0 + t) * p.DK + col]) : 0.f;
                    }
                }
                tmem_wait_ld();
                float prs[16], prs2[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int t = g * 16 + u;
                    const float d1 = __uint_as_float(r1[u]), d2 = __uint_as_float(r2[u]);
                    const float w = tokw[t];
                    float o, pr = 0.f, pr2 = 0.f;
                    if (KIND == 0) {
                        const float dqi = w * (d2 + ddv[t] * colv);   // the inter-chunk term
                        o = (d1 + dqi) * scale;
                        pr = pv[u] * scale * dqi;
                    } else if (KIND == 1) {
                        const float dki = w * (d2 + colv);
                        o = scale * d1 + dki;
                        pr = pv[u] * o;
                        pr2 = pv[u] * dki;
                    } else {
                        o = d1 + w * d2;
                    }
                    if (t < len) p.out[(g0 + t) * NCOL + col] = __float2bfloat16_rn(o);
                    prs[u] = pr;
                    prs2[u] = pr2;
                }
                // per token over the warp's 32 columns: q . dq^inter (KIND 0), k . dk and k . dk^inter
                if (KIND < 2) {
                    const float sum = warp_sum16(prs, lane);
                    const int t = g * 16 + sum16_index(lane);
                    if ((lane & 1) == 0 && t < len) p.part[(g0 + t) * p.NTK + (col >> 5)] = sum;
                }
                if (KIND == 1) {
                    const float sum = warp_sum16(prs2, lane);
                    const int t = g * 16 + sum16_index(lane);
                    if ((lane & 1) == 0 && t < len) p.part2[(g0 + t) * p.NTK + (col >> 5)] = sum;
                }
            }
            // the accumulators of this buffer have been read: the MMAs of tile it + 2 may take them
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tfree[buf]);
            if (KIND == 3) {
                // the row sums of g . hh over each 64 value columns: the two warps of a 64-column half
                named_sync(1, 128);
                for (int e = et; e < 2 * L; e += 128) {
                    const int h2 = e / L, t = e % L;
                    if (t < len)
                        p.DOTP[((size_t)bh * p.S + t0 + t) * p.NJT + (m0 >> 6) + h2] = red[(2 * h2) * L + t] + red[(2 * h2 + 1) * L + t];
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (*reinterpret_cast<volatile uint32_t *>(abort_flag)) {
        // a wait gave up: let MMAs and copies this CTA may still have in flight finish (bounded)
        const unsigned long long tb = global_timer();
        while (global_timer() - tb < 100000ull) { }
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, SM::TMEM_COLS);
    }
}

// [BH][R][C] bf16 maps (boxes of 64 rows x 64 columns) over the arrays the products read.
static bool map3(CUtensorMap *m, const void *base, int C, int R, int Z) { return tcfwd::make_map(m, base, C, R, Z, 64); }

template <int KIND, int L>
static cudaError_t launch_kind(const Args &a, const CUtensorMap &a1, const CUtensorMap &b1, const CUtensorMap &a2,
                               const CUtensorMap &b2)
{
    using SM = Smem<L>;
    KParams p;
    p.S = a.S; p.NC = a.NC; p.DK = a.DK; p.DV = a.DV; p.NTK = a.NTK; p.NJT = a.NJT;
    p.dh = a.dh; p.o = a.o; p.NRM = a.NRM; p.DOTP = a.DOTP; p.g16w = a.g16w; p.dog = a.dog;
    p.sg16 = a.sg16;
    p.A = a.A; p.P = a.P; p.MC = a.MC; p.G = a.G; p.ig = a.ig; p.DD = a.DD; p.NS = a.NS; p.GN = a.GN;
    p.pq = KIND == 0 ? a.q : a.k;
    p.out = KIND == 0 ? a.dq : KIND == 1 ? a.dk : a.dv;
    p.part = KIND == 0 ? a.QD : KIND == 1 ? a.KD : nullptr;
    p.part2 = KIND == 1 ? a.KI : nullptr;
    p.status = a.status;
    p.BH = a.BH;
    cudaError_t e = ensure_dynamic_smem((const void *)grad_tc_kernel<KIND, L>, SM::TOTAL);
    if (e != cudaSuccess) return e;
    int sms = 0;
    if ((e = sm_count(&sms)) != cudaSuccess) return e;
    // persistent CTAs, SM::CTAS_PER_SM on every SM (fewer when there are fewer tiles)
    const long long tiles = (long long)a.BH * a.NC * ((KIND >= 2 ? a.DV : a.DK) / TM);
    const int grid = (int)std::min<long long>(tiles, (long long)sms * SM::CTAS_PER_SM);
    return launch_kernel(grad_tc_kernel<KIND, L>, dim3(grid), dim3(THREADS), SM::TOTAL, a.stream, 1, a1,
                         b1, a2, b2, p);
}

template <int L>
static cudaError_t launch_l(const Args &a)
{
    CUtensorMap mq, mk, mv, mg, mds, ma, mc, mG;
    const int CL = a.NC * L;   // rows of the per-chunk score arrays (A and C_c: two parts each)
    if (!map3(&mq, a.q, a.DK, a.S, a.BH) || !map3(&mk, a.k, a.DK, a.S, a.BH) || !map3(&mv, a.v, a.DV, a.S, a.BH) ||
        !map3(&mg, a.g16, a.DV, a.S, 2 * a.BH) || !map3(&mds, a.dS16, L, CL, a.BH) || !map3(&ma, a.A16, L, 2 * CL, a.BH) ||
        !map3(&mc, a.C16, a.DV, a.DK, 2 * a.BH * a.NC) || !map3(&mG, a.G16, a.DV, a.DK, a.BH * a.NC))
        return cudaErrorInvalidValue;
    cudaError_t e = launch_kind<0, L>(a, mk, mds, mc, mg);
    if (e == cudaSuccess) e = launch_kind<1, L>(a, mq, mds, mG, mv);
    if (e == cudaSuccess) e = launch_kind<2, L>(a, mg, ma, mG, mk);
    return e;
}

template <int L>
static cudaError_t launch_num_l(const Args &a)
{
    CUtensorMap mq, mv, ma, mc;
    if (!map3(&mq, a.q, a.DK, a.S, a.BH) || !map3(&mv, a.v, a.DV, a.S, a.BH) ||
        !map3(&ma, a.A16, L, 2 * a.NC * L, a.BH) || !map3(&mc, a.C16, a.DV, a.DK, 2 * a.BH * a.NC))
        return cudaErrorInvalidValue;
    return launch_kind<3, L>(a, mv, ma, mc, mq);
}

cudaError_t launch_num(const Args &a)
{
    if (!supported(a.DK, a.DV, a.L)) return cudaErrorInvalidValue;
    return a.L == 64 ? launch_num_l<64>(a) : launch_num_l<128>(a);
}

// ---------------------------------------------------------------- the forward carry
// w_s k_s[d] as two bf16 parts, w_s = exp(g_c - a_s + i~_s - m_{c+1}) (c the chunk of token s): the
// weight of token s in the state at its chunk's end, in that state's stabilized frame (<= 1).
__global__ void __launch_bounds__(256) wk_parts_kernel(const __nv_bfloat16 *__restrict__ k, const float *__restrict__ A,
                                                       const float *__restrict__ ig, const float *__restrict__ G,
                                                       const float *__restrict__ MC, int BH, int S, int L, int NC,
                                                       int DK, __nv_bfloat16 *__restrict__ wk)
{
    griddep_wait();
    griddep_launch_dependents();
    const int n8 = DK / 8;
    const size_t items = (size_t)BH * S * n8;
    for (size_t it = (size_t)blockIdx.x * blockDim.x + threadIdx.x; it < items; it += (size_t)gridDim.x * blockDim.x) {
        const size_t tok = it / n8;                // bh * S + s
        const int d0 = (int)(it % n8) * 8;
        const int bh = (int)(tok / S), s = (int)(tok % S), c = s / L;
        const float w = expf(G[(size_t)bh * NC + c] - A[tok] + ig[tok] - MC[(size_t)bh * (NC + 1) + c + 1]);
        const uint4 u = *reinterpret_cast<const uint4 *>(k + tok * DK + d0);
        const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
        __nv_bfloat16 hi[8], lo[8];
#pragma unroll
        for (int z = 0; z < 4; ++z) {
            bf16_parts(w * __uint_as_float(wd[z] << 16), hi[2 * z], lo[2 * z]);
            bf16_parts(w * __uint_as_float(wd[z] & 0xffff0000u), hi[2 * z + 1], lo[2 * z + 1]);
        }
        __nv_bfloat16 *dst = wk + ((size_t)(2 * bh) * S + s) * DK + d0;
        *reinterpret_cast<uint4 *>(dst) = *reinterpret_cast<const uint4 *>(hi);
        *reinterpret_cast<uint4 *>(dst + (size_t)S * DK) = *reinterpret_cast<const uint4 *>(lo);
    }
}

// The walk over the chunks of one 128 x 64 tile of the state (rows d, columns j): per chunk the
// contribution U_c = sum_s (w_s k_s) v_s^T as MMAs (A = w k, two parts, MN-major; B = v, MN-major)
// into one of two TMEM buffers, and in the tiles of columns 0..63 also sum_s w_s k_s (B = a tile of
// ones), while the epilogue warps, which hold the fp32 state in registers (a TMEM lane = a row d,
// 64 columns per thread), write the state at the chunk's start as two bf16 parts and n, then
// C <- exp(g_c + m_c - m_{c+1}) C + U_c.
constexpr int CSTAGES = 4;
struct CarrySmem {
    static constexpr uint32_t STAGE = 2 * 16384 + 8192;      // w k: 2 parts x 64 tokens x 128 rows; v: 64 x 64
    static constexpr uint32_t ONES = CSTAGES * STAGE;        // 16 rows x 64 bf16 ones (K-major B of n)
    // per epilogue warp, tiles of its 32 state rows x 64 columns (bf16, 128-byte swizzle, 4 KB each)
    // that TMA moves: the carry's chunk-start state (two parts) out; the state-gradient walk's
    // chunk-end gradient out (one) and C_c in (two buffers)
    static constexpr uint32_t STG = ONES + 2048;
    static constexpr uint32_t STG_BYTES = 4 * 3 * 4096;
    static constexpr uint32_t BAR = STG + STG_BYTES;
    static constexpr uint32_t NBAR = 2 * CSTAGES + 4 + 8;   // (+ the C_c tiles' barriers, two per warp)
    static constexpr uint32_t TOTAL = BAR + NBAR * 8 + 16 + 1024;
    static_assert(STG % 1024 == 0 && TOTAL <= 232448, "carry smem");
};

// Byte offset of 16-byte chunk x (0..7) of row r in a [rows][64] bf16 tile under the 128-byte swizzle.
__device__ __forceinline__ uint32_t sw_tile(int r, int x) { return (uint32_t)(r * 128 + ((x ^ (r & 7)) << 4)); }

template <int L>
__global__ void __launch_bounds__(THREADS, 1)
carry_tc_kernel(const __grid_constant__ CUtensorMap tm_wk, const __grid_constant__ CUtensorMap tm_v,
                const __grid_constant__ CUtensorMap tm_cs, KParams p, float *__restrict__ NSo)
{
    using SM = CarrySmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::BAR);
    uint64_t *full = bars, *empty = bars + CSTAGES, *ufull = bars + 2 * CSTAGES, *ufree = ufull + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + SM::NBAR);
    uint32_t *abort_flag = tmem_slot + 1;
    const int bh = blockIdx.x, d0 = blockIdx.y * 128, j0 = blockIdx.z * 64;
    const bool with_n = blockIdx.z == 0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int KB = L / 64;                 // 64-token blocks per chunk
    const int nblk = (p.NC - 1) * KB;          // (the last chunk's contribution is not needed)
    WaitCtx wc{abort_flag, p.status};

    if (threadIdx.x == 0) {
        for (int s = 0; s < CSTAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ufull[b], 1);
            mbar_init(&ufree[b], 4);   // one arrival per epilogue warp
        }
        *abort_flag = 0u;
        fence_barrier_init();
        tma_prefetch(&tm_wk);
        tma_prefetch(&tm_v);
        tma_prefetch(&tm_cs);
    }
    // the ones tile (every element 1.0, so its layout needs no swizzle care)
    for (int e = threadIdx.x; e < 2048 / 16; e += blockDim.x)
        reinterpret_cast<uint4 *>(smem + SM::ONES)[e] = make_uint4(0x3f803f80u, 0x3f803f80u, 0x3f803f80u, 0x3f803f80u);
    fence_proxy_async();
    if (warp == 1) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;   // U buffers at columns 0 and 64, n buffers at 128 and 144
    griddep_wait();
    griddep_launch_dependents();

    if (warp == 0) {
        if (lane == 0) {
            int kb = 0;
            for (; kb < nblk; ++kb) {
                const int st = kb % CSTAGES;
                if (kb >= CSTAGES && !mbar_wait(&empty[st], (uint32_t)((kb / CSTAGES) - 1) & 1u, wc)) break;
                mbar_arrive_expect_tx(&full[st], SM::STAGE);
                uint8_t *a = smem + st * SM::STAGE, *b = a + 32768;
                const int t = kb * 64;   // first token of the block
#pragma unroll
                for (int part = 0; part < 2; ++part)
#pragma unroll
                    for (int mb = 0; mb < 2; ++mb)
                        tma_load_3d(a + part * 16384 + mb * 8192, &tm_wk, d0 + 64 * mb, t, 2 * bh + part, &full[st]);
                tma_load_3d(b, &tm_v, j0, t, bh, &full[st]);
            }
            for (int s = 0; s < CSTAGES && s < kb; ++s) {
                const int last = kb - 1 - s;
                mbar_wait_drain(&full[last % CSTAGES], (uint32_t)(last / CSTAGES) & 1u);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t IDU = idesc_bf16(128, 64, 1, 1), IDN = idesc_bf16(128, 16, 1, 0);
            const uint64_t ones = smem_desc(smem_u32(smem + SM::ONES), 16, 1024);
            bool ok = true;
            for (int c = 0; c < p.NC - 1 && ok; ++c) {
                const int ub = c & 1;
                if (c >= 2 && !mbar_wait(&ufree[ub], (uint32_t)((c >> 1) - 1) & 1u, wc)) { ok = false; break; }
                for (int q = 0; q < KB; ++q) {
                    const int kb = c * KB + q, st = kb % CSTAGES;
                    if (!mbar_wait(&full[st], (uint32_t)(kb / CSTAGES) & 1u, wc)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a = smem_u32(smem + st * SM::STAGE), b = a + 32768;
#pragma unroll
                    for (int part = 0; part < 2; ++part)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t ad = smem_desc(a + part * 16384 + kk * 2048, 8192, 1024);
                            const uint32_t acc = (q > 0 || part > 0 || kk > 0) ? 1u : 0u;
                            mma_ss(tmem + ub * 64, ad, smem_desc(b + kk * 2048, 8192, 1024), IDU, acc);
                            if (with_n) mma_ss(tmem + 128 + ub * 16, ad, ones + (uint64_t)(kk * 2), IDN, acc);
                        }
                    mma_commit(&empty[st]);
                }
                if (ok) mma_commit(&ufull[ub]);
            }
        }
    } else {
        const int q4 = warp & 3;
        const int d = d0 + q4 * 32 + lane;   // this thread's state row
        const float *MCb = p.MC + (size_t)bh * (p.NC + 1);
        const float *Gb = p.G + (size_t)bh * p.NC;
        float C[64];
#pragma unroll
        for (int x = 0; x < 64; ++x) C[x] = 0.f;
        float n = 0.f;
        // the chunk's decay terms, loaded one chunk ahead (off the chain of chunk steps)
        float g_c = Gb[0], mc_c = MCb[0], mn_c = MCb[p.NC > 1 ? 1 : 0];
        for (int c = 0; c < p.NC; ++c) {
            const float decay = expf(g_c + mc_c - mn_c);
            if (c + 2 <= p.NC - 1) {
                g_c = Gb[c + 1];
                mc_c = mn_c;
                mn_c = MCb[c + 2];
            }
            // the state at the chunk's start: its two bf16 parts (this warp's 32 rows through a swizzled
            // tile per part and a TMA store each, once the previous chunk's stores have read the tiles),
            // and n
            {
                uint8_t *stg = smem + SM::STG + q4 * 8192;
                if (lane == 0) bulk_wait_read0();
                __syncwarp();
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    __nv_bfloat16 hi[8], lo[8];
#pragma unroll
                    for (int z = 0; z < 8; ++z) bf16_parts(C[8 * x + z], hi[z], lo[z]);
                    *reinterpret_cast<uint4 *>(stg + sw_tile(lane, x)) = *reinterpret_cast<const uint4 *>(hi);
                    *reinterpret_cast<uint4 *>(stg + 4096 + sw_tile(lane, x)) = *reinterpret_cast<const uint4 *>(lo);
                }
                fence_proxy_async();
                __syncwarp();
                if (lane == 0) {
                    const int z0 = 2 * (bh * p.NC + c);
                    tma_store_3d(&tm_cs, stg, j0, d0 + q4 * 32, z0);
                    tma_store_3d(&tm_cs, stg + 4096, j0, d0 + q4 * 32, z0 + 1);
                    bulk_commit();
                }
            }
            if (with_n) NSo[((size_t)bh * p.NC + c) * p.DK + d] = n;
            if (c == p.NC - 1) break;   // (the final state is not needed)
            const int ub = c & 1;
            bool failed = false;
            if (lane == 0) failed = !mbar_wait(&ufull[ub], (uint32_t)(c >> 1) & 1u, wc);
            if (__shfl_sync(0xffffffffu, failed ? 1 : 0, 0)) break;
            tc_fence_after();
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                uint32_t r[16];
                tmem_ld16(tmem_addr(tmem, q4 * 32, ub * 64 + g * 16), r);
                tmem_wait_ld();
#pragma unroll
                for (int z = 0; z < 16; ++z) C[g * 16 + z] = fmaf(decay, C[g * 16 + z], __uint_as_float(r[z]));
            }
            if (with_n) {
                uint32_t r4[4];
                tmem_ld4(tmem_addr(tmem, q4 * 32, 128 + ub * 16), r4);
                tmem_wait_ld();
                n = fmaf(decay, n, __uint_as_float(r4[0]));
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ufree[ub]);
        }
        if (lane == 0) bulk_wait0();   // this warp's state stores are complete
    }
    tc_fence_before();
    __syncthreads();
    if (*reinterpret_cast<volatile uint32_t *>(abort_flag)) {
        const unsigned long long tb = global_timer();
        while (global_timer() - tb < 100000ull) { }
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// The reverse walk of the state gradients over the chunks of one 128 x 64 tile (rows d, columns j); it
// also leaves, per warp and chunk, the tile's share of E_c (the pairs of tokens that skip chunk c):
// per chunk the read-out's dC_c = scale sum_t q_t (sc_t g_t)^T as MMAs (A = q, MN-major; B = sc g,
// two parts, MN-major) into one of two TMEM buffers, while the epilogue warps, which hold the fp32
// gradient in registers, write the gradient of the state at the chunk's end (bf16) and then
// G <- dC_c + exp(g_c + m_c - m_{c+1}) G; the tiles of columns 0..63 run the normalizer's gradient
// through GN the same way, in place (dn_c in, the chunk-end gradient out).
template <int L>
__global__ void __launch_bounds__(THREADS, 1)
gstate_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_sg,
                 const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_c, KParams p,
                 float *__restrict__ GN, float *__restrict__ EP, int NEP)
{
    using SM = CarrySmem;   // (a stage: q 64 tokens x 128 rows, then sc g 2 parts x 64 tokens x 64)
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::BAR);
    uint64_t *full = bars, *empty = bars + CSTAGES, *ufull = bars + 2 * CSTAGES, *ufree = ufull + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + SM::NBAR);
    uint32_t *abort_flag = tmem_slot + 1;
    const int bh = blockIdx.x, d0 = blockIdx.y * 128, j0 = blockIdx.z * 64;
    const bool with_n = blockIdx.z == 0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int KB = L / 64;
    const int nblk = (p.NC - 1) * KB;          // chunks NC - 1 .. 1 (the gradient of the start state is not needed)
    WaitCtx wc{abort_flag, p.status};

    if (threadIdx.x == 0) {
        for (int s = 0; s < CSTAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ufull[b], 1);
            mbar_init(&ufree[b], 4);
        }
        for (int b = 0; b < 8; ++b) mbar_init(&ufree[2 + b], 1);   // the C_c tiles, two per epilogue warp
        *abort_flag = 0u;
        fence_barrier_init();
        tma_prefetch(&tm_q);
        tma_prefetch(&tm_sg);
        tma_prefetch(&tm_g);
        tma_prefetch(&tm_c);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;   // dC buffers at columns 0 and 64
    griddep_wait();
    griddep_launch_dependents();

    if (warp == 0) {
        if (lane == 0) {
            int kb = 0;
            for (; kb < nblk; ++kb) {
                const int st = kb % CSTAGES;
                if (kb >= CSTAGES && !mbar_wait(&empty[st], (uint32_t)((kb / CSTAGES) - 1) & 1u, wc)) break;
                mbar_arrive_expect_tx(&full[st], 2 * 16384);
                uint8_t *a = smem + st * SM::STAGE, *b = a + 16384;
                const int c = p.NC - 1 - kb / KB, t = c * L + 64 * (kb % KB);
#pragma unroll
                for (int mb = 0; mb < 2; ++mb) tma_load_3d(a + mb * 8192, &tm_q, d0 + 64 * mb, t, bh, &full[st]);
#pragma unroll
                for (int part = 0; part < 2; ++part) tma_load_3d(b + part * 8192, &tm_sg, j0, t, 2 * bh + part, &full[st]);
            }
            for (int s = 0; s < CSTAGES && s < kb; ++s) {
                const int last = kb - 1 - s;
                mbar_wait_drain(&full[last % CSTAGES], (uint32_t)(last / CSTAGES) & 1u);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t IDU = idesc_bf16(128, 64, 1, 1);
            bool ok = true;
            for (int i = 0; i < p.NC - 1 && ok; ++i) {   // i-th chunk from the end
                const int ub = i & 1;
                if (i >= 2 && !mbar_wait(&ufree[ub], (uint32_t)((i >> 1) - 1) & 1u, wc)) { ok = false; break; }
                for (int q = 0; q < KB; ++q) {
                    const int kb = i * KB + q, st = kb % CSTAGES;
                    if (!mbar_wait(&full[st], (uint32_t)(kb / CSTAGES) & 1u, wc)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a = smem_u32(smem + st * SM::STAGE), b = a + 16384;
#pragma unroll
                    for (int part = 0; part < 2; ++part)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_ss(tmem + ub * 64, smem_desc(a + kk * 2048, 8192, 1024),
                                   smem_desc(b + part * 8192 + kk * 2048, 8192, 1024), IDU,
                                   (q > 0 || part > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(&empty[st]);
                }
                if (ok) mma_commit(&ufull[ub]);
            }
        }
    } else {
        const int q4 = warp & 3;
        const int d = d0 + q4 * 32 + lane;   // this thread's state row
        const float *MCb = p.MC + (size_t)bh * (p.NC + 1);
        const float *Gb = p.G + (size_t)bh * p.NC;
        const float scale = rsqrtf((float)p.DK);
        float Gs[64];
#pragma unroll
        for (int x = 0; x < 64; ++x) Gs[x] = 0.f;
        float gn = 0.f;
        int c = p.NC - 1;
        float g_c = Gb[c], mc_c = MCb[c], mn_c = MCb[c + 1];
        // E_c = exp(g_c + m_c - m_{c+1}) (<G_end, C_c> + <dn_end, n_c>), the pairs of tokens that skip
        // chunk c (the forget-gate gradients): per warp its 32 rows of the tile, from C_c's bf16 value
        // part, which TMA brings into a swizzled tile two chunks ahead
        uint64_t *cfull = ufree + 2 + q4 * 2;
        uint8_t *cbuf = smem + SM::STG + 16384 + q4 * 8192;   // two 4 KB tiles
        uint8_t *gstg = smem + SM::STG + q4 * 4096;           // the chunk-end gradient out
        auto load_c = [&](int cc, int b) {
            mbar_arrive_expect_tx(&cfull[b], 4096);
            tma_load_3d(cbuf + b * 4096, &tm_c, j0, d0 + q4 * 32, 2 * (bh * p.NC + cc), &cfull[b]);
        };
        if (lane == 0) {
            load_c(c, 0);
            if (c >= 1) load_c(c - 1, 1);
        }
        auto nval = [&](int cc) { return with_n ? p.NS[((size_t)bh * p.NC + cc) * p.DK + d] : 0.f; };
        float nsv = nval(c);
        const int ep0 = ((int)blockIdx.y * (p.DV / 64) + (int)blockIdx.z) * 4 + q4;
        for (int i = 0; i < p.NC; ++i, --c) {
            const float decay = expf(g_c + mc_c - mn_c);
            if (c >= 1) {   // the next chunk's terms, one step ahead
                mn_c = mc_c;
                g_c = Gb[c - 1];
                mc_c = MCb[c - 1];
            }
            // this thread's share (8 independent sums); the warp's sum is taken and stored once the
            // chunk's step is handed back to the MMA warp
            const int b = i & 1;
            const bool cok = mbar_wait(&cfull[b], (uint32_t)(i >> 1) & 1u, wc);
            if (!__all_sync(0xffffffffu, cok)) break;
            float epart;
            {
                const uint8_t *crow = cbuf + b * 4096;
                float e8[8];
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    const uint4 cr = *reinterpret_cast<const uint4 *>(crow + sw_tile(lane, x));
                    const uint32_t w4[4] = {cr.x, cr.y, cr.z, cr.w};
                    float e = 0.f;
#pragma unroll
                    for (int z = 0; z < 4; ++z) {
                        e = fmaf(Gs[8 * x + 2 * z], __uint_as_float(w4[z] << 16), e);
                        e = fmaf(Gs[8 * x + 2 * z + 1], __uint_as_float(w4[z] & 0xffff0000u), e);
                    }
                    e8[x] = e;
                }
                epart = (((e8[0] + e8[1]) + (e8[2] + e8[3])) + ((e8[4] + e8[5]) + (e8[6] + e8[7]))) + gn * nsv;
                epart *= decay;   // (nsv is 0 outside the tiles of columns 0..63)
                __syncwarp();     // the tile has been read: it takes chunk c - 2
                if (lane == 0 && c >= 2) {
                    fence_proxy_async();
                    load_c(c - 2, b);
                }
                if (c >= 1) nsv = nval(c - 1);
            }
            const int c_ep = c;
            auto store_ep = [&]() {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) epart += __shfl_xor_sync(0xffffffffu, epart, o);
                if (lane == 0) EP[((size_t)bh * p.NC + c_ep) * NEP + ep0] = epart;
            };
            // the gradient of the state at this chunk's end: this warp's 32 rows through a swizzled
            // tile and a TMA store, once the previous chunk's store has read the tile
            if (lane == 0) bulk_wait_read0();
            __syncwarp();
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                uint4 w;
                w.x = bf16x2_bits(Gs[8 * x], Gs[8 * x + 1]);
                w.y = bf16x2_bits(Gs[8 * x + 2], Gs[8 * x + 3]);
                w.z = bf16x2_bits(Gs[8 * x + 4], Gs[8 * x + 5]);
                w.w = bf16x2_bits(Gs[8 * x + 6], Gs[8 * x + 7]);
                *reinterpret_cast<uint4 *>(gstg + sw_tile(lane, x)) = w;
            }
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) {
                tma_store_3d(&tm_g, gstg, j0, d0 + q4 * 32, bh * p.NC + c);
                bulk_commit();
            }
            float dn = 0.f;
            if (with_n) {
                float *slot = GN + ((size_t)bh * p.NC + c) * p.DK + d;
                dn = *slot;
                *slot = gn;
            }
            if (c == 0) {        // (the gradient of the start state is not needed)
                store_ep();
                break;
            }
            if (with_n) gn = fmaf(decay, gn, dn);
            const int ub = i & 1;
            bool failed = false;
            if (lane == 0) failed = !mbar_wait(&ufull[ub], (uint32_t)(i >> 1) & 1u, wc);
            if (__shfl_sync(0xffffffffu, failed ? 1 : 0, 0)) break;
            tc_fence_after();
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                uint32_t r[16];
                tmem_ld16(tmem_addr(tmem, q4 * 32, ub * 64 + g * 16), r);
                tmem_wait_ld();
#pragma unroll
                for (int z = 0; z < 16; ++z) Gs[g * 16 + z] = fmaf(decay, Gs[g * 16 + z], scale * __uint_as_float(r[z]));
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ufree[ub]);
            store_ep();
        }
        if (lane == 0) bulk_wait0();   // this warp's gradient stores are complete
    }
    tc_fence_before();
    __syncthreads();
    if (*reinterpret_cast<volatile uint32_t *>(abort_flag)) {
        const unsigned long long tb = global_timer();
        while (global_timer() - tb < 100000ull) { }
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

template <int L>
static cudaError_t launch_gstate_l(const Args &a)
{
    using SM = CarrySmem;
    CUtensorMap mq, msg, mg, mc;
    if (!map3(&mq, a.q, a.DK, a.S, a.BH) || !map3(&msg, a.sg16, a.DV, a.S, 2 * a.BH) ||
        !tcfwd::make_map(&mg, a.G16w, a.DV, a.DK, a.BH * a.NC, 32) ||
        !tcfwd::make_map(&mc, a.C16, a.DV, a.DK, 2 * a.BH * a.NC, 32))
        return cudaErrorInvalidValue;
    KParams p{};
    p.S = a.S; p.NC = a.NC; p.DK = a.DK; p.DV = a.DV;
    p.MC = a.MC; p.G = a.G; p.NS = a.NS;
    p.status = a.status;
    cudaError_t e = ensure_dynamic_smem((const void *)gstate_tc_kernel<L>, SM::TOTAL);
    if (e != cudaSuccess) return e;
    return launch_kernel(gstate_tc_kernel<L>, dim3(a.BH, a.DK / 128, a.DV / 64), dim3(THREADS), SM::TOTAL, a.stream, 1,
                         mq, msg, mg, mc, p, a.GNw, a.EPw, a.NEP);
}

cudaError_t launch_gstate(const Args &a)
{
    if (!supported(a.DK, a.DV, a.L)) return cudaErrorInvalidValue;
    return a.L == 64 ? launch_gstate_l<64>(a) : launch_gstate_l<128>(a);
}

template <int L>
static cudaError_t launch_carry_l(const Args &a)
{
    using SM = CarrySmem;
    const size_t items = (size_t)a.BH * a.S * (a.DK / 8);
    const unsigned nblk = (unsigned)std::min<size_t>((items + 255) / 256, 148 * 16);
    cudaError_t e = launch_kernel(wk_parts_kernel, dim3(nblk), dim3(256), 0, a.stream, 1, a.k, a.A, a.ig, a.G, a.MC,
                                  a.BH, a.S, L, a.NC, a.DK, a.wk16);
    if (e != cudaSuccess) return e;
    CUtensorMap mwk, mv, mcs;
    if (!map3(&mwk, a.wk16, a.DK, a.S, 2 * a.BH) || !map3(&mv, a.v, a.DV, a.S, a.BH) ||
        !tcfwd::make_map(&mcs, a.C16w, a.DV, a.DK, 2 * a.BH * a.NC, 32))
        return cudaErrorInvalidValue;
    KParams p{};
    p.S = a.S; p.NC = a.NC; p.DK = a.DK; p.DV = a.DV;
    p.MC = a.MC; p.G = a.G;
    p.status = a.status;
    if ((e = ensure_dynamic_smem((const void *)carry_tc_kernel<L>, SM::TOTAL)) != cudaSuccess) return e;
    return launch_kernel(carry_tc_kernel<L>, dim3(a.BH, a.DK / 128, a.DV / 64), dim3(THREADS), SM::TOTAL, a.stream, 1,
                         mwk, mv, mcs, p, a.NSw);
}

cudaError_t launch_carry(const Args &a)
{
    if (!supported(a.DK, a.DV, a.L)) return cudaErrorInvalidValue;
    return a.L == 64 ? launch_carry_l<64>(a) : launch_carry_l<128>(a);
}

// ---------------------------------------------------------------- the chunk's scores and dS
// One CTA per 128 consecutive tokens of a head (128 / L chunks): D = X Y^T over those tokens
// (M = N = 128, both operands K-major), of which only the blocks of each chunk with itself (on
// the diagonal) are used.  KIND 0: X = q, Y = k (bf16 inputs: the products are exact in the fp32
// accumulator), K = DK; A = D * scale * exp(x_s - mx_t) on the causal triangle (two bf16 parts),
// den_t = rowsum(A)_t + sc_t scale n_c . q_t and N_t.  KIND 1: X = g (two bf16 parts), Y = v,
// K = DV; dden_t, dS = (D + dden_t) exp(x_s - mx_t) on the causal triangle (bf16),
// dn_c = sum_t sc_t dden_t scale q_t and, for the forget-gate gradients, RECT_j = the sum of
// R_ts = dA_ts A_ts (dA = D + dden_t, A read back as its two parts) over the pairs s < j <= t of the
// chunk.  A TMEM lane is a token t (row), a column a token s.
constexpr int XSTAGES = 4;
struct ChunkSmem {
    static constexpr uint32_t STAGE = 2 * 16384;              // X and Y: 128 rows x 64 each
    // (once the MMAs are done, the stages take the epilogue's output tiles: per warp its 32 rows of A's
    // two parts or of dS, in [32][64] bf16 tiles under the 128-byte swizzle, stored by TMA)
    static constexpr uint32_t ATILE = XSTAGES * STAGE;        // the dS kernel's A rows, loaded by TMA
    static constexpr uint32_t F = ATILE + 4 * 2 * 2 * 4096;   // floats: xs, mx, fl, sc, dd [128]; ns [2][512]
    static constexpr uint32_t BAR = F + (5 * 128 + 2 * 512) * 4;
    static constexpr uint32_t NBAR = 2 * XSTAGES + 2;         // full, empty, accf, the A rows
    static constexpr uint32_t TOTAL = BAR + NBAR * 8 + 16 + 1024;
    static_assert(TOTAL <= 232448, "chunk smem");
};

template <int KIND, int L>
__global__ void __launch_bounds__(THREADS, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_y,
                const __grid_constant__ CUtensorMap tm_st, const __grid_constant__ CUtensorMap tm_a, Args a)
{
    using SM = ChunkSmem;
    constexpr int NPART = KIND == 1 ? 2 : 1;
    constexpr int CPB = 128 / L;                 // chunks per block
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    float *xs = reinterpret_cast<float *>(smem + SM::F), *mx = xs + 128, *fl = mx + 128, *sc = fl + 128;
    float *dd = sc + 128, *ns = dd + 128;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::BAR);
    uint64_t *full = bars, *empty = bars + XSTAGES, *accf = bars + 2 * XSTAGES, *abar = accf + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + SM::NBAR);
    constexpr int NB = L / 64;                   // 64-column boxes per row of the chunk's block
    constexpr int NPS = KIND == 0 ? 2 : 1;       // parts of the stored array (A: two, dS: one)
    uint32_t *abort_flag = tmem_slot + 1;
    const int bh = blockIdx.x, tb = blockIdx.y * 128;   // first token of the block
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nkb = NPART * (KIND == 0 ? a.DK : a.DV) / 64;
    WaitCtx wc{abort_flag, a.status};

    if (threadIdx.x == 0) {
        for (int s = 0; s < XSTAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accf, 1);
        mbar_init(abar, 1);
        *abort_flag = 0u;
        fence_barrier_init();
        tma_prefetch(&tm_x);
        tma_prefetch(&tm_y);
        tma_prefetch(&tm_st);
        if (KIND == 1) tma_prefetch(&tm_a);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    griddep_wait();
    griddep_launch_dependents();

    if (warp == 0) {
        if (lane == 0) {
            if (KIND == 1) {   // the rows of A (two parts) that the epilogue reads, first
                uint32_t bytes = 0;
                for (int w = 0; w < 4; ++w)
                    if ((tb + 32 * w) / L < a.NC) bytes += 2 * NB * 4096;
                mbar_arrive_expect_tx(abar, bytes);
                for (int w = 0; w < 4; ++w) {
                    const int t0w = tb + 32 * w, cw = t0w / L;
                    if (cw >= a.NC) continue;
                    for (int part = 0; part < 2; ++part)
                        for (int h = 0; h < NB; ++h)
                            tma_load_3d(smem + SM::ATILE + ((w * 2 + part) * NB + h) * 4096, &tm_a, 64 * h,
                                        (cw * 2 + part) * L + t0w % L, bh, abar);
                }
            }
            int kb = 0;
            for (; kb < nkb; ++kb) {
                const int st = kb % XSTAGES;
                if (kb >= XSTAGES && !mbar_wait(&empty[st], (uint32_t)((kb / XSTAGES) - 1) & 1u, wc)) break;
                mbar_arrive_expect_tx(&full[st], SM::STAGE);
                uint8_t *x = smem + st * SM::STAGE, *y = x + 16384;
                const int per = nkb / NPART, part = kb / per, k0 = 64 * (kb % per);
#pragma unroll
                for (int h = 0; h < 2; ++h) {   // rows tb .. tb + 127 in two boxes of 64
                    tma_load_3d(x + h * 8192, &tm_x, k0, tb + 64 * h, NPART * bh + part, &full[st]);
                    tma_load_3d(y + h * 8192, &tm_y, k0, tb + 64 * h, bh, &full[st]);
                }
            }
            for (int s = 0; s < XSTAGES && s < kb; ++s) {
                const int last = kb - 1 - s;
                mbar_wait_drain(&full[last % XSTAGES], (uint32_t)(last / XSTAGES) & 1u);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t ID = idesc_bf16(128, 128, 0, 0);
            bool ok = true;
            for (int kb = 0; kb < nkb; ++kb) {
                const int st = kb % XSTAGES;
                if (!mbar_wait(&full[st], (uint32_t)(kb / XSTAGES) & 1u, wc)) { ok = false; break; }
                tc_fence_after();
                const uint32_t x = smem_u32(smem + st * SM::STAGE), y = x + 16384;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ss(tmem, smem_desc(x, 16, 1024) + (uint64_t)(kk * 2), smem_desc(y, 16, 1024) + (uint64_t)(kk * 2),
                           ID, (kb > 0 || kk > 0) ? 1u : 0u);
                mma_commit(&empty[st]);
            }
            if (ok) mma_commit(accf);
        }
    } else {
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;          // this thread's token row in the block (TMEM lane: a
        const int r = row;                       // warp reaches its lane quadrant only)
        const int t = tb + row;                  // token within the head
        const int c = t / L, tl = t % L;         // its chunk and place in the chunk
        const int cb = (row / L) * L;            // the chunk's first column in the block
        const bool chunk_ok = c < a.NC;
        const int len = chunk_ok ? min(L, a.S - c * L) : 0;
        const bool ok_t = tl < len;
        const size_t gt = (size_t)bh * a.S + t;
        const float scale = rsqrtf((float)a.DK);
        // per-token gate terms (forms in which the chunk-local cumulative log decay cancels)
        {
            const float mc = chunk_ok ? a.MC[(size_t)bh * (a.NC + 1) + c] : 0.f;
            const float av = ok_t ? a.A[gt] : 0.f;
            const float m = ok_t ? fmaxf(mc, a.P[gt]) : 0.f;
            xs[r] = ok_t ? a.ig[gt] - av : -INFINITY;
            mx[r] = m;
            fl[r] = ok_t ? expf(-(av + m)) : 1.f;
            sc[r] = ok_t ? expf(mc - m) : 0.f;
        }
        float ddv = 0.f;
        if (KIND == 0) {   // n of the block's chunks
            for (int e = r; e < CPB * a.DK; e += 128) {
                const int cc = tb / L + e / a.DK;
                ns[e] = cc < a.NC ? a.NS[((size_t)bh * a.NC + cc) * a.DK + e % a.DK] : 0.f;
            }
        } else if (ok_t) {   // dden_t
            float dot = 0.f;
            for (int u = 0; u < a.NJT; ++u) dot += a.DOTP[gt * a.NJT + u];
            const float den = a.DENw[gt];   // (written by the scores kernel)
            if (fabsf(den) > fl[r]) ddv = -dot * copysignf(1.f, den);
            a.DDw[gt] = ddv;
        }
        dd[r] = ddv;
        named_sync(1, 128);
        bool failed = false;
        if (r == 0) failed = !mbar_wait(accf, 0, wc) || (KIND == 1 && !mbar_wait(abar, 0, wc));
        failed = group_any(2, 128, failed);
        // KIND 1: R_ts = dA_ts A_ts over the pairs s < t of the chunk (the derivative of the loss by
        // the log decay between s and t), summed along this row (rowl) and, per warp, down the columns
        // (cpart [4][128], in the n array's place)
        float rowl = 0.f;
        float *cpart = ns;
        if (!failed) {
            tc_fence_after();
            const float mxr = mx[r];
            float rsum = 0.f;
            // this row of the chunk's L x L block, A (two parts) or dS (one) with zeros off the triangle,
            // into the warp's output tiles (the stages, free now), then out by TMA
            uint8_t *stg = smem + q4 * (2 * NB * 4096);
            const uint8_t *atl = smem + SM::ATILE + q4 * (2 * NB * 4096);   // this warp's rows of A
#pragma unroll 1
            for (int g = 0; g < L / 16; ++g) {
                uint32_t rr[16];
                tmem_ld16(tmem_addr(tmem, q4 * 32, cb + g * 16), rr);
                const int hb = g >> 2, x0 = 2 * (g & 3);   // box and 16-byte chunk of columns 16 g ..
                uint4 ah[2] = {}, al[2] = {};
                if (KIND == 1) {   // this row of A (two parts: value and residue)
                    ah[0] = *reinterpret_cast<const uint4 *>(atl + hb * 4096 + sw_tile(lane, x0));
                    ah[1] = *reinterpret_cast<const uint4 *>(atl + hb * 4096 + sw_tile(lane, x0 + 1));
                    al[0] = *reinterpret_cast<const uint4 *>(atl + (NB + hb) * 4096 + sw_tile(lane, x0));
                    al[1] = *reinterpret_cast<const uint4 *>(atl + (NB + hb) * 4096 + sw_tile(lane, x0 + 1));
                }
                tmem_wait_ld();
                __nv_bfloat16 hi[16], lo[16];
                float rv[16];
#pragma unroll
                for (int z = 0; z < 16; ++z) {
                    const int sl = g * 16 + z;
                    float v = 0.f;
                    rv[z] = 0.f;
                    if (sl <= tl && ok_t) {
                        const float dcy = expf(xs[cb + sl] - mxr);
                        if (KIND == 0) {
                            v = __uint_as_float(rr[z]) * scale * dcy;
                        } else {
                            const float da = __uint_as_float(rr[z]) + ddv;
                            v = da * dcy;
                            const uint32_t wh = reinterpret_cast<const uint32_t *>(ah)[z >> 1];
                            const uint32_t wl = reinterpret_cast<const uint32_t *>(al)[z >> 1];
                            const float av = (z & 1) ? __uint_as_float(wh & 0xffff0000u) + __uint_as_float(wl & 0xffff0000u)
                                                     : __uint_as_float(wh << 16) + __uint_as_float(wl << 16);
                            if (sl < tl) rv[z] = da * av;
                        }
                    }
                    rsum += v;
                    if (KIND == 0) bf16_parts(v, hi[z], lo[z]);
                    else hi[z] = __float2bfloat16_rn(v);
                }
                if (KIND == 1) {
#pragma unroll
                    for (int z = 0; z < 16; ++z) rowl += rv[z];
                    const float cs = warp_sum16(rv, lane);   // the warp's 32 rows, column sum16_index(lane)
                    if ((lane & 1) == 0) cpart[q4 * 128 + cb + g * 16 + sum16_index(lane)] = cs;
                }
                *reinterpret_cast<uint4 *>(stg + hb * 4096 + sw_tile(lane, x0)) = *reinterpret_cast<const uint4 *>(hi);
                *reinterpret_cast<uint4 *>(stg + hb * 4096 + sw_tile(lane, x0 + 1)) = *reinterpret_cast<const uint4 *>(hi + 8);
                if (KIND == 0) {
                    *reinterpret_cast<uint4 *>(stg + (NB + hb) * 4096 + sw_tile(lane, x0)) = *reinterpret_cast<const uint4 *>(lo);
                    *reinterpret_cast<uint4 *>(stg + (NB + hb) * 4096 + sw_tile(lane, x0 + 1)) = *reinterpret_cast<const uint4 *>(lo + 8);
                }
            }
            fence_proxy_async();
            __syncwarp();
            if (lane == 0 && chunk_ok) {   // (a warp's 32 rows lie in one chunk)
                for (int part = 0; part < NPS; ++part)
                    for (int h = 0; h < NB; ++h)
                        tma_store_3d(&tm_st, stg + (part * NB + h) * 4096, 64 * h, (c * NPS + part) * L + (tl - lane), bh);
                bulk_commit();
            }
            if (KIND == 0 && ok_t) {   // den and N
                const float *nc = ns + (row / L) * a.DK;
                const __nv_bfloat16 *qr = a.q + gt * a.DK;
                float qn = 0.f;
                for (int d = 0; d < a.DK; d += 8) {
                    const uint4 u = *reinterpret_cast<const uint4 *>(qr + d);
                    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int z = 0; z < 4; ++z) {
                        qn = fmaf(nc[d + 2 * z], __uint_as_float(w4[z] << 16), qn);
                        qn = fmaf(nc[d + 2 * z + 1], __uint_as_float(w4[z] & 0xffff0000u), qn);
                    }
                }
                const float den = rsum + qn * scale * sc[r];
                a.DENw[gt] = den;
                a.NRMw[gt] = fmaxf(fabsf(den), fl[r]);
            }
        }
        if (KIND == 1) {   // dn_c = sum_t sc_t dden_t scale q_t of each chunk of the block
            named_sync(1, 128);
            float *drow = ns + 512;   // [128] colb_t - rowl_t
            if (!failed) {
                for (int cc = 0; cc < CPB; ++cc) {
                    const int ch = tb / L + cc;
                    if (ch >= a.NC) break;
                    const int clen = min(L, a.S - ch * L);
                    const __nv_bfloat16 *qb = a.q + ((size_t)bh * a.S + ch * L) * a.DK;
                    // a thread per column pair; four independent sums, so that the loads of q overlap
                    for (int i = 2 * r; i < a.DK; i += 256) {
                        float ax[4] = {0.f, 0.f, 0.f, 0.f}, ay[4] = {0.f, 0.f, 0.f, 0.f};
                        int u = 0;
                        for (; u + 4 <= clen; u += 4) {
#pragma unroll
                            for (int z = 0; z < 4; ++z) {
                                const float w = sc[cc * L + u + z] * dd[cc * L + u + z];
                                const uint32_t qq = *reinterpret_cast<const uint32_t *>(qb + (size_t)(u + z) * a.DK + i);
                                ax[z] = fmaf(w, __uint_as_float(qq << 16), ax[z]);
                                ay[z] = fmaf(w, __uint_as_float(qq & 0xffff0000u), ay[z]);
                            }
                        }
                        for (; u < clen; ++u) {
                            const float w = sc[cc * L + u] * dd[cc * L + u];
                            const uint32_t qq = *reinterpret_cast<const uint32_t *>(qb + (size_t)u * a.DK + i);
                            ax[0] = fmaf(w, __uint_as_float(qq << 16), ax[0]);
                            ay[0] = fmaf(w, __uint_as_float(qq & 0xffff0000u), ay[0]);
                        }
                        float *gd = a.GNw + ((size_t)bh * a.NC + ch) * a.DK + i;
                        gd[0] = ((ax[0] + ax[1]) + (ax[2] + ax[3])) * scale;
                        gd[1] = ((ay[0] + ay[1]) + (ay[2] + ay[3])) * scale;
                    }
                }
                // colb_t: the column sum of R below the diagonal, over the warps of this row's chunk
                const int w0 = (r / L) * (L / 32);
                float colb = 0.f;
                for (int w2 = w0; w2 < w0 + L / 32; ++w2) colb += cpart[w2 * 128 + r];
                drow[r] = colb - rowl;
            }
            named_sync(1, 128);
            // RECT_j = sum_{s < j} drow_s over the chunk: the pairs s < j <= t inside it (a warp per
            // chunk, a scan in fp64)
            if (!failed && q4 < CPB) {
                const int ch = tb / L + q4;
                if (ch < a.NC) {
                    constexpr int PER = L / 32;
                    const int clen = min(L, a.S - ch * L);
                    const float *dv = drow + q4 * L + lane * PER;
                    double loc = 0.0;
#pragma unroll
                    for (int u = 0; u < PER; ++u) loc += (double)dv[u];
                    double inc = loc;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const double y = __shfl_up_sync(0xffffffffu, inc, o);
                        if (lane >= o) inc += y;
                    }
                    double run = inc - loc;
#pragma unroll
                    for (int u = 0; u < PER; ++u) {
                        const int tl2 = lane * PER + u;
                        if (tl2 < clen) a.RECTw[(size_t)bh * a.S + (size_t)ch * L + tl2] = (float)run;
                        run += (double)dv[u];
                    }
                }
            }
        }
        if (lane == 0) bulk_wait0();   // this warp's output tiles are stored
    }
    tc_fence_before();
    __syncthreads();
    if (*reinterpret_cast<volatile uint32_t *>(abort_flag)) {
        const unsigned long long tq = global_timer();
        while (global_timer() - tq < 100000ull) { }
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

template <int KIND, int L>
static cudaError_t launch_chunk_l(const Args &a)
{
    using SM = ChunkSmem;
    CUtensorMap mx, my, mst, ma;
    // the stored array's rows: A [NC][2][L][L] or dS [NC][L][L] per head, in [32][64] boxes; the dS
    // kernel also reads A's rows
    if (!tcfwd::make_map(&mst, KIND == 0 ? (const void *)a.A16w : (const void *)a.dS16w, L,
                         (KIND == 0 ? 2 : 1) * a.NC * L, a.BH, 32) ||
        !tcfwd::make_map(&ma, a.A16, L, 2 * a.NC * L, a.BH, 32))
        return cudaErrorInvalidValue;
    if (KIND == 0) {
        if (!map3(&mx, a.q, a.DK, a.S, a.BH) || !map3(&my, a.k, a.DK, a.S, a.BH)) return cudaErrorInvalidValue;
    } else {
        if (!map3(&mx, a.g16, a.DV, a.S, 2 * a.BH) || !map3(&my, a.v, a.DV, a.S, a.BH)) return cudaErrorInvalidValue;
    }
    cudaError_t e = ensure_dynamic_smem((const void *)chunk_tc_kernel<KIND, L>, SM::TOTAL);
    if (e != cudaSuccess) return e;
    return launch_kernel(chunk_tc_kernel<KIND, L>, dim3(a.BH, (a.S + 127) / 128), dim3(THREADS), SM::TOTAL, a.stream, 1,
                         mx, my, mst, ma, a);
}

cudaError_t launch_scores(const Args &a)
{
    if (!supported(a.DK, a.DV, a.L)) return cudaErrorInvalidValue;
    return a.L == 64 ? launch_chunk_l<0, 64>(a) : launch_chunk_l<0, 128>(a);
}

cudaError_t launch_ds(const Args &a)
{
    if (!supported(a.DK, a.DV, a.L)) return cudaErrorInvalidValue;
    return a.L == 64 ? launch_chunk_l<1, 64>(a) : launch_chunk_l<1, 128>(a);
}

bool supported(int DK, int DV, int L)
{
    return (L == 64 || L == 128) && DK % TM == 0 && DV % TM == 0 && DK <= 512 && DV <= 512;
}

cudaError_t launch(const Args &a)
{
    if (!supported(a.DK, a.DV, a.L)) return cudaErrorInvalidValue;
    return a.L == 64 ? launch_l<64>(a) : launch_l<128>(a);
}

}  // namespace bwdtc
}  // namespace mlstm
