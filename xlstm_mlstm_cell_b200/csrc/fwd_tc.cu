// fwd_tc.cu -- chunkwise forward pass on the 5th-generation tensor cores (tcgen05, TMEM, TMA).
//
// Inputs q, k, v, o are bf16; gates, states and accumulation are fp32.  The
// sequence of every (batch, head) is cut into chunks of L tokens, and the chunks
// into NSEG segments of R chunks.  Three kernels follow the gate preprocessing:
//
// 1. segsum (tensor cores): for every segment, its contribution to the state,
//      dC_s^T = V_s^T diag(w) K_s,  dn_s = K_s^T w,
//      w_t = exp(G_s - A_t + i~_t - b_s) <= 1
//    where A_t is the segment-local cumulative log decay, G_s its total and
//    (G_s, b_s) the max-plus map of the segment (the composition of its chunk
//    maps).  One long-K GEMM per (segment, value tile); K rows are scaled by w
//    in shared memory between the TMA load and the MMA.
// 2. seg_scan (CUDA cores): the state at every segment start by an in-place
//    exclusive scan over segments,
//      C_{s+1} = exp(G_s + M_s - M_{s+1}) C_s + exp(b_s - M_{s+1}) dC_s,
//    and the final state.  This is the scan across chunks of the xLSTM Guide's
//    "Exploit Chunkwise Hardware Kernels for Production Training", taken per
//    segment.
// 3. walk (tensor cores): one CTA per (segment, 128-wide value tile) starts from
//    the segment's state, kept in TMEM in fp32, and walks its chunks in order.
//    Per chunk, with the per-token stabilizer m and chunk-local cumulative log
//    decay a of the gate preprocessing:
//      S   = Q K^T                                      (tcgen05, fp32 in TMEM)
//      P   = S * D * d^-1/2,  D_ts = exp(a_t - a_s + i~_s - m_t), s <= t      (<= 1)
//      H^T = Cb^T Q'^T + V^T P'^T                       (tcgen05; Cb^T read from TMEM)
//      h_t = o_t * r_t H_t / max(|rowsum(P)_t + sc_t q_t . n|, exp(-m_t))
//      C^T += V^T K',  n += sum_s W_s k_s               (state for the next chunk)
//    with sc_t = exp(a_t + m_c - m_t) / sqrt(d) = r_t 2^e_t (r_t in [1, 2)),
//    Q' = diag(2^(e_t + kc)) Q and Cb = C_c 2^-kc in fp16 (kc a power-of-two range
//    scale per chunk; q is bf16, so Q' is exact), P' = diag(1/r) P in bf16 and
//    K' = diag(W) K in bf16.  The causal decay matrix D and the inter-chunk term
//    are those of the guide's "The Dual Formulation" restricted to a chunk.
//    The normalizer and the inter-chunk part of the denominator are computed in
//    fp32 from the unrounded q and k: rounding them dominated the error through
//    cancellation in the denominator, and the fp16 inter-chunk product keeps
//    inputs with one dominant token (huge input gates) within the error budget.
//
//    At chunk 64 the inter-chunk product instead reads the fp32 state in TMEM
//    directly as a tf32 operand (kind::tf32, Q' in fp32 shared memory), so no
//    fp16 copy Cb is made per chunk.
//
//    The state in TMEM is kept in a lazily rescaled frame: TMEM holds
//    X = Cbar exp(-rho) (Cbar the unstabilized state), the chunk decay is folded
//    into rho instead of rescaling TMEM, and new tokens enter with weight
//    W_s = exp(i~_s - a_s - rho) <= exp(THRESH).  TMEM is rescaled only when that
//    bound would be exceeded, between the chunk's read-out and its state update, so
//    that the read-out always sees the chunk's starting frame (rho >= m_c - THRESH).
//    Cb is always the stabilized C_c = X exp(rho - m_c).
#include "common.cuh"
#include "mlstm_internal.h"
#include "tc_common.cuh"
#include "tc_fwd.h"

#include <cudaTypedefs.h>

namespace mlstm {
namespace tcfwd {

using namespace tc;

constexpr int DVT = 128;         // value columns per CTA (TMEM lanes of the state)
constexpr int TB = 64;           // tokens per pipeline stage in segsum
constexpr int SS_STAGES = 4;
constexpr float THRESH = 20.f;   // log of the largest weight before TMEM is rescaled
constexpr float LOG2E = 1.4426950408889634f;

// Optional timeline trace of the walk (build with -DMLSTM_WALK_TRACE): clock64 stamps of
// the three roles of tile 0, head 0, per segment and chunk.  Off in normal builds.
#ifdef MLSTM_WALK_TRACE
constexpr int TR_SLOTS = 24, TR_CHUNKS = 256, TR_SEGS = 64;
__device__ long long g_walk_trace[TR_SEGS * TR_CHUNKS * TR_SLOTS];
#define WALK_TRACE_AT(slot, ci)                                                                            \
    do {                                                                                                   \
        if (tile == 0 && bh == 0 && seg < TR_SEGS && (ci) < TR_CHUNKS)                                     \
            g_walk_trace[((size_t)seg * TR_CHUNKS + (ci)) * TR_SLOTS + (slot)] = clock64();                \
    } while (0)
// segment sums of CTA (0, 1, 0): clock64 per stage (rows 0..63) and per kernel phase (row 64)
__device__ long long g_seg_trace[65 * 8];
#define SEG_TRACE(row, slot)                                                                               \
    do {                                                                                                   \
        if (blockIdx.x == 0 && blockIdx.y == 1 && blockIdx.z == 0 && (row) < 65)                           \
            g_seg_trace[(row) * 8 + (slot)] = clock64();                                                   \
    } while (0)
#else
#define WALK_TRACE_AT(slot, ci) do { } while (0)
#define SEG_TRACE(row, slot) do { } while (0)
#endif
#define WALK_TRACE(slot) WALK_TRACE_AT(slot, i)


// ---------------------------------------------------------------- segsum

// NT value tiles of 128 columns per CTA (one TMEM accumulator of DK columns each): with NT = 2
// a K tile loaded and scaled once serves 256 value columns.
template <int DK, int NT>
struct SegSmem {
    static constexpr int STAGES = NT == 2 ? 3 : SS_STAGES;
    static constexpr uint32_t K_BYTES = DK * TB * 2;
    static constexpr uint32_t V_BYTES = NT * DVT * TB * 2;
    static constexpr uint32_t STAGE = K_BYTES + V_BYTES;
    static constexpr uint32_t BAR_OFF = STAGE * STAGES;
    static constexpr uint32_t TOTAL = BAR_OFF + 128 + TB * 4 + 1024;   // + barriers, weights, alignment slack
    static constexpr uint32_t TMEM_COLS = NT * DK < 32 ? 32 : NT * DK;
};

constexpr int SS_SCALERS = 8;                     // scaler warps of segsum_kernel
constexpr int SS_THREADS = 64 + SS_SCALERS * 32;  // producer warp, MMA warp, scalers

template <int DK, int NT>
__global__ void __launch_bounds__(SS_THREADS, 1)
segsum_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, Params p)
{
    using SM = SegSmem<DK, NT>;
    constexpr int SS_STAGES = SM::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + SM::BAR_OFF);
    uint64_t *scaled = full + SS_STAGES;
    uint64_t *empty = scaled + SS_STAGES;
    uint64_t *acc_full = empty + SS_STAGES;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 1);
    uint32_t *abort_flag = tmem_slot + 1;
    float *wst = reinterpret_cast<float *>(smem + SM::BAR_OFF + 128);   // [TB] weights of the stage

    const int tile = blockIdx.x, seg = blockIdx.y, bh = blockIdx.z;
    const int j0 = tile * DVT * NT;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t_begin = seg * p.R * p.L;
    const int t_end = min(t_begin + p.R * p.L, p.S);
    const int nstage = (t_end - t_begin + TB - 1) / TB;
    WaitCtx wc{abort_flag, p.status};

    if (threadIdx.x == 0) {
        for (int i = 0; i < SS_STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&scaled[i], SS_SCALERS);
            mbar_init(&empty[i], 1);
        }
        mbar_init(acc_full, 1);
        *abort_flag = 0u;
        fence_barrier_init();
        tma_prefetch(&tm_k);
        tma_prefetch(&tm_v);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, SM::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // The TMA producer (warp 0) loads only the inputs q, k, v, which no kernel of this call writes
    // (this kernel launches only once every earlier grid of the stream has passed its own
    // griddepcontrol.wait, so their producers have finished), and the MMA warp (warp 1) reads
    // shared memory and TMEM only: their first loads and MMAs go out while the preceding kernel
    // is still running.  The warps that read its outputs wait for them.
    if (warp >= 2) griddep_wait();
    griddep_launch_dependents();
    if (threadIdx.x == 0) SEG_TRACE(64, 0);

    if (warp == 0) {
        if (lane == 0) {   // TMA producer
            int issued = 0;
            for (int it = 0; it < nstage; ++it) {
                const int st = it % SS_STAGES;
                const uint32_t ph = (uint32_t)(it / SS_STAGES) & 1u;
                if (it >= SS_STAGES && !mbar_wait(&empty[st], ph ^ 1u, wc)) break;
                SEG_TRACE(it, 0);
                ++issued;
                uint8_t *kb = smem + st * SM::STAGE;
                uint8_t *vb = kb + SM::K_BYTES;
                const int t0 = t_begin + it * TB;
                mbar_arrive_expect_tx(&full[st], SM::STAGE);
                for (int b = 0; b < DK / 64; ++b) tma_load_3d(kb + b * TB * 128, &tm_k, b * 64, t0, bh, &full[st]);
                for (int b = 0; b < NT * DVT / 64; ++b)
                    tma_load_3d(vb + b * TB * 128, &tm_v, j0 + b * 64, t0, bh, &full[st]);
            }
            for (int it = issued > SS_STAGES ? issued - SS_STAGES : 0; it < issued; ++it)   // drain
                mbar_wait_drain(&full[it % SS_STAGES], (uint32_t)(it / SS_STAGES) & 1u);
        }
    } else if (warp == 1) {
        if (lane == 0) {   // MMA issuer: dC^T (DVT x DK) += V^T (DVT x TB) * K' (TB x DK)
            constexpr uint32_t IDESC = idesc_bf16(DVT, DK, 1, 1);
            int it = 0;
            for (; it < nstage; ++it) {
                const int st = it % SS_STAGES;
                const uint32_t ph = (uint32_t)(it / SS_STAGES) & 1u;
                if (!mbar_wait(&scaled[st], ph, wc)) break;
                SEG_TRACE(it, 3);
                tc_fence_after();
                const uint32_t kb = smem_u32(smem + st * SM::STAGE);
                const uint32_t vb = kb + SM::K_BYTES;
#pragma unroll
                for (int t = 0; t < NT; ++t)
#pragma unroll
                    for (int k = 0; k < TB / 16; ++k) {
                        const uint64_t a = smem_desc(vb + t * 2 * TB * 128 + k * 2048, TB * 128, 1024);
                        const uint64_t b = smem_desc(kb + k * 2048, TB * 128, 1024);
                        mma_ss(tmem + t * DK, a, b, IDESC, (it > 0 || k > 0) ? 1u : 0u);
                    }
                mma_commit(&empty[st]);
                SEG_TRACE(it, 4);
            }
            mma_commit(acc_full);
            mbar_wait_drain(acc_full, 0);
        }
    } else {
        // scalers (warps 2..): K rows *= w in place; tile 0 also sums dn = sum_t w_t k_t in fp32 from
        // the unrounded bf16 k.  A warp takes RPW rows at a time, one 16-byte chunk per lane.
        constexpr int NST = SS_SCALERS * 32;             // scaler threads
        const int ct = threadIdx.x - 64;                 // 0..NST-1
        const int sw = ct >> 5;                          // scaler warp
        constexpr int CPR = DK / 8;                      // 16-byte chunks per row
        constexpr int RPW = 32 / CPR;                    // rows per warp step
        constexpr int RSTEP = SS_SCALERS * RPW;
        constexpr int NB = (TB / RSTEP) < 4 ? (TB / RSTEP) : 4;   // rows in flight per iteration
        static_assert(TB % (RSTEP * NB) == 0, "segsum row pass unroll");
        const int rsub = lane / CPR, jc = lane % CPR;
        const float Gs = p.SGb[((size_t)bh * p.NSEG + seg) * 2 + 0];
        const float bs = p.SGb[((size_t)bh * p.NSEG + seg) * 2 + 1];
        const float *Ab = p.A + (size_t)bh * p.S;
        const float *igb = p.ig + (size_t)bh * p.S;
        const float *GPb = p.GP + (size_t)bh * p.NC;
        float nacc[8];
#pragma unroll
        for (int z = 0; z < 8; ++z) nacc[z] = 0.f;
        bool ok = true;
        // this thread's token weight of the next stage, loaded one stage ahead (threads 0..TB-1)
        float pa = 0.f, pi = 0.f, pgp = 0.f;
        if (ct < TB && t_begin + ct < t_end) {
            pa = Ab[t_begin + ct];
            pi = igb[t_begin + ct];
            pgp = GPb[(t_begin + ct) / p.L];
        }
        for (int it = 0; it < nstage; ++it) {
            const int st = it % SS_STAGES;
            const uint32_t ph = (uint32_t)(it / SS_STAGES) & 1u;
            const int t = t_begin + it * TB + ct;
            const float ca = pa, ci = pi, cgp = pgp;
            if (ct < TB && t + TB < t_end) {             // prefetch the next stage's gate values
                pa = Ab[t + TB];
                pi = igb[t + TB];
                pgp = GPb[(t + TB) / p.L];
            }
            named_sync(1, NST);                          // the previous stage's readers of wst are done
            if (ct < TB) wst[ct] = (t < t_end) ? expf(Gs - cgp - ca + ci - bs) : 0.f;
            named_sync(1, NST);
            if (!mbar_wait(&full[st], ph, wc)) { ok = false; break; }
            if (ct == 0) SEG_TRACE(it, 1);
            uint8_t *kb = smem + st * SM::STAGE;
            for (int row0 = sw * RPW + rsub; row0 < TB; row0 += RSTEP * NB) {
                uint4 uk[NB];
#pragma unroll
                for (int b2 = 0; b2 < NB; ++b2)
                    uk[b2] = *reinterpret_cast<const uint4 *>(kb + sw128_chunk(row0 + b2 * RSTEP, jc, TB));
#pragma unroll
                for (int b2 = 0; b2 < NB; ++b2) {
                    const int row = row0 + b2 * RSTEP;
                    const float w = wst[row];
                    const float2 f0 = unpack_bf16(uk[b2].x), f1 = unpack_bf16(uk[b2].y), f2 = unpack_bf16(uk[b2].z),
                                 f3 = unpack_bf16(uk[b2].w);
                    if (tile == 0) {
                        nacc[0] += w * f0.x; nacc[1] += w * f0.y; nacc[2] += w * f1.x; nacc[3] += w * f1.y;
                        nacc[4] += w * f2.x; nacc[5] += w * f2.y; nacc[6] += w * f3.x; nacc[7] += w * f3.y;
                    }
                    *reinterpret_cast<uint4 *>(kb + sw128_chunk(row, jc, TB)) =
                        make_uint4(pack_bf16(f0.x * w, f0.y * w), pack_bf16(f1.x * w, f1.y * w),
                                   pack_bf16(f2.x * w, f2.y * w), pack_bf16(f3.x * w, f3.y * w));
                }
            }
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(&scaled[st]);
            if (ct == 0) SEG_TRACE(it, 2);
        }
        if (tile == 0) {    // reduce the n partial sums of the scaler warps (and lanes sharing a chunk)
            float *npart = reinterpret_cast<float *>(smem);      // stage buffers are idle once acc_full fires
            if (ok && mbar_wait(acc_full, 0, wc)) {
#pragma unroll
                for (int z = 0; z < 8; ++z) npart[(sw * RPW + rsub) * DK + jc * 8 + z] = nacc[z];
            }
            named_sync(1, NST);
            if (ok) {
                for (int d = ct; d < DK; d += NST) {
                    float acc = 0.f;
                    for (int pr = 0; pr < SS_SCALERS * RPW; ++pr) acc += npart[pr * DK + d];
                    p.DN[((size_t)bh * p.NSEG + seg) * DK + d] = acc;
                }
            }
        }
        // epilogue: TMEM (lane = value column, columns = DK) -> workspace, quad layout [DK/4][DV][4]
        if (ok && mbar_wait(acc_full, 0, wc)) {
            if (ct == 0) SEG_TRACE(64, 1);
            tc_fence_after();
            const int q = warp & 3;                      // TMEM lane quadrant of the warp
            const int half = (warp - 2) >> 2;            // two scaler warps per quadrant share its columns
            float *dst = p.DC + ((size_t)bh * p.NSEG + seg) * (size_t)DK * p.DV;
            for (int tc = half * 32; tc < NT * DK; tc += 64) {
                const int t = tc / DK, c0 = tc % DK;
                const int j = t * DVT + q * 32 + lane;
                uint32_t r[32];
                tmem_ld32(tmem_addr(tmem, q * 32, tc), r);
                tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    float4 v4 = make_float4(__uint_as_float(r[4 * u]), __uint_as_float(r[4 * u + 1]),
                                            __uint_as_float(r[4 * u + 2]), __uint_as_float(r[4 * u + 3]));
                    *reinterpret_cast<float4 *>(dst + ((size_t)((c0 >> 2) + u) * p.DV + j0 + j) * 4) = v4;
                }
            }
        }
    }
    if (threadIdx.x == 64) SEG_TRACE(64, 2);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, SM::TMEM_COLS);
    }
}

// ---------------------------------------------------------------- scan over segments

constexpr int SCAN_MAX_SEG = 256;   // segments per head handled by seg_scan_kernel's shared tables

__global__ void __launch_bounds__(256)
seg_scan_kernel(Params p, float *C_final, float *n_final, float *__restrict__ m_final, const float *C0,
                const float *n0)
{
    griddep_wait();
    griddep_launch_dependents();
    __shared__ float gam[SCAN_MAX_SEG], bet[SCAN_MAX_SEG];
    const int bh = blockIdx.y;
    const int nquad = p.DK * p.DV / 4;
    const int e = blockIdx.x * blockDim.x + threadIdx.x;    // quad index: (i4, j) = (e / DV, e % DV)
    const float *MCb = p.MC + (size_t)bh * (p.NC + 1);
    const float *SG = p.SGb + (size_t)bh * p.NSEG * 2;
    constexpr int BATCH = 8;                           // contributions loaded ahead of the stores
    float4 *__restrict__ slot0 = reinterpret_cast<float4 *>(p.DC + (size_t)bh * p.NSEG * p.DK * p.DV) + e;
    const size_t stride = (size_t)p.DK * p.DV / 4;
    // the first batch of contributions is requested before the per-segment factors are formed,
    // so that the two memory latencies overlap
    float4 d[BATCH];
#pragma unroll
    for (int u = 0; u < BATCH; ++u)
        if (e < nquad && u < p.NSEG) d[u] = __ldcs(slot0 + u * stride);
    // decay of the running state and weight of the segment's contribution, per segment
    for (int s = threadIdx.x; s < p.NSEG; s += blockDim.x) {
        const float Ms = MCb[s * p.R], Mn = MCb[min((s + 1) * p.R, p.NC)];
        gam[s] = expf(SG[2 * s] + Ms - Mn);
        bet[s] = expf(SG[2 * s + 1] - Mn);
    }
    __syncthreads();
    if (e < nquad) {
        float4 C = make_float4(0.f, 0.f, 0.f, 0.f);
        if (C0) {   // initial state (user layout); C_final may alias C0: each element is read before written
            const int i4 = e / p.DV, j = e % p.DV;
            const float *c0 = C0 + (size_t)bh * p.DK * p.DV;
            C = make_float4(c0[(size_t)(4 * i4 + 0) * p.DV + j], c0[(size_t)(4 * i4 + 1) * p.DV + j],
                            c0[(size_t)(4 * i4 + 2) * p.DV + j], c0[(size_t)(4 * i4 + 3) * p.DV + j]);
        }
        for (int s0 = 0; s0 < p.NSEG; s0 += BATCH) {
            if (s0 > 0) {
#pragma unroll
                for (int u = 0; u < BATCH; ++u)
                    if (s0 + u < p.NSEG) d[u] = __ldcs(slot0 + (s0 + u) * stride);
            }
#pragma unroll
            for (int u = 0; u < BATCH; ++u) {
                const int s = s0 + u;
                if (s < p.NSEG) {
                    slot0[s * stride] = C;
                    const float ga = gam[s], be = bet[s];
                    C.x = ga * C.x + be * d[u].x;
                    C.y = ga * C.y + be * d[u].y;
                    C.z = ga * C.z + be * d[u].z;
                    C.w = ga * C.w + be * d[u].w;
                }
            }
        }
        if (C_final) {
            const int i4 = e / p.DV, j = e % p.DV;
            float *cf = C_final + (size_t)bh * p.DK * p.DV;
            cf[(size_t)(4 * i4 + 0) * p.DV + j] = C.x;
            cf[(size_t)(4 * i4 + 1) * p.DV + j] = C.y;
            cf[(size_t)(4 * i4 + 2) * p.DV + j] = C.z;
            cf[(size_t)(4 * i4 + 3) * p.DV + j] = C.w;
        }
    }
    if (blockIdx.x == 0) {
        for (int i = threadIdx.x; i < p.DK; i += blockDim.x) {
            float n = n0 ? n0[(size_t)bh * p.DK + i] : 0.f;
            for (int s = 0; s < p.NSEG; ++s) {
                float *slot = p.DN + ((size_t)bh * p.NSEG + s) * p.DK + i;
                const float d = *slot;
                *slot = n;
                n = gam[s] * n + bet[s] * d;
            }
            if (n_final) n_final[(size_t)bh * p.DK + i] = n;
        }
        if (m_final && threadIdx.x == 0) m_final[bh] = MCb[p.NC];
    }
}

// ---------------------------------------------------------------- walk

template <int DK, int L>
struct WalkSmem {
    static constexpr bool TF = (L == 64);           // see Q32_OFF
    static constexpr int KB = TF ? 2 : 1;           // K tiles in flight (chunk 64: the next chunk's K
                                                    // loads while this chunk's K' feeds the state update)
    static constexpr uint32_t KBYTES = DK * L * 2;
    static constexpr uint32_t Q_OFF = 0;
    static constexpr uint32_t K_OFF = Q_OFF + DK * L * 2;
    static constexpr uint32_t V_OFF = K_OFF + KB * KBYTES;
    static constexpr uint32_t P_OFF = V_OFF + DVT * L * 2;
    // transpose staging of the output epilogue (16 warps x 2 KB): the P tile when it is 32 KB
    static constexpr uint32_t T_OFF = (L * L * 2 >= 32768) ? P_OFF : P_OFF + L * L * 2;
    static constexpr uint32_t T_END = T_OFF == P_OFF ? P_OFF + L * L * 2 : T_OFF + 32768;
    // chunk 64: the inter-chunk product runs in tf32 straight from the fp32 state in TMEM, with
    // Q' in fp32 (a 128-byte-swizzled K-major tile of DK / 32 blocks); chunk 128 keeps the fp16
    // state copy in TMEM and Q' in fp16 in place of Q (an fp32 Q' would not fit in shared memory)
    static constexpr uint32_t Q32_OFF = T_END;
    static constexpr uint32_t F_OFF = Q32_OFF + (TF ? DK * L * 4 : 0);   // float arrays
    // float arrays: arow, mrow, icol, srow, wcol [L]; rs [4][L]; inv, qexp, rrow, ccol [L];
    // dpart [512] (partial q . n of the Q pass); bcol [16]; nX [DK]; red [16]
    static constexpr uint32_t NF = L * 13 + 512 + 16 + DK + 16;
    static constexpr uint32_t BAR_OFF = F_OFF + NF * 4;
    static constexpr uint32_t TOTAL = BAR_OFF + 16 * 8 + 16 + 1024;
    static constexpr uint32_t C_COL = 0, CB_COL = DK, HS_COL = TF ? DK : DK + DK / 2;
    // chunk 128: S and H^T share one accumulator; chunk 64: separate ones, so that the next chunk's
    // S = Q K^T runs while this chunk's outputs are read
    static constexpr uint32_t S_COL = HS_COL, H_COL = TF ? HS_COL + L : HS_COL;
    static constexpr uint32_t TMEM_USED = H_COL + L;
    static constexpr uint32_t TMEM_COLS = TMEM_USED <= 128 ? 128 : (TMEM_USED <= 256 ? 256 : 512);
};

constexpr int WALK_THREADS = 64 + 16 * 32;   // producer warp, MMA warp, 16 epilogue warps

template <int DK, int L>
__global__ void __launch_bounds__(WALK_THREADS, 1)
walk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const __grid_constant__ CUtensorMap tm_v, Params p)
{
    using SM = WalkSmem<DK, L>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *Qs = smem + SM::Q_OFF;
    uint8_t *Ks = smem + SM::K_OFF;
    uint8_t *Vs = smem + SM::V_OFF;
    uint8_t *Ps = smem + SM::P_OFF;
    uint8_t *Ts = smem + SM::T_OFF;
    float *F = reinterpret_cast<float *>(smem + SM::F_OFF);
    float *arow = F, *mrow = F + L, *icol = F + 2 * L, *srow = F + 3 * L, *wcol = F + 4 * L;
    float *rs = F + 5 * L, *inv = F + 9 * L, *qexp = F + 10 * L, *rrow = F + 11 * L, *ccol = F + 12 * L;
    float *dpart = F + 13 * L, *bcol = dpart + 512, *nX = bcol + 16, *red = nX + DK;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::BAR_OFF);
    uint64_t *q_full = bars + 0, *k_full = bars + 1, *v_full = bars + 2, *s_full = bars + 3, *h_full = bars + 4;
    uint64_t *c_upd = bars + 5, *q_empty = bars + 6, *k_empty = bars + 7, *v_empty = bars + 8, *ep1 = bars + 9;
    uint64_t *hs_free = bars + 10, *drain = bars + 11, *kready = bars + 12;
    // per K buffer b: full and empty barriers (b = 0: k_full, k_empty; b = 1: bars 13, 14)
    auto kf = [&](int b) { return b ? bars + 13 : k_full; };
    auto ke = [&](int b) { return b ? bars + 14 : k_empty; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 16);
    uint32_t *abort_flag = tmem_slot + 1;

    const int tile = blockIdx.x, seg = blockIdx.y, bh = blockIdx.z;
    const int j0 = tile * DVT;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c_begin = seg * p.R;
    const int nck = min(p.R, p.NC - c_begin);
    WaitCtx wc{abort_flag, p.status};

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(k_full, 1);
        mbar_init(v_full, 1);
        mbar_init(s_full, 1);
        mbar_init(h_full, 1);
        mbar_init(c_upd, 1);
        mbar_init(q_empty, SM::TF ? 16 : 1);   // chunk 64: released by the compute warps at ep1
        mbar_init(k_empty, 1);
        mbar_init(bars + 13, 1);
        mbar_init(bars + 14, 1);
        mbar_init(v_empty, 1);
        mbar_init(ep1, 16);
        mbar_init(hs_free, 16);
        mbar_init(drain, 1);
        mbar_init(kready, 16);
        *abort_flag = 0u;
        fence_barrier_init();
        tma_prefetch(&tm_q);
        tma_prefetch(&tm_k);
        tma_prefetch(&tm_v);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, SM::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // The TMA producer (warp 0) loads only the inputs q, k, v, which no kernel of this call writes
    // (this kernel launches only once every earlier grid of the stream has passed its own
    // griddepcontrol.wait, so their producers have finished), and the MMA warp (warp 1) reads
    // shared memory and TMEM only: their first loads and MMAs go out while the preceding kernel
    // is still running.  The warps that read its outputs wait for them.
    if (warp >= 2) griddep_wait();
    griddep_launch_dependents();

    if (warp == 0) {
        if (lane == 0) {   // TMA producer: Q, K (all DK) and the V tile of every chunk
            int nq = 0, nv = 0, nk0 = 0, nk1 = 0;   // loads issued per buffer
            for (int i = 0; i < nck; ++i) {
                const int t0 = (c_begin + i) * L;
                const uint32_t pp = (uint32_t)(i - 1) & 1u;
                if (i > 0 && !mbar_wait(q_empty, pp, wc)) break;
                WALK_TRACE(0);
                mbar_arrive_expect_tx(q_full, DK * L * 2);
                for (int b = 0; b < DK / 64; ++b) tma_load_3d(Qs + b * L * 128, &tm_q, b * 64, t0, bh, q_full);
                ++nq;
                const int kb = i % SM::KB;
                if (i >= SM::KB && !mbar_wait(ke(kb), (uint32_t)(i / SM::KB - 1) & 1u, wc)) break;
                WALK_TRACE(1);
                mbar_arrive_expect_tx(kf(kb), DK * L * 2);
                for (int b = 0; b < DK / 64; ++b)
                    tma_load_3d(Ks + kb * SM::KBYTES + b * L * 128, &tm_k, b * 64, t0, bh, kf(kb));
                (kb ? nk1 : nk0) += 1;
                if (i > 0 && !mbar_wait(v_empty, pp, wc)) break;
                WALK_TRACE(2);
                mbar_arrive_expect_tx(v_full, DVT * L * 2);
                for (int b = 0; b < DVT / 64; ++b)
                    tma_load_3d(Vs + b * L * 128, &tm_v, j0 + b * 64, t0, bh, v_full);
                ++nv;
            }
            // drain: the last load issued into each buffer has landed
            if (nq > 0) mbar_wait_drain(q_full, (uint32_t)(nq - 1) & 1u);
            if (nk0 > 0) mbar_wait_drain(kf(0), (uint32_t)(nk0 - 1) & 1u);
            if (nk1 > 0) mbar_wait_drain(kf(1), (uint32_t)(nk1 - 1) & 1u);
            if (nv > 0) mbar_wait_drain(v_full, (uint32_t)(nv - 1) & 1u);
        }
    } else if (warp == 1) {
        if (lane == 0) {   // MMA issuer
            constexpr uint32_t ID_S = idesc_bf16(L, L, 0, 0);       // S  = Q K^T
            constexpr uint32_t ID_HC = SM::TF ? idesc_tf32(DVT, L)  // H^T = C^T Q'^T    (tf32, A in TMEM)
                                              : idesc_f16(DVT, L, 0, 0);  // H^T = Cb^T Q'^T (fp16, A in TMEM)
            constexpr uint32_t ID_HP = idesc_bf16(DVT, L, 1, 0);    // H^T += V^T P^T
            constexpr uint32_t ID_C = idesc_bf16(DVT, DK, 1, 1);    // C^T += V^T K'
            const uint32_t qa = smem_u32(Qs), ka = smem_u32(Ks), va = smem_u32(Vs), pa = smem_u32(Ps);
            const uint32_t hs = tmem + SM::HS_COL;
            if constexpr (SM::TF) {
                // chunk 64: S(i + 1) is issued right after the state update of chunk i (separate S and
                // H^T accumulators, K double-buffered), so it runs while chunk i's outputs are read
                const uint32_t sa = tmem + SM::S_COL, ha = tmem + SM::H_COL;
                const uint32_t q32 = smem_u32(smem + SM::Q32_OFF);
                auto issue_s = [&](int ci) -> bool {
                    if (!mbar_wait(q_full, (uint32_t)ci & 1u, wc)) return false;
                    WALK_TRACE_AT(3, ci);
                    if (!mbar_wait(kf(ci % SM::KB), (uint32_t)(ci / SM::KB) & 1u, wc)) return false;
                    WALK_TRACE_AT(4, ci);
                    tc_fence_after();
                    const uint32_t kab = ka + (ci % SM::KB) * SM::KBYTES;
#pragma unroll
                    for (int k = 0; k < DK / 16; ++k) {
                        const uint32_t off = (k >> 2) * L * 128 + (k & 3) * 32;
                        mma_ss(sa, smem_desc(qa + off, 16, 1024), smem_desc(kab + off, 16, 1024), ID_S,
                               k > 0 ? 1u : 0u);
                    }
                    mma_commit(s_full);
                    WALK_TRACE_AT(5, ci);
                    return true;
                };
                bool run = nck > 0 && issue_s(0);
                for (int i = 0; i < nck && run; ++i) {
                    const uint32_t ph = (uint32_t)i & 1u;
                    // the compute warps arrive on ep1 after their last reads of the previous H^T
                    if (!mbar_wait(ep1, ph, wc)) break;
                    WALK_TRACE(6);
                    if (!mbar_wait(v_full, ph, wc)) break;
                    WALK_TRACE(7);
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < DK / 8; ++k) {     // 8 tf32 = 32 bytes of a 128-byte row per step
                        const uint32_t off = (k >> 2) * L * 128 + (k & 3) * 32;
                        mma_ts_tf32(ha, tmem + SM::C_COL + k * 8, smem_desc(q32 + off, 16, 1024), ID_HC,
                                    k > 0 ? 1u : 0u);
                    }
#pragma unroll
                    for (int k = 0; k < L / 16; ++k) {
                        const uint32_t poff = (k >> 2) * L * 128 + (k & 3) * 32;
                        mma_ss(ha, smem_desc(va + k * 2048, L * 128, 1024), smem_desc(pa + poff, 16, 1024), ID_HP,
                               1u);
                    }
                    mma_commit(h_full);
                    WALK_TRACE(8);
                    const int kb = i % SM::KB;
                    if (i < nck - 1) {
                        if (!mbar_wait(kready, ph, wc)) break;
                        WALK_TRACE(9);
                        tc_fence_after();
                        const uint32_t kab = ka + kb * SM::KBYTES;
#pragma unroll
                        for (int k = 0; k < L / 16; ++k)
                            mma_ss(tmem + SM::C_COL, smem_desc(va + k * 2048, L * 128, 1024),
                                   smem_desc(kab + k * 2048, L * 128, 1024), ID_C, 1u);
                        mma_commit(c_upd);
                    }
                    mma_commit(ke(kb));
                    mma_commit(v_empty);
                    if (i < nck - 1 && !issue_s(i + 1)) break;
                }
            } else
            for (int i = 0; i < nck; ++i) {
                const uint32_t ph = (uint32_t)i & 1u;
                if (!mbar_wait(q_full, ph, wc)) break;
                WALK_TRACE(3);
                if (!mbar_wait(k_full, ph, wc)) break;
                WALK_TRACE(4);
                if (i > 0 && !mbar_wait(hs_free, ph ^ 1u, wc)) break;
                WALK_TRACE(5);
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < DK / 16; ++k) {
                    const uint32_t off = (k >> 2) * L * 128 + (k & 3) * 32;
                    mma_ss(hs, smem_desc(qa + off, 16, 1024), smem_desc(ka + off, 16, 1024), ID_S, k > 0 ? 1u : 0u);
                }
                mma_commit(s_full);
                if (!mbar_wait(ep1, ph, wc)) break;
                WALK_TRACE(6);
                if (!mbar_wait(v_full, ph, wc)) break;
                WALK_TRACE(7);
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < DK / 16; ++k) {
                    const uint32_t off = (k >> 2) * L * 128 + (k & 3) * 32;
                    mma_ts(hs, tmem + SM::CB_COL + k * 8, smem_desc(qa + off, 16, 1024), ID_HC, k > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int k = 0; k < L / 16; ++k) {
                    const uint32_t poff = (k >> 2) * L * 128 + (k & 3) * 32;
                    mma_ss(hs, smem_desc(va + k * 2048, L * 128, 1024), smem_desc(pa + poff, 16, 1024), ID_HP, 1u);
                }
                mma_commit(h_full);
                mma_commit(q_empty);
                WALK_TRACE(8);
                if (i < nck - 1) {
                    if (!mbar_wait(kready, ph, wc)) break;
                    WALK_TRACE(9);
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < L / 16; ++k)
                        mma_ss(tmem + SM::C_COL, smem_desc(va + k * 2048, L * 128, 1024),
                               smem_desc(ka + k * 2048, L * 128, 1024), ID_C, 1u);
                    mma_commit(c_upd);
                }
                mma_commit(k_empty);
                mma_commit(v_empty);
            }
            mma_commit(drain);           // every MMA of this CTA has completed
            mbar_wait_drain(drain, 0);
        }
    } else {
        // compute warps 2..17: four per TMEM lane quadrant
        const int ct = threadIdx.x - 64;          // 0..511
        const int cw = ct >> 5;                   // compute warp 0..15
        const int q = warp & 3;                   // TMEM lane quadrant
        const int hq = (warp - 2) >> 2;           // which quarter of the columns / tokens
        const float scale = rsqrtf((float)DK);
        const float *Ab = p.A + (size_t)bh * p.S;
        const float *Mb = p.Mtok + (size_t)bh * p.S;   // chunk-local prefix maxima p
        const float *igb = p.ig + (size_t)bh * p.S;
        const float *MCb = p.MC + (size_t)bh * (p.NC + 1);
        const float *Gb = p.G + (size_t)bh * p.NC;
        constexpr int CQ = DK / 4;                // state columns of a warp (a quarter of DK)
        static_assert(CQ % 16 == 0, "state quarter");

        // the segment's start state -> TMEM (C^T, lane = value column) and shared (n)
        {
            const float *src = p.DC + ((size_t)bh * p.NSEG + seg) * (size_t)DK * p.DV;
            const int j = q * 32 + lane;
            for (int c0 = hq * CQ; c0 < (hq + 1) * CQ; c0 += 16) {
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
            for (int i = ct; i < DK; i += 512) nX[i] = p.DN[((size_t)bh * p.NSEG + seg) * DK + i];
        }
        float rho = MCb[c_begin];
        bool ok = true;

        // gate values of the next chunk, loaded one chunk ahead
        float pa = 0.f, pm = 0.f, pi = 0.f;
        float pmc = MCb[c_begin], pmn = MCb[c_begin + 1], pg = Gb[c_begin];
        if (ct < L && c_begin * L + ct < p.S) {
            const int t = c_begin * L + ct;
            pa = Ab[t];
            pm = Mb[t];
            pi = igb[t];
        }
        // output epilogue mapping: a warp takes 16-token blocks of its quarter of the chunk; a lane
        // then holds token (lane >> 1) of the block and 16 of the warp's 32 value columns
        constexpr int TQ = L / 4;                 // tokens of a warp's quarter (32 or 16)
        constexpr int NBLK = TQ / 16;             // 16-token blocks per warp (2 or 1)

        for (int i = 0; i < nck && ok; ++i) {
            const int c = c_begin + i;
            const int t0 = c * L;
            const int len = min(L, p.S - t0);
            const uint32_t ph = (uint32_t)i & 1u;
            const float mc = pmc, mn = pmn, g = pg;
            const float ca = pa, cm = pm, ci = pi;
            if (i + 1 < nck) {                    // prefetch the next chunk's gate values
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
            const bool rescale = !last && (mn - (rho + g) > THRESH);
            const float rho_new = rescale ? (mn - g) : rho;
            const float alpha = expf(rho - mc);
            const float beta = expf(rho - rho_new);
            // scale of the TMEM state as the tf32 inter product reads it: the chunk's starting frame rho
            // (the frame moves only after that product, see the K pass)
            const float ahc = SM::TF ? alpha : 1.f;

            if (p.o) {   // bring this thread's output-gate rows of the epilogue into L2 early
#pragma unroll
                for (int u = 0; u < NBLK; ++u) {
                    const int tau = hq * TQ + u * 16 + (lane >> 1);
                    if (tau < len)
                        asm volatile("prefetch.global.L2 [%0];" ::"l"(p.o + ((size_t)bh * p.S + t0 + tau) * p.DV + j0 +
                                                                        q * 32 + (lane & 1) * 16));
                }
            }
            // No barrier here: the previous chunk's last reads of the per-row arrays written below (in
            // (c), (d), the K pass and the denominators) all precede the barrier before its output
            // epilogue, which reads only inv[] and the staging tile; inv[] and the P tile (the staging
            // tile at chunk 128) are next written after the barrier of (b).
            if (ct == 0) WALK_TRACE(10);
            if (ct < L) {
                if (ct < len) {
                    const float mt = ca + fmaxf(mc, cm);   // per-token stabilizer from the prefix maximum p
                    arow[ct] = (ca - mt) * LOG2E;
                    mrow[ct] = mt;
                    icol[ct] = (ci - ca) * LOG2E;
                    const float sc = expf(ca + mc - mt) * scale;
                    srow[ct] = sc;
                    const float sct = sc * ahc;                 // row scale of the inter product
                    int ex = 0;
                    const float fr = frexpf(sct, &ex);           // sct = fr 2^ex, fr in [0.5, 1)
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
                // column factors for the blocks of S below the diagonal: 2^(icol - bcol) with bcol
                // the maximum of icol over the block's L/4 columns (so the factor is at most 1)
                constexpr int BW = L / 4;
                const float ic = ct < len ? (ci - ca) * LOG2E : -INFINITY;
                float bm = ic;
#pragma unroll
                for (int o = BW / 2; o > 0; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
                ccol[ct] = bm == -INFINITY ? 0.f : exp2f(ic - bm);
                if ((ct & (BW - 1)) == 0) bcol[ct / BW] = bm;
            }

            // (b) Cb = fp16(C_c 2^-kc) into TMEM, kc from max |C_c| over the tile; rescale the
            //     fp32 state when the frame moves (at chunk 64 the state is read in place, and the
            //     frame moves in the K pass)
            if (ct == 0) WALK_TRACE(11);
            // the previous chunk's state update must be complete before the state is read or
            // rescaled here; at chunk 64 nothing here touches it (the inter-chunk MMA is ordered
            // after the update in the MMA pipe, and Q', P are free since h_full)
            if (i > 0 && !SM::TF && !mbar_wait(c_upd, ph ^ 1u, wc)) { ok = false; break; }
            if (ct == 0) WALK_TRACE(12);
            tc_fence_after();
            int kc = 0;
            if constexpr (SM::TF) {
                named_sync(1, 512);                   // the per-row arrays are complete
            } else {
            float cmax = 0.f;
#pragma unroll
            for (int uc = 0; uc < CQ / 16; ++uc) {
                const int c0 = hq * CQ + uc * 16;
                uint32_t r[16];
                tmem_ld16(tmem_addr(tmem, q * 32, SM::C_COL + c0), r);
                tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 16; ++u) cmax = fmaxf(cmax, fabsf(__uint_as_float(r[u])));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, o));
            if (lane == 0) red[cw] = cmax;
            named_sync(1, 512);                   // red[] and the per-row arrays are complete
            cmax = red[0];
#pragma unroll
            for (int w16 = 1; w16 < 16; ++w16) cmax = fmaxf(cmax, red[w16]);
            cmax *= alpha;
            if (cmax > 0.f) {
                int ex = 0;
                frexpf(cmax, &ex);                       // cmax < 2^ex
                kc = min(max(ex - 8, -120), 14);         // |Cb| < 2^8
            }
            const float cbs = ldexpf(alpha, -kc);
#pragma unroll
            for (int uc = 0; uc < CQ / 16; ++uc) {
                const int c0 = hq * CQ + uc * 16;
                uint32_t r[16];
                tmem_ld16(tmem_addr(tmem, q * 32, SM::C_COL + c0), r);
                tmem_wait_ld();
                uint32_t pk[8];
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    pk[u] = pack_f16(__uint_as_float(r[2 * u]) * cbs, __uint_as_float(r[2 * u + 1]) * cbs);
                tmem_st8(tmem_addr(tmem, q * 32, SM::CB_COL + c0 / 2), pk);
                if (rescale) {
#pragma unroll
                    for (int u = 0; u < 16; ++u) r[u] = __float_as_uint(__uint_as_float(r[u]) * beta);
                    tmem_st16(tmem_addr(tmem, q * 32, SM::C_COL + c0), r);
                }
            }
            tmem_wait_st();
            }

            // (c) S -> P (bf16, shared, K-major swizzled), partial row sums over a quarter of the columns
            if (ct == 0) WALK_TRACE(13);
            if (!mbar_wait(s_full, ph, wc)) { ok = false; break; }
            if (ct == 0) WALK_TRACE(14);
            tc_fence_after();
            if (L == 128) {
                const int tau = q * 32 + lane;
                const int s0 = hq * 32;
                float sum = 0.f;
                uint32_t pk[16];
                if (s0 > q * 32) {                 // whole 32 x 32 block above the diagonal: zeros
#pragma unroll
                    for (int e = 0; e < 16; ++e) pk[e] = 0u;
                } else {
                    uint32_t r[32];
                    tmem_ld32(tmem_addr(tmem, q * 32, SM::S_COL + s0), r);
                    tmem_wait_ld();
                    const float at = arow[tau];
                    const float ri = 1.f / rrow[tau];
                    if (s0 == q * 32) {            // diagonal block: the decay per element, causal mask
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            float v2[2];
#pragma unroll
                            for (int z = 0; z < 2; ++z) {
                                const int sg = s0 + 2 * e + z;
                                float d = exp2f(at + icol[sg]);
                                if (sg > tau) d = 0.f;
                                v2[z] = __uint_as_float(r[2 * e + z]) * d * scale;
                                sum += v2[z];
                            }
                            pk[e] = pack_bf16(v2[0] * ri, v2[1] * ri);
                        }
                    } else {                       // below the diagonal: row factor x column factor
                        const float rf = tau < len ? exp2f(at + bcol[hq]) * scale : 0.f;
                        const uint64_t rf2 = f2_pack(rf, rf), ri2 = f2_pack(ri, ri);
                        const uint64_t *cc2 = reinterpret_cast<const uint64_t *>(ccol + s0);
                        uint64_t sum2 = 0ull;
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const uint64_t v = f2_mul(f2_pack(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1])),
                                                      f2_mul(cc2[e], rf2));
                            sum2 = f2_add(sum2, v);
                            pk[e] = f2_to_bf16x2(f2_mul(v, ri2));
                        }
                        const float2 sd = f2_unpack(sum2);
                        sum = sd.x + sd.y;
                    }
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int jcs = (s0 >> 3) + e;          // 16-byte chunk index within the row
                    *reinterpret_cast<uint4 *>(Ps + sw128_chunk(tau, jcs, L)) =
                        make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
                }
                rs[hq * L + tau] = sum;
            } else {   // L == 64: M = 64 accumulator, rows 16q..16q+15 in lanes 0..15 of quadrant q.
                // The four warps of a quadrant share all of its blocks by columns: warp hq takes
                // columns 4 hq .. 4 hq + 3 of every 16-column block, so that the diagonal block's
                // per-element decay is spread over the four warps instead of falling on one
                const int tau = q * 16 + (lane & 15);
                const float at = arow[tau];
                const float ri = 1.f / rrow[tau];
                float sum = 0.f;
#pragma unroll
                for (int blk = 0; blk < 4; ++blk) {
                    const int s0 = blk * 16 + hq * 4;          // this warp's first column of the block
                    const bool above = blk > q;                // the whole block is masked
                    uint32_t r[4];
                    if (!above) {
                        tmem_ld4(tmem_addr(tmem, q * 32, SM::S_COL + s0), r);
                        tmem_wait_ld();
                    }
                    if (lane < 16) {
                        float v[4];
                        if (above) {
#pragma unroll
                            for (int z = 0; z < 4; ++z) v[z] = 0.f;
                        } else if (blk < q) {                  // row factor x column factor
                            const float rf = tau < len ? exp2f(at + bcol[blk]) * scale : 0.f;
#pragma unroll
                            for (int z = 0; z < 4; ++z) v[z] = __uint_as_float(r[z]) * (ccol[s0 + z] * rf);
                        } else {                               // diagonal block: per element, causal mask
#pragma unroll
                            for (int z = 0; z < 4; ++z) {
                                const int sg = s0 + z;
                                float d = exp2f(at + icol[sg]);
                                if (sg > tau) d = 0.f;
                                v[z] = __uint_as_float(r[z]) * d * scale;
                            }
                        }
                        sum += (v[0] + v[1]) + (v[2] + v[3]);
                        // 4 bf16 = the first or second half of the row's 16-byte chunk s0 / 8
                        *reinterpret_cast<uint2 *>(Ps + sw128_chunk(tau, s0 >> 3, L) + ((s0 >> 2) & 1) * 8) =
                            make_uint2(pack_bf16(v[0] * ri, v[1] * ri), pack_bf16(v[2] * ri, v[3] * ri));
                    }
                }
                if (lane < 16) rs[hq * L + tau] = sum;
            }

            if (ct == 0) WALK_TRACE(15);
            // (d) Q pass, a thread per (row, range of CPT 16-byte chunks): the partial inter-chunk
            //     denominator q . nX from the unscaled bf16 q (fp32), then Q' = 2^(e + kc) q in fp16
            //     (exact), in place as the MMA operand
            {
                constexpr int CPT = DK * L / 4096;       // chunks per thread
                constexpr int PARTS = 512 / L;           // threads per row
                static_assert(CPT >= 1 && CPT <= 8 && PARTS * CPT * 8 == DK, "Q pass mapping");
                const int row = ct % L, part = ct / L;
                const int jc0 = part * CPT;
                const int qe = (int)qexp[row] + kc;
                const float s2 = qe >= -126 ? __int_as_float((qe + 127) << 23) : 0.f;
                const uint64_t ss = f2_pack(s2, s2);
                uint64_t dot2 = 0ull;                    // packed pair of partial dot products
#pragma unroll
                for (int u = 0; u < CPT; ++u) {
                    const uint32_t off = sw128_chunk(row, jc0 + u, L);
                    const uint4 uq = *reinterpret_cast<const uint4 *>(Qs + off);
                    const ulonglong2 na = *reinterpret_cast<const ulonglong2 *>(nX + (jc0 + u) * 8);
                    const ulonglong2 nb = *reinterpret_cast<const ulonglong2 *>(nX + (jc0 + u) * 8 + 4);
                    const uint64_t q0 = f2_from_bf16x2(uq.x), q1 = f2_from_bf16x2(uq.y), q2 = f2_from_bf16x2(uq.z),
                                   q3 = f2_from_bf16x2(uq.w);
                    dot2 = f2_fma(q0, na.x, dot2);
                    dot2 = f2_fma(q1, na.y, dot2);
                    dot2 = f2_fma(q2, nb.x, dot2);
                    dot2 = f2_fma(q3, nb.y, dot2);
                    if constexpr (SM::TF) {   // fp32 Q': the chunk's 8 values are two 16-byte chunks of the tile
                        const int j32 = ((jc0 + u) >> 2) * 8 + ((jc0 + u) & 3) * 2;
                        uint8_t *q32 = smem + SM::Q32_OFF;
                        *reinterpret_cast<ulonglong2 *>(q32 + sw128_chunk(row, j32, L)) =
                            make_ulonglong2(f2_mul(q0, ss), f2_mul(q1, ss));
                        *reinterpret_cast<ulonglong2 *>(q32 + sw128_chunk(row, j32 + 1, L)) =
                            make_ulonglong2(f2_mul(q2, ss), f2_mul(q3, ss));
                    } else {
                        const float2 a0 = f2_unpack(f2_mul(q0, ss)), a1 = f2_unpack(f2_mul(q1, ss)),
                                     a2 = f2_unpack(f2_mul(q2, ss)), a3 = f2_unpack(f2_mul(q3, ss));
                        *reinterpret_cast<uint4 *>(Qs + off) = make_uint4(pack_f16(a0.x, a0.y), pack_f16(a1.x, a1.y),
                                                                          pack_f16(a2.x, a2.y), pack_f16(a3.x, a3.y));
                    }
                }
                const float2 dd = f2_unpack(dot2);
                dpart[part * L + row] = dd.x + dd.y;
            }
            fence_proxy_async();
            tc_fence_before();
            named_sync(1, 512);
            if (lane == 0) {
                mbar_arrive(ep1);                    // P, Q' and Cb are ready: the output MMA can start
                if constexpr (SM::TF) mbar_arrive(q_empty);   // the bf16 Q tile has been read
            }
            if (ct == 0) WALK_TRACE(16);

            // (e) while the output MMA runs: K pass, n sums W k from the unscaled bf16 k (fp32) and
            //     K' = W k in bf16 in place, the operand of the state update.  A warp owns CPW 16-byte
            //     chunks of every row (lane = row), so that its n sums reduce inside the warp and go
            //     straight into nX
            // The frame move of the tf32 path, per warp on its part of the state before its K' arrival:
            // the output MMA reads the state in the chunk's starting frame, so the state is rescaled
            // only once that MMA has completed, and before the update adds the chunk's tokens in the new
            // frame.  (One fp32 frame cannot serve both ends of a chunk whose log decay is in the
            // hundreds: exp(rho_new - m_c) overflows while exp(rho - rho_new) underflows.)
            auto move_frame = [&]() {
                if constexpr (SM::TF) {
                    uint32_t done = 1u;
                    if (lane == 0) done = mbar_wait(h_full, ph, wc) ? 1u : 0u;
                    if (!__shfl_sync(0xffffffffu, done, 0)) return;   // aborted: (g) leaves the loop
                    tc_fence_after();
#pragma unroll 1
                    for (int uc = 0; uc < CQ / 16; ++uc) {
                        const int c0 = hq * CQ + uc * 16;
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
            };
            if (!last) {
                constexpr int NCH = DK / 8;                   // chunks per row
                constexpr int CPW = NCH >= 16 ? NCH / 16 : 1; // chunks per warp
                constexpr int NV = 8 * CPW;                   // n sums per lane before the reduction
                static_assert(NV == 8 || NV == 16, "K pass mapping");
                uint8_t *Kc = Ks + (i % SM::KB) * SM::KBYTES;  // this chunk's K tile
                if (cw < NCH) {                               // DK = 64: warps 8..15 have no chunk
                    uint64_t nacc2[NV / 2];                   // packed pairs of n sums
#pragma unroll
                    for (int z = 0; z < NV / 2; ++z) nacc2[z] = 0ull;
#pragma unroll
                    for (int rg = 0; rg < L / 32; ++rg) {
                        const int row = rg * 32 + lane;
                        const float w = wcol[row];
                        const uint64_t ww = f2_pack(w, w);
                        uint4 uk[CPW];
#pragma unroll
                        for (int cc = 0; cc < CPW; ++cc)
                            uk[cc] = *reinterpret_cast<const uint4 *>(Kc + sw128_chunk(row, cw * CPW + cc, L));
#pragma unroll
                        for (int cc = 0; cc < CPW; ++cc) {
                            const uint64_t k0 = f2_from_bf16x2(uk[cc].x), k1 = f2_from_bf16x2(uk[cc].y),
                                           k2 = f2_from_bf16x2(uk[cc].z), k3 = f2_from_bf16x2(uk[cc].w);
                            uint64_t *na = nacc2 + cc * 4;
                            na[0] = f2_fma(ww, k0, na[0]);
                            na[1] = f2_fma(ww, k1, na[1]);
                            na[2] = f2_fma(ww, k2, na[2]);
                            na[3] = f2_fma(ww, k3, na[3]);
                            *reinterpret_cast<uint4 *>(Kc + sw128_chunk(row, cw * CPW + cc, L)) =
                                make_uint4(f2_to_bf16x2(f2_mul(k0, ww)), f2_to_bf16x2(f2_mul(k1, ww)),
                                           f2_to_bf16x2(f2_mul(k2, ww)), f2_to_bf16x2(f2_mul(k3, ww)));
                        }
                    }
                    float nacc[NV];
#pragma unroll
                    for (int z = 0; z < NV / 2; ++z) {
                        const float2 v = f2_unpack(nacc2[z]);
                        nacc[2 * z] = v.x;
                        nacc[2 * z + 1] = v.y;
                    }
                    fence_proxy_async();
                    __syncwarp();
                    if (beta < 1.f) move_frame();            // (beta < exp(-THRESH) exactly when the frame moves)
                    if (lane == 0) mbar_arrive(kready);      // K' is ready: the state update can start
                    // transposed reduction over the 32 lanes: each exchange halves the values a lane
                    // holds, so that lane l ends with the sum of value l / (32 / NV)
                    int nv = NV;
#pragma unroll
                    for (int o = 16; o >= 1; o >>= 1) {
                        if (nv > 1) {
                            const bool up = (lane & o) != 0;
                            const int h = nv / 2;
#pragma unroll
                            for (int z = 0; z < NV / 2; ++z) {
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
                    if ((lane & (32 / NV - 1)) == 0) {
                        const int d = cw * NV + lane / (32 / NV);
                        nX[d] = nX[d] * beta + nacc[0];
                    }
                } else {
                    __syncwarp();
                    if (beta < 1.f) move_frame();
                    if (lane == 0) mbar_arrive(kready);
                }
            }
            // output gate of this thread's epilogue rows, loaded after the K pass so that the loads overlap the
            // normalizer update and the wait for the output MMA
            // (rows past the end of the sequence read the last row; their outputs are not stored)
            uint4 ou[NBLK][2];
            if (p.o) {
                const int er = lane >> 1, jh = lane & 1;
#pragma unroll
                for (int u = 0; u < NBLK; ++u) {
                    const int tau = min(hq * TQ + u * 16 + er, len - 1);
                    const size_t off = ((size_t)bh * p.S + t0 + tau) * p.DV + j0 + q * 32 + jh * 16;
#pragma unroll
                    for (int c8 = 0; c8 < 2; ++c8) ou[u][c8] = *reinterpret_cast<const uint4 *>(p.o + off + c8 * 8);
                }
            } else {
#pragma unroll
                for (int u = 0; u < NBLK; ++u)
#pragma unroll
                    for (int c8 = 0; c8 < 2; ++c8)   // bf16 1.0 = 0x3F80 when there is no output gate
                        ou[u][c8] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
            }

            // 1 / denominator (times r) of this chunk (rs, dpart and the row arrays are complete since ep1)
            if (ct < L) {
                float qn = 0.f;
#pragma unroll
                for (int pp = 0; pp < 512 / L; ++pp) qn += dpart[pp * L + ct];
                const float den = rs[ct] + rs[L + ct] + rs[2 * L + ct] + rs[3 * L + ct] + qn * alpha * srow[ct];
                inv[ct] = rrow[ct] / fmaxf(fabsf(den), expf(-mrow[ct]));
            }
            named_sync(1, 512);
            if (ct == 0) WALK_TRACE(17);

            // (g) outputs: H^T (lane = value column j, columns = tokens)
            if (!mbar_wait(h_full, ph, wc)) { ok = false; break; }
            if (ct == 0) WALK_TRACE(18);
            tc_fence_after();
            {
                // each warp owns value columns [32q, 32q + 32) and the tokens of its quarter; per block of
                // 16 tokens the 16 x 32 tile goes through shared memory (2 KB per warp, granules of four
                // floats XOR-swizzled by the row) so that a lane then holds 16 columns of one token and
                // reads o / writes h with 16-byte vectors
                float *tile = reinterpret_cast<float *>(Ts) + cw * 512;
                __nv_bfloat16 *__restrict__ hp = p.h;
                const int er = lane >> 1, jh = lane & 1;   // token row of the block, column half
#pragma unroll
                for (int u = 0; u < NBLK; ++u) {
                    const int tb = hq * TQ + u * 16;
                    if (ct == 0 && u == 1) WALK_TRACE(20);
                    uint32_t r[16];
                    tmem_ld16(tmem_addr(tmem, q * 32, SM::H_COL + tb), r);
                    tmem_wait_ld();
                    // lane = value column j: element (token e, column lane), 16 tokens
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        tile[e * 32 + ((((lane >> 2) ^ (e & 7)) << 2) | (lane & 3))] = __uint_as_float(r[e]);
                    __syncwarp();
                    // lane -> token er of the block, columns [16 jh, 16 jh + 16)
                    float hv[16];
#pragma unroll
                    for (int gq = 0; gq < 4; ++gq) {
                        const float4 v4 =
                            *reinterpret_cast<const float4 *>(tile + er * 32 + (((jh * 4 + gq) ^ (er & 7)) << 2));
                        hv[4 * gq] = v4.x; hv[4 * gq + 1] = v4.y; hv[4 * gq + 2] = v4.z; hv[4 * gq + 3] = v4.w;
                    }
                    __syncwarp();
                    const int tau = tb + er;
                    if (tau < len) {
                        const size_t off = ((size_t)bh * p.S + t0 + tau) * p.DV + j0 + q * 32 + jh * 16;
                        const float iv = inv[tau];
                        const uint64_t iv2 = f2_pack(iv, iv);
#pragma unroll
                        for (int c8 = 0; c8 < 2; ++c8) {
                            // o h / den in packed pairs (bf16 1.0 = 0x3F80 when there is no output gate)
                            const float *hh = hv + c8 * 8;
                            uint32_t w4[4];
                            const uint32_t og4[4] = {ou[u][c8].x, ou[u][c8].y, ou[u][c8].z, ou[u][c8].w};
#pragma unroll
                            for (int z = 0; z < 4; ++z)
                                w4[z] = f2_to_bf16x2(f2_mul(f2_from_bf16x2(og4[z]),
                                                            f2_mul(f2_pack(hh[2 * z], hh[2 * z + 1]), iv2)));
                            *reinterpret_cast<uint4 *>(hp + off + c8 * 8) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (!SM::TF && lane == 0) mbar_arrive(hs_free);
            if (ct == 0) WALK_TRACE(19);
            rho = rho_new + g;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, SM::TMEM_COLS);
    }
}

// ---------------------------------------------------------------- host side

// The driver's tensor-map encoder, looked up once (a failed lookup is retried on the next call).
PFN_cuTensorMapEncodeTiled_v12000 get_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::lock_guard<std::mutex> guard(host_cache_mutex());
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *ptr = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// [BH][S][D] bf16 tensor, boxes of 64 columns x rows tokens x 1 head, 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *base, int D, int S, int BH, int rows)
{
    auto enc = get_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)S, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)S * D * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int DK, int L>
cudaError_t launch_dk_l(const FwdArgs &a, const FwdWorkspace &w, const PhaseMark &mark)
{
    Params p;
    p.S = a.S; p.L = L; p.NC = w.NC; p.R = w.R; p.NSEG = w.NSEG; p.DK = DK; p.DV = a.DHV; p.BH = a.BH;
    p.A = w.A; p.Mtok = w.M; p.ig = a.igate; p.MC = w.MC; p.G = w.G; p.GP = w.GP; p.SGb = w.SGb;
    p.DC = w.DC; p.DN = w.DN;
    p.o = static_cast<const __nv_bfloat16 *>(a.ogate);
    p.h = static_cast<__nv_bfloat16 *>(a.h);
    p.status = w.status;

    CUtensorMap mq, mk, mv, mk64, mv64;
    if (!make_map(&mq, a.outputs ? a.q : a.k, DK, a.S, a.BH, L) || !make_map(&mk, a.k, DK, a.S, a.BH, L) ||
        !make_map(&mv, a.v, a.DHV, a.S, a.BH, L) || !make_map(&mk64, a.k, DK, a.S, a.BH, TB) ||
        !make_map(&mv64, a.v, a.DHV, a.S, a.BH, TB))
        return cudaErrorInvalidValue;
    const int ntile = a.DHV / DVT;
    cudaError_t e;

    // two value tiles per segment-sum CTA when that costs fewer whole waves of 148 SMs
    const long long ctas1 = (long long)ntile * w.NSEG * a.BH;
    const bool two = ntile % 2 == 0 && 1.4 * ((ctas1 / 2 + 147) / 148) < (double)((ctas1 + 147) / 148);
    if (two) {
        if ((e = ensure_dynamic_smem((const void *)segsum_kernel<DK, 2>, SegSmem<DK, 2>::TOTAL)) != cudaSuccess) return e;
        e = launch_kernel(segsum_kernel<DK, 2>, dim3(ntile / 2, w.NSEG, a.BH), dim3(SS_THREADS), SegSmem<DK, 2>::TOTAL,
                          a.stream, 1, mk64, mv64, p);
    } else {
        if ((e = ensure_dynamic_smem((const void *)segsum_kernel<DK, 1>, SegSmem<DK, 1>::TOTAL)) != cudaSuccess) return e;
        e = launch_kernel(segsum_kernel<DK, 1>, dim3(ntile, w.NSEG, a.BH), dim3(SS_THREADS), SegSmem<DK, 1>::TOTAL,
                          a.stream, 1, mk64, mv64, p);
    }
    if (e != cudaSuccess) return e;
    if ((e = mark(2)) != cudaSuccess) return e;

    const int nquad = DK * a.DHV / 4;
    e = launch_kernel(seg_scan_kernel, dim3((nquad + 255) / 256, a.BH), dim3(256), 0, a.stream, 1, p, a.C_final,
                      a.n_final, a.m_final, a.C0, a.n0);
    if (e != cudaSuccess) return e;
    if ((e = mark(3)) != cudaSuccess) return e;

    if (!a.outputs) return cudaSuccess;   // the final state is complete after the segment scan
    if (walk_pair_supported(DK, a.DHV, L)) return launch_walk_pair(p, a.q, a.k, a.v, a.stream);
    using WS = WalkSmem<DK, L>;
    if ((e = ensure_dynamic_smem((const void *)walk_kernel<DK, L>, WS::TOTAL)) != cudaSuccess) return e;
    return launch_kernel(walk_kernel<DK, L>, dim3(ntile, w.NSEG, a.BH), dim3(WALK_THREADS), WS::TOTAL, a.stream, 1,
                         mq, mk, mv, p);
}

}  // namespace tcfwd

#ifdef MLSTM_WALK_TRACE
extern "C" int mlstm_walk_trace_copy(void *dst, size_t bytes)
{
    return (int)cudaMemcpyFromSymbol(dst, tcfwd::g_walk_trace, bytes);
}
extern "C" int mlstm_seg_trace_copy(void *dst, size_t bytes)
{
    return (int)cudaMemcpyFromSymbol(dst, tcfwd::g_seg_trace, bytes);
}
#endif

bool tc_path_supported(bool bf16, int DHQK, int DHV, int chunk)
{
    return bf16 && (DHQK == 64 || DHQK == 128 || DHQK == 256) && DHV % tcfwd::DVT == 0 &&
           (chunk == 64 || chunk == 128);
}

// Segments per head: balances whole waves of one CTA per SM (148 SMs) against
// the number of chunks each CTA walks.
int tc_num_segments(int BH, int DHV, int NC)
{
    const int ntile = DHV / tcfwd::DVT;
    const long long ctas_per_seg = (long long)BH * ntile;
    long long best_cost = -1;
    int best = 1;
    for (int nseg = 1; nseg <= NC && nseg <= tcfwd::SCAN_MAX_SEG; ++nseg) {
        const int R = (NC + nseg - 1) / nseg;
        const int ns = (NC + R - 1) / R;
        if (ns != nseg) continue;
        const long long rounds = (ctas_per_seg * ns + 147) / 148;
        const long long cost = rounds * (R + 1) * 100 + ns;     // +1: a chunk's worth of start-up per CTA
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = ns;
        }
    }
    return best;
}

cudaError_t launch_fwd_tc(const FwdArgs &a, const FwdWorkspace &w, const PhaseMark &mark)
{
    using namespace tcfwd;
    if (a.DHQK == 256 && a.chunk == 128) return launch_dk_l<256, 128>(a, w, mark);
    if (a.DHQK == 256 && a.chunk == 64) return launch_dk_l<256, 64>(a, w, mark);
    if (a.DHQK == 128 && a.chunk == 128) return launch_dk_l<128, 128>(a, w, mark);
    if (a.DHQK == 128 && a.chunk == 64) return launch_dk_l<128, 64>(a, w, mark);
    if (a.DHQK == 64 && a.chunk == 128) return launch_dk_l<64, 128>(a, w, mark);
    if (a.DHQK == 64 && a.chunk == 64) return launch_dk_l<64, 64>(a, w, mark);
    return cudaErrorInvalidValue;
}

}  // namespace mlstm
