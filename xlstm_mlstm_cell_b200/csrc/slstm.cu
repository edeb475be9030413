// slstm.cu -- the sLSTM recurrence: one persistent kernel over all S steps.
//
// The recurrence ("xLSTM Guide: Extended LSTM Architecture & Matrix Memory", "The Twin
// Cells: sLSTM and mLSTM Mathematical Formulations", part 1) is sequential in t: step t
// needs every h_{t-1} of the head, through the recurrent matrices R.  Its work per step
// is a matrix-vector product per (batch item, head, gate) of DH x DH, so the kernel is
// bound by the latency of one step, not by HBM (wx is read once, h written once).
//
// Layout of the work: the DH cells of one head are spread over a thread-block cluster of
// G = DH / 32 CTAs, 32 cells per CTA; a cluster carries BG batch items of one head through
// all S steps.  A CTA has 256 threads, 8 lanes per cell; a lane holds the cell's four gate
// rows of R over one eighth of k in registers for the whole sequence (DH / 2 floats; k in
// 16-byte pieces interleaved over the 8 lanes, so that the lanes of a cell read 128
// consecutive bytes of h and each value of h read feeds four rows).  Per step:
//   1. each lane forms its partial sums of the four gate pre-activations from h_{t-1}
//      (shared memory, fp32) for the BG batch items; lanes 0..3 add wx of gate i, f, z, o;
//   2. a butterfly over the cell's 8 lanes leaves the four sums in every lane, and all of
//      them update the cell's (c, n, m) in registers;
//   3. the lanes of a cell send h_t into the shared memory of every cluster rank with st.async
//      stores that count their bytes on that rank's mbarrier for the buffer;
//   4. the next step waits on its own mbarrier until the whole head's h_t has arrived (no
//      cluster-wide barrier and no release fence per step).
// h_{t-1} and h_t live in two shared buffers that alternate between steps.  A CTA sends into a
// peer's buffer for step t + 1 only after it has received h_t from every CTA, that is after every
// CTA has finished its step-t reads of that buffer.
#include "common.cuh"
#include "mlstm.h"
#include "slstm.h"
#include "tc_common.cuh"

namespace mlstm {
namespace slstm {

constexpr int THREADS = 256;
constexpr int CELLS = 32;   // cells of a head per CTA
constexpr int MAX_BG = 8;

MLSTM_DEVINL uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

MLSTM_DEVINL void cluster_sync_release_acquire()
{
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

MLSTM_DEVINL uint32_t map_rank(const void *local, uint32_t rank)
{
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"((uint32_t)__cvta_generic_to_shared(local)),
                 "r"(rank));
    return ra;
}

// Stores v at the offset of `local` in the CTA of cluster rank `rank` and counts its 4 bytes on
// that CTA's mbarrier at the offset of `bar` (asynchronous; no fence on this side).
MLSTM_DEVINL void st_async_cluster(const float *local, const uint64_t *bar, uint32_t rank, float v)
{
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(
                     map_rank(local, rank)),
                 "r"(__float_as_uint(v)), "r"(map_rank(bar, rank))
                 : "memory");
}

// Bounded wait for the phase of parity `parity` of a local mbarrier whose bytes come from other
// CTAs of the cluster (acquire at cluster scope).  False once the limit has passed.
MLSTM_DEVINL bool wait_cluster_fill(uint64_t *bar, uint32_t parity)
{
    const uint32_t a = (uint32_t)__cvta_generic_to_shared(bar);
    unsigned long long t0 = 0ull;
    for (uint32_t it = 0;; ++it) {
        uint32_t done;
        asm volatile("{\n\t.reg .pred p;\n\t"
                     "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}"
                     : "=r"(done)
                     : "r"(a), "r"(parity)
                     : "memory");
        if (done) return true;
        if ((it & 15u) == 0u) {
            const unsigned long long now = tc::global_timer();
            if (t0 == 0ull)
                t0 = now;
            else if (now - t0 > tc::WAIT_LIMIT_NS)
                return false;
        }
    }
}

MLSTM_DEVINL float sigmoidf_(float x) { return 1.f / (1.f + expf(-x)); }

// Packed pairs of fp32 (low half = first element): one instruction for two fused multiply-adds.
MLSTM_DEVINL uint64_t pack2(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
MLSTM_DEVINL float sum2(uint64_t r)
{
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r));
    return lo + hi;
}
MLSTM_DEVINL uint64_t fma2(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

template <typename T, int DH, int BG>
__global__ void __launch_bounds__(THREADS, 1)
slstm_kernel(const T *__restrict__ wx, const T *__restrict__ R, int B, int S, int NH, int forget_sigmoid,
             float *__restrict__ c_st, float *__restrict__ n_st, float *__restrict__ m_st, float *__restrict__ h_st,
             T *__restrict__ h_out, uint32_t *__restrict__ status)
{
    constexpr int G = DH / CELLS;        // CTAs per head (cluster size)
    constexpr int NQ = DH / 32;          // 4-value groups of k per lane
    __shared__ __align__(16) float hs[2][BG][DH];
    __shared__ __align__(8) uint64_t fill[2];      // hs[p] holds the whole head's h of a step
    __shared__ uint32_t stuck;                     // a wait gave up: later waits are skipped
    constexpr uint32_t FILL_BYTES = (uint32_t)(BG * DH * 4);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cl = lane >> 3, l8 = lane & 7;                 // cell of the warp, eighth of k
    const uint32_t rank = G > 1 ? cluster_rank() : 0u;
    const int cid = blockIdx.x / G;
    const int head = cid % NH, grp = cid / NH;
    const int b0 = grp * BG;
    const int j = (int)rank * CELLS + warp * 4 + cl;        // this lane's cell in the head
    const size_t HD = (size_t)NH * DH;                      // stride of one gate in wx

    if (tid == 0) {
        stuck = 0u;
        if constexpr (G > 1) {
            tc::mbar_init(&fill[0], 1);
            tc::mbar_init(&fill[1], 1);
            tc::fence_barrier_init();
            tc::mbar_arrive_expect_tx(&fill[0], FILL_BYTES);   // the first fill of each buffer
            tc::mbar_arrive_expect_tx(&fill[1], FILL_BYTES);
        }
    }
    griddep_wait();

    // the four gate rows of cell j over this lane's k: k = 32 q + 4 l8 + e (the 8 lanes of a
    // cell read 8 consecutive 16-byte pieces of h, so one load instruction covers 128 bytes)
    // (as packed pairs (k, k + 1), the operands of the paired multiply-adds)
    uint64_t wr[4][NQ * 2];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        const T *row = R + (((size_t)head * 4 + g) * DH + j) * DH + 4 * l8;
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
            const float4 v = load4(row + 32 * q);
            wr[g][2 * q] = pack2(v.x, v.y);
            wr[g][2 * q + 1] = pack2(v.z, v.w);
        }
    }
    // lane l8 of a cell keeps the state of batch item it = l8 mod BG (the 8 / BG lanes with the
    // same item are copies; copy ci = l8 / BG)
    constexpr int DUP = 8 / BG;
    const int it = l8 % BG, ci = l8 / BG;
    const bool item_ok = b0 + it < B;
    float c = 0.f, n = 0.f, m = 0.f;
    if (item_ok) {
        const size_t s = ((size_t)(b0 + it) * NH + head) * DH + j;
        c = c_st[s];
        n = n_st[s];
        m = m_st[s];
    }
    // h_0 of the whole head for every batch item
    for (int e = tid; e < BG * DH; e += THREADS) {
        const int b = e / DH, k = e % DH;
        hs[0][b][k] = (b0 + b < B) ? h_st[((size_t)(b0 + b) * NH + head) * DH + k] : 0.f;
        hs[1][b][k] = 0.f;          // the rows of batch items past B stay zero
    }
    // wx of gate l8 (lanes 0..3 of the cell) enters that lane's partial sum before the
    // reduction; step 0's value now, each next one a step ahead
    const bool has_x = l8 < 4;
    const T *wxr = wx + (size_t)(l8 & 3) * HD + (size_t)head * DH + j;     // + (b S + t) 4 HD
    float xw[BG];
#pragma unroll
    for (int b = 0; b < BG; ++b)
        xw[b] = (has_x && b0 + b < B) ? to_f32(wxr[((size_t)(b0 + b) * S) * 4 * HD]) : 0.f;
    __syncthreads();
    if (G > 1) cluster_sync_release_acquire();     // every CTA of the cluster has started

    const bool exp_forget = forget_sigmoid == 0;
    float hv = 0.f;
    float xsel[4];                      // 1 for the gate whose wx this lane adds, else 0 (no branch)
#pragma unroll
    for (int g = 0; g < 4; ++g) xsel[g] = (g == l8) ? 1.f : 0.f;
    for (int t = 0; t < S; ++t) {
        const int cur = t & 1;
        if constexpr (G > 1) {
            // h_{t-1} of the whole head: fill (t - 1) / 2 of buffer cur, written by every CTA of
            // the cluster during step t - 1
            if (t > 0) {
                if (!*(volatile uint32_t *)&stuck && !wait_cluster_fill(&fill[cur], (uint32_t)((t - 1) >> 1) & 1u)) {
                    stuck = 1u;
                    if (status != nullptr) atomicExch(status, (uint32_t)MLSTM_ERR_TIMEOUT);
                }
                if (tid == 0) tc::mbar_arrive_expect_tx(&fill[cur], FILL_BYTES);   // its next fill
            }
        }
        // 1. partial gate pre-activations over this lane's k (wx added by lanes 0..3 afterwards,
        //    so that its load, issued during the previous step's barrier, has the products' time)
        float acc[BG][4];
        {
            uint64_t acc2[BG][4];            // even and odd k summed apart, added at the end
#pragma unroll
            for (int b = 0; b < BG; ++b)
#pragma unroll
                for (int g = 0; g < 4; ++g) acc2[b][g] = 0ull;
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
#pragma unroll
                for (int b = 0; b < BG; ++b) {
                    const ulonglong2 h4 = *reinterpret_cast<const ulonglong2 *>(&hs[cur][b][32 * q + 4 * l8]);
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        acc2[b][g] = fma2(wr[g][2 * q], h4.x, acc2[b][g]);
                        acc2[b][g] = fma2(wr[g][2 * q + 1], h4.y, acc2[b][g]);
                    }
                }
            }
#pragma unroll
            for (int b = 0; b < BG; ++b)
#pragma unroll
                for (int g = 0; g < 4; ++g) acc[b][g] = fmaf(xsel[g], xw[b], sum2(acc2[b][g]));
        }
        // 2. sum over the cell's 8 lanes: a butterfly over the lane bits above the batch items'
        //    and a halving exchange over the others, after which slot 0 of lane l8 holds the four
        //    gate pre-activations of item l8 mod BG; then that item's state update
#pragma unroll
        for (int M = 4; M >= 1; M >>= 1) {
            if (M >= BG) {
#pragma unroll
                for (int b = 0; b < BG; ++b)
#pragma unroll
                    for (int g = 0; g < 4; ++g) acc[b][g] += __shfl_xor_sync(0xffffffffu, acc[b][g], M);
            } else {
                // the live slots are 0 .. 2M - 1 (item bits below 2M); keep the half whose bit M
                // matches this lane's bit M, in slots 0 .. M - 1
                const bool up = (l8 & M) != 0;
#pragma unroll
                for (int b = 0; b < M; ++b) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const float send = up ? acc[b][g] : acc[b | M][g];
                        const float keep = up ? acc[b | M][g] : acc[b][g];
                        acc[b][g] = keep + __shfl_xor_sync(0xffffffffu, send, M);
                    }
                }
            }
        }
        {
            const float gi = acc[0][0], gf = acc[0][1], gz = acc[0][2], go = acc[0][3];
            const float lf = exp_forget ? gf : log_sigmoid(gf);
            const float mn = fmaxf(lf + m, gi);
            const float fw = expf(lf + m - mn);
            const float iw = expf(gi - mn);
            c = fw * c + iw * tanhf(gz);
            n = fw * n + iw;
            m = mn;
            hv = sigmoidf_(go) * (c / n);
        }
        // 3. publish h_t to every CTA of the cluster (not after the last step: nobody reads it).
        //    The copies of item it share the ranks (copy ci writes ranks ci, ci + 8 / BG, ...);
        //    every (item, cell) slot is written, so that each fill is exactly FILL_BYTES.  A CTA
        //    writes buffer nxt of a peer only after it has h_t of every CTA, that is after every
        //    CTA has finished step t's reads of that buffer's previous contents.
        const int nxt = cur ^ 1;
        if constexpr (G > 1) {
            if (t + 1 < S) {
#pragma unroll
                for (int r = 0; r < G; r += DUP)
                    if (r + ci < G) st_async_cluster(&hs[nxt][it][j], &fill[nxt], (uint32_t)(r + ci), hv);
            }
        } else {
            hs[nxt][it][j] = hv;
        }
        if (item_ok && h_out != nullptr && ci == 0)
            h_out[(((size_t)(b0 + it) * S + t) * NH + head) * DH + j] = from_f32<T>(hv);
#pragma unroll
        for (int b = 0; b < BG; ++b) {
            const bool ld = has_x && b0 + b < B && t + 1 < S;
            const size_t off = ((size_t)(b0 + b) * S + t + 1) * 4 * HD;
            xw[b] = ld ? to_f32(wxr[off]) : 0.f;
            if (ld && t + 16 < S)                              // warm L2 further ahead
                asm volatile("prefetch.global.L2 [%0];" ::"l"(wxr + off + 15 * 4 * HD));
        }
        if constexpr (G == 1) __syncthreads();
    }
    // no CTA leaves while a peer may still address its shared memory
    if (G > 1) cluster_sync_release_acquire();
    griddep_launch_dependents();
    // the state after step S (copy 0 of each item)
    if (item_ok && ci == 0) {
        const size_t s = ((size_t)(b0 + it) * NH + head) * DH + j;
        c_st[s] = c;
        n_st[s] = n;
        m_st[s] = m;
        h_st[s] = hv;
    }
}

template <typename T, int DH, int BG>
static cudaError_t launch_bg(const void *wx, const void *R, int B, int S, int NH, int fs, float *c, float *n, float *m,
                             float *h, void *h_out, uint32_t *status, cudaStream_t st)
{
    constexpr int G = DH / CELLS;
    const int ngrp = (B + BG - 1) / BG;
    const dim3 grid((unsigned)(NH * ngrp * G));
    return launch_kernel(slstm_kernel<T, DH, BG>, grid, dim3(THREADS), 0, st, G, static_cast<const T *>(wx),
                         static_cast<const T *>(R), B, S, NH, fs, c, n, m, h, static_cast<T *>(h_out), status);
}

// Clusters of this kernel that fit on the device at once (cached per kernel and device, under the
// library's host-cache lock).
template <typename T, int DH, int BG>
static int max_clusters()
{
    struct Entry { int dev; int v; };
    static Entry cache[16];
    static int used = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> guard(host_cache_mutex());
    for (int i = 0; i < used; ++i)
        if (cache[i].dev == dev) return cache[i].v;
    constexpr int G = DH / CELLS;
    int v = 0;
    if (G > 1) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(G * 64);
        cfg.blockDim = dim3(THREADS);
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = G;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&v, slstm_kernel<T, DH, BG>, &cfg) != cudaSuccess) {
            cudaGetLastError();
            v = 0;
        }
    } else {
        int per_sm = 0, sms = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, slstm_kernel<T, DH, BG>, THREADS, 0) ==
                cudaSuccess &&
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
            v = per_sm * sms;
        else
            cudaGetLastError();
    }
    if (used < 16) cache[used++] = Entry{dev, v};
    return v;
}

// Smallest batch group whose clusters all fit on the device at once, else the largest.
template <typename T, int DH>
static int choose_bg(int B, int NH)
{
    const int caps[4] = {max_clusters<T, DH, 1>(), max_clusters<T, DH, 2>(), max_clusters<T, DH, 4>(),
                         max_clusters<T, DH, 8>()};
    const int bgs[4] = {1, 2, 4, 8};
    for (int i = 0; i < 4; ++i) {
        const long long need = (long long)NH * ((B + bgs[i] - 1) / bgs[i]);
        if (caps[i] > 0 && need <= caps[i]) return bgs[i];
    }
    return MAX_BG;
}

template <typename T, int DH>
static cudaError_t launch_dh(const void *wx, const void *R, int B, int S, int NH, int fs, float *c, float *n, float *m,
                             float *h, void *h_out, uint32_t *status, cudaStream_t st)
{
    switch (choose_bg<T, DH>(B, NH)) {
    case 1: return launch_bg<T, DH, 1>(wx, R, B, S, NH, fs, c, n, m, h, h_out, status, st);
    case 2: return launch_bg<T, DH, 2>(wx, R, B, S, NH, fs, c, n, m, h, h_out, status, st);
    case 4: return launch_bg<T, DH, 4>(wx, R, B, S, NH, fs, c, n, m, h, h_out, status, st);
    default: return launch_bg<T, DH, 8>(wx, R, B, S, NH, fs, c, n, m, h, h_out, status, st);
    }
}

template <typename T>
static cudaError_t launch_t(const void *wx, const void *R, int B, int S, int NH, int DH, int fs, float *c, float *n,
                            float *m, float *h, void *h_out, uint32_t *status, cudaStream_t st)
{
    switch (DH) {
    case 32: return launch_dh<T, 32>(wx, R, B, S, NH, fs, c, n, m, h, h_out, status, st);
    case 64: return launch_dh<T, 64>(wx, R, B, S, NH, fs, c, n, m, h, h_out, status, st);
    case 128: return launch_dh<T, 128>(wx, R, B, S, NH, fs, c, n, m, h, h_out, status, st);
    case 192: return launch_dh<T, 192>(wx, R, B, S, NH, fs, c, n, m, h, h_out, status, st);
    default: return launch_dh<T, 256>(wx, R, B, S, NH, fs, c, n, m, h, h_out, status, st);
    }
}

template <typename T>
static int bg_t(int B, int NH, int DH)
{
    switch (DH) {
    case 32: return choose_bg<T, 32>(B, NH);
    case 64: return choose_bg<T, 64>(B, NH);
    case 128: return choose_bg<T, 128>(B, NH);
    case 192: return choose_bg<T, 192>(B, NH);
    default: return choose_bg<T, 256>(B, NH);
    }
}

static bool supported_dh(int DH) { return DH == 32 || DH == 64 || DH == 128 || DH == 192 || DH == 256; }

static bool aligned(const void *p, unsigned a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1u)) == 0; }

}  // namespace slstm
}  // namespace mlstm

extern "C" mlstm_status slstm_fwd(const void *wx, const void *R, mlstm_dtype dt, int B, int S, int NH, int DH,
                                  int forget_sigmoid, float *c, float *n, float *m, float *h, void *h_out,
                                  unsigned int *status, void *stream)
{
    using namespace mlstm::slstm;
    if (B < 0 || S < 0 || NH < 1 || DH < 1) return MLSTM_ERR_INVALID_ARG;
    if (dt != MLSTM_F32 && dt != MLSTM_BF16) return MLSTM_ERR_UNSUPPORTED;
    if (!supported_dh(DH)) return MLSTM_ERR_UNSUPPORTED;
    if (B == 0 || S == 0) return MLSTM_OK;           // nothing to run; the state stays as it is
    if (!wx || !R || !c || !n || !m || !h) return MLSTM_ERR_INVALID_ARG;
    const unsigned es = dt == MLSTM_F32 ? 4u : 2u;
    if (!aligned(wx, es) || !aligned(R, 16u) || (h_out && !aligned(h_out, es))) return MLSTM_ERR_INVALID_ARG;
    if (!aligned(c, 4u) || !aligned(n, 4u) || !aligned(m, 4u) || !aligned(h, 4u)) return MLSTM_ERR_INVALID_ARG;
    if (status && !aligned(status, 4u)) return MLSTM_ERR_INVALID_ARG;
    if ((long long)B * NH * (DH / CELLS) > (1ll << 31) - 1) return MLSTM_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint32_t *sw = reinterpret_cast<uint32_t *>(status);
    const cudaError_t e = dt == MLSTM_F32
                              ? launch_t<float>(wx, R, B, S, NH, DH, forget_sigmoid, c, n, m, h, h_out, sw, st)
                              : launch_t<__nv_bfloat16>(wx, R, B, S, NH, DH, forget_sigmoid, c, n, m, h, h_out, sw, st);
    return e == cudaSuccess ? MLSTM_OK : MLSTM_ERR_CUDA;
}

extern "C" int slstm_batch_per_cluster(int B, int NH, int DH, mlstm_dtype dt)
{
    using namespace mlstm::slstm;
    if (B < 0 || NH < 1 || !supported_dh(DH) || (dt != MLSTM_F32 && dt != MLSTM_BF16)) return 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return dt == MLSTM_F32 ? bg_t<float>(B, NH, DH) : bg_t<__nv_bfloat16>(B, NH, DH);
}
