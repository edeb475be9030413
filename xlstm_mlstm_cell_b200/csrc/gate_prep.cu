// gate_prep.cu -- gate preprocessing of the chunkwise forward pass.
//
// For every (batch, head) and chunk c of length L (the last chunk may be
// shorter), with log f_t = logsigmoid(f~_t):
//   a_tau   = sum_{s <= tau} log f_s            chunk-local inclusive cumulative sum
//   g_c     = a at the chunk's last token       total log decay of the chunk
//   p_tau   = max_{s <= tau} (i~_s - a_s)       chunk-local prefix maximum
//   m_{c+1} = max(m_c + g_c, g_c + p_last)      stabilizer at the next chunk start
//   m_tau   = a_tau + max(m_c, p_tau)           stabilizer of every token
// which is the running-max stabilizer m_t = max(m_{t-1} + log f_t, i~_t) of
// "The Stabilizer State" (xLSTM Guide: Extended LSTM Architecture & Matrix
// Memory) unrolled over a chunk.  The maps m -> max(m + g, b) compose
// associatively ((g1, b1) then (g2, b2) = (g1 + g2, max(b1 + g2, b2))), so the
// scan across chunks is a parallel max-plus scan, the "low-overhead
// associative scan" of the guide's "Exploit Chunkwise Hardware Kernels".
//
// Two kernels (one, gate_fused_kernel, for heads of at most 4096 tokens).
// gate_local_kernel is parallel over all chunks of all heads (a warp per chunk,
// 32 tokens per pass, warp shuffles for the sums and maxima) and writes a and p
// per token, g and b per chunk.  gate_scan_kernel runs one CTA per head: it scans the chunk maps (m_c for every chunk start from the initial m_0),
// and, for the tensor-core path, composes the maps of each segment of R chunks
// and the in-segment prefix of the chunk decays.  The per-token stabilizer m_tau
// is not stored: the consumers form it from a_tau, p_tau and m_c.
#include "common.cuh"
#include "mlstm_internal.h"

namespace mlstm {

constexpr int GL_WARPS = 8;   // chunks per CTA of gate_local_kernel

// One warp: chunk c of head bh.
__device__ __forceinline__ void local_chunk(const float *__restrict__ igate, const float *__restrict__ fgate, int S,
                                            int L, int NC, int bh, int c, int lane, float *__restrict__ A,
                                            float *__restrict__ P, float *__restrict__ G, float *__restrict__ Bc,
                                            float *g_sm = nullptr, float *b_sm = nullptr)
{
    const float *ig = igate + (size_t)bh * S;
    const float *fg = fgate + (size_t)bh * S;
    float *a_out = A + (size_t)bh * S;
    float *p_out = P + (size_t)bh * S;
    const int t0 = c * L;
    const int t1 = min(t0 + L, S);
    // the chunk's gate values (at most four passes of 32 tokens: L <= 128) are requested before
    // the serial passes, so that one memory latency covers them all
    float fv[4], iv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int t = t0 + u * 32 + lane;
        fv[u] = t < t1 ? fg[t] : 0.f;
        iv[u] = t < t1 ? ig[t] : 0.f;
    }
    float carry_a = 0.f, carry_p = -INFINITY;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int base = t0 + u * 32;
        if (base >= t1) break;
        const int t = base + lane;
        const bool ok = t < t1;
        float x = ok ? log_sigmoid(fv[u]) : 0.f;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        const float a = carry_a + x;
        float p = ok ? iv[u] - a : -INFINITY;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, p, o);
            if (lane >= o) p = fmaxf(p, y);
        }
        p = fmaxf(p, carry_p);
        if (ok) {
            a_out[t] = a;
            p_out[t] = p;
        }
        const int last = min(31, t1 - 1 - base);
        carry_a = __shfl_sync(0xffffffffu, a, last);
        carry_p = __shfl_sync(0xffffffffu, p, last);
    }
    if (lane == 0) {
        G[(size_t)bh * NC + c] = carry_a;
        Bc[(size_t)bh * NC + c] = carry_a + carry_p;
        if (g_sm) {              // the fused kernel's scan reads them from shared memory
            g_sm[c] = carry_a;
            b_sm[c] = carry_a + carry_p;
        }
    }
}

__global__ void __launch_bounds__(GL_WARPS * 32)
gate_local_kernel(const float *__restrict__ igate, const float *__restrict__ fgate, int S, int L, int NC,
                  float *__restrict__ A, float *__restrict__ P, float *__restrict__ G, float *__restrict__ Bc,
                  uint32_t *__restrict__ status)
{
    griddep_wait();
    // this call's status word, reset before any kernel that may report into it starts
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *status = 0u;
    griddep_launch_dependents();
    const int c = blockIdx.x * GL_WARPS + (threadIdx.x >> 5);
    if (c < NC) local_chunk(igate, fgate, S, L, NC, blockIdx.y, c, threadIdx.x & 31, A, P, G, Bc);
}

constexpr int GS_THREADS = 1024;   // most threads of gate_scan_kernel; a launch uses a multiple of 32 up to this
constexpr int GS_STAGE = 4096;     // chunk maps per head staged in shared memory by the scan
// One kernel does both steps when a head has at most FUSED_MAX_S tokens: its warps then walk at
// most FUSED_MAX_S / 1024 serial passes of 32 tokens, fewer than the second launch costs.
constexpr int FUSED_MAX_S = 4096;

// One CTA: the chunk maps of head bh (G, Bc written before by this CTA or an earlier kernel).
// g_in, b_in: the head's chunk maps, in shared memory when they fit (the serial loops below then
// read shared memory instead of waiting on one global load after another), else in global memory.
__device__ __forceinline__ void scan_head(int NC, const float *g_in, const float *b_in, float *__restrict__ MC,
                                          int R, int NSEG, float *__restrict__ GP, float *__restrict__ SGb,
                                          const float *__restrict__ m0, int bh)
{
    __shared__ float wa[32], wb[32];                 // per-warp totals, then their exclusive prefixes
    const int tid = threadIdx.x;
    const int nthr = blockDim.x;
    float *mc_out = MC + (size_t)bh * (NC + 1);

    // each thread composes the maps of a contiguous range of chunks
    const int per = (NC + nthr - 1) / nthr;
    const int c0 = min(tid * per, NC), c1 = min(c0 + per, NC);
    float ga = 0.f, gb = -INFINITY;
    for (int c = c0; c < c1; ++c) {
        const float g = g_in[c];
        ga += g;
        gb = fmaxf(gb + g, b_in[c]);
    }
    // exclusive scan of the maps across threads, composing (earlier) then (later):
    // (a1, b1) then (a2, b2) = (a1 + a2, max(b1 + a2, b2)).  Shuffle scan inside each warp, then
    // the first warp scans the warp totals.
    const int lane = tid & 31, warp = tid >> 5, nwarp = (nthr + 31) >> 5;
    float ia = ga, ib = gb;            // inclusive within the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float pa = __shfl_up_sync(0xffffffffu, ia, o), pb = __shfl_up_sync(0xffffffffu, ib, o);
        if (lane >= o) {
            ib = fmaxf(pb + ia, ib);
            ia = pa + ia;
        }
    }
    float xa = __shfl_up_sync(0xffffffffu, ia, 1), xb = __shfl_up_sync(0xffffffffu, ib, 1);
    if (lane == 0) {                   // exclusive within the warp
        xa = 0.f;
        xb = -INFINITY;
    }
    if (lane == 31) {
        wa[warp] = ia;
        wb[warp] = ib;
    }
    __syncthreads();
    if (warp == 0) {
        float ta = lane < nwarp ? wa[lane] : 0.f, tb = lane < nwarp ? wb[lane] : -INFINITY;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float pa = __shfl_up_sync(0xffffffffu, ta, o), pb = __shfl_up_sync(0xffffffffu, tb, o);
            if (lane >= o) {
                tb = fmaxf(pb + ta, tb);
                ta = pa + ta;
            }
        }
        float ua = __shfl_up_sync(0xffffffffu, ta, 1), ub = __shfl_up_sync(0xffffffffu, tb, 1);
        if (lane == 0) {
            ua = 0.f;
            ub = -INFINITY;
        }
        wa[lane] = ua;                 // exclusive prefix of the warp totals
        wb[lane] = ub;
    }
    __syncthreads();
    // the thread's exclusive prefix: the warp's prefix, then the lanes before it
    const float ea = wa[warp] + xa, eb = fmaxf(wb[warp] + xa, xb);
    const float m_init = m0 ? m0[bh] : 0.f;
    float mm = fmaxf(m_init + ea, eb);   // m at this thread's first chunk
    for (int c = c0; c < c1; ++c) {
        mc_out[c] = mm;
        mm = fmaxf(mm + g_in[c], b_in[c]);
    }
    if (c1 == NC && c0 < c1) mc_out[NC] = mm;
    if (NC == 0 && tid == 0) mc_out[0] = m_init;

    // segments of R chunks: in-segment prefix of the chunk decays and the composed segment map
    for (int sg = tid; sg < NSEG; sg += nthr) {
        float sga = 0.f, sgb = -INFINITY;
        const int e1 = min((sg + 1) * R, NC);
        for (int c = sg * R; c < e1; ++c) {
            GP[(size_t)bh * NC + c] = sga;
            const float g = g_in[c];
            sga += g;
            sgb = fmaxf(sgb + g, b_in[c]);
        }
        SGb[((size_t)bh * NSEG + sg) * 2 + 0] = sga;
        SGb[((size_t)bh * NSEG + sg) * 2 + 1] = sgb;
    }
}

__global__ void __launch_bounds__(GS_THREADS)
gate_scan_kernel(int NC, const float *__restrict__ G, const float *__restrict__ Bc, float *__restrict__ MC,
                 int R, int NSEG, float *__restrict__ GP, float *__restrict__ SGb, const float *__restrict__ m0)
{
    griddep_wait();
    griddep_launch_dependents();
    __shared__ float g_st[GS_STAGE], b_st[GS_STAGE];
    const int bh = blockIdx.x;
    const float *g_in = G + (size_t)bh * NC, *b_in = Bc + (size_t)bh * NC;
    if (NC <= GS_STAGE) {   // parallel, coalesced loads into shared memory
        for (int c = threadIdx.x; c < NC; c += blockDim.x) {
            g_st[c] = g_in[c];
            b_st[c] = b_in[c];
        }
        __syncthreads();
        g_in = g_st;
        b_in = b_st;
    }
    scan_head(NC, g_in, b_in, MC, R, NSEG, GP, SGb, m0, bh);
}

// Both steps in one CTA per head for short sequences (at most FUSED_MAX_S tokens): the CTA's
// warps take the chunks in turn, then the CTA scans the maps it has just written.
__global__ void __launch_bounds__(GS_THREADS)
gate_fused_kernel(const float *__restrict__ igate, const float *__restrict__ fgate, int S, int L, int NC,
                  float *__restrict__ A, float *__restrict__ P, float *__restrict__ G, float *__restrict__ Bc,
                  float *__restrict__ MC, int R, int NSEG, float *__restrict__ GP, float *__restrict__ SGb,
                  const float *__restrict__ m0, uint32_t *__restrict__ status)
{
    griddep_wait();
    const int bh = blockIdx.x;
    // this call's status word, reset before any kernel that may report into it starts
    if (bh == 0 && threadIdx.x == 0) *status = 0u;
    griddep_launch_dependents();
    __shared__ float g_st[FUSED_MAX_S / 16], b_st[FUSED_MAX_S / 16];   // chunk 16 at most 256 chunks
    for (int c = threadIdx.x >> 5; c < NC; c += GS_THREADS / 32)
        local_chunk(igate, fgate, S, L, NC, bh, c, threadIdx.x & 31, A, P, G, Bc, g_st, b_st);
    __syncthreads();   // the head's chunk maps are in shared memory
    scan_head(NC, g_st, b_st, MC, R, NSEG, GP, SGb, m0, bh);
}

int gate_prep_launches(int S, int NC)
{
    return NC == 0 ? 0 : (S <= FUSED_MAX_S ? 1 : 2);
}

cudaError_t launch_gate_prep(const GatePrepArgs &a)
{
    if (a.NC == 0) return cudaSuccess;
    if (a.S <= FUSED_MAX_S) {
        return launch_kernel(gate_fused_kernel, dim3(a.BH), dim3(GS_THREADS), 0, a.stream, 1, a.igate, a.fgate, a.S,
                             a.L, a.NC, a.A, a.M, a.G, a.Bc, a.MC, a.R, a.NSEG, a.GP, a.SGb, a.m0, a.status);
    }
    dim3 g1((a.NC + GL_WARPS - 1) / GL_WARPS, a.BH);
    cudaError_t e = launch_kernel(gate_local_kernel, g1, dim3(GL_WARPS * 32), 0, a.stream, 1, a.igate, a.fgate, a.S,
                                  a.L, a.NC, a.A, a.M, a.G, a.Bc, a.status);
    if (e != cudaSuccess) return e;
    const int scan_threads = a.NC >= GS_THREADS ? GS_THREADS : (a.NC + 31) / 32 * 32;
    return launch_kernel(gate_scan_kernel, dim3(a.BH), dim3(scan_threads), 0, a.stream, 1, a.NC, a.G, a.Bc, a.MC,
                         a.R, a.NSEG, a.GP, a.SGb, a.m0);
}

}  // namespace mlstm
