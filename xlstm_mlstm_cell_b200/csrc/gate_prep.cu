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
// One CTA per (batch, head), 32 warps.  Phase 1: each warp takes whole chunks
// (32 tokens per pass, warp shuffles for the sums and maxima) and writes a and
// p per token, g and b per chunk.  Phase 2: warp 0 scans the chunk maps.
// Phase 3: all threads write m per token.  The cost is a few bytes per token.
#include "common.cuh"
#include "mlstm_internal.h"

namespace mlstm {

__global__ void __launch_bounds__(1024)
gate_prep_kernel(const float *__restrict__ igate, const float *__restrict__ fgate, int S, int L, int NC,
                 float *__restrict__ A, float *__restrict__ Mtok, float *__restrict__ G,
                 float *__restrict__ Bc, float *__restrict__ MC, int R, int NSEG,
                 float *__restrict__ GP, float *__restrict__ SGb)
{
    const int bh = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
    const float *ig = igate + (size_t)bh * S;
    const float *fg = fgate + (size_t)bh * S;
    float *a_out = A + (size_t)bh * S;
    float *m_out = Mtok + (size_t)bh * S;   // holds p until phase 3
    float *g_out = G + (size_t)bh * NC;
    float *b_out = Bc + (size_t)bh * NC;
    float *mc_out = MC + (size_t)bh * (NC + 1);

    // Phase 1: chunk-local cumulative log decay and prefix maximum.
    for (int c = warp; c < NC; c += nwarp) {
        const int t0 = c * L;
        const int t1 = min(t0 + L, S);
        float carry_a = 0.f, carry_p = -INFINITY;
        for (int base = t0; base < t1; base += 32) {
            const int t = base + lane;
            const bool ok = t < t1;
            float x = ok ? log_sigmoid(fg[t]) : 0.f;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            const float a = carry_a + x;
            float p = ok ? ig[t] - a : -INFINITY;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, p, o);
                if (lane >= o) p = fmaxf(p, y);
            }
            p = fmaxf(p, carry_p);
            if (ok) {
                a_out[t] = a;
                m_out[t] = p;
            }
            const int last = min(31, t1 - 1 - base);
            carry_a = __shfl_sync(0xffffffffu, a, last);
            carry_p = __shfl_sync(0xffffffffu, p, last);
        }
        if (lane == 0) {
            g_out[c] = carry_a;
            b_out[c] = carry_a + carry_p;
        }
    }
    __syncthreads();

    // Phase 1b (segments of R chunks): in-segment prefix of the chunk decays and the
    // segment map, the composition of its chunk maps.
    for (int sg = threadIdx.x; sg < NSEG; sg += blockDim.x) {
        float ga = 0.f, gb = -INFINITY;
        const int c1 = min((sg + 1) * R, NC);
        for (int c = sg * R; c < c1; ++c) {
            GP[(size_t)bh * NC + c] = ga;
            const float g = g_out[c];
            ga += g;
            gb = fmaxf(gb + g, b_out[c]);
        }
        SGb[((size_t)bh * NSEG + sg) * 2 + 0] = ga;
        SGb[((size_t)bh * NSEG + sg) * 2 + 1] = gb;
    }

    // Phase 2: max-plus scan of the chunk maps m -> max(m + g_c, b_c), m_0 = 0.
    if (warp == 0) {
        const int per = (NC + 31) / 32;
        const int c0 = min(lane * per, NC), c1 = min(c0 + per, NC);
        float ga = 0.f, gb = -INFINITY;                 // this lane's composed map
        for (int c = c0; c < c1; ++c) {
            const float g = g_out[c];
            ga += g;
            gb = fmaxf(gb + g, b_out[c]);
        }
        // inclusive scan of maps across lanes, then shift to exclusive
        float sa = ga, sb = gb;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float pa = __shfl_up_sync(0xffffffffu, sa, o);
            const float pb = __shfl_up_sync(0xffffffffu, sb, o);
            if (lane >= o) {           // (pa, pb) then (sa, sb)
                sb = fmaxf(pb + sa, sb);
                sa = pa + sa;
            }
        }
        float ea = __shfl_up_sync(0xffffffffu, sa, 1);
        float eb = __shfl_up_sync(0xffffffffu, sb, 1);
        if (lane == 0) { ea = 0.f; eb = -INFINITY; }
        float mm = fmaxf(0.f + ea, eb);
        for (int c = c0; c < c1; ++c) {
            mc_out[c] = mm;
            mm = fmaxf(mm + g_out[c], b_out[c]);
        }
        if (c1 == NC && c0 < c1) mc_out[NC] = mm;
        if (NC == 0 && lane == 0) mc_out[0] = 0.f;
    }
    __syncthreads();

    // Phase 3: per-token stabilizer m_tau = a_tau + max(m_c, p_tau).
    for (int t = threadIdx.x; t < S; t += blockDim.x) {
        const int c = t / L;
        m_out[t] = a_out[t] + fmaxf(mc_out[c], m_out[t]);
    }
}

cudaError_t launch_gate_prep(const GatePrepArgs &a)
{
    gate_prep_kernel<<<a.BH, 1024, 0, a.stream>>>(a.igate, a.fgate, a.S, a.L, a.NC, a.A, a.M, a.G, a.Bc,
                                                  a.MC, a.R, a.NSEG, a.GP, a.SGb);
    return cudaGetLastError();
}

}  // namespace mlstm
