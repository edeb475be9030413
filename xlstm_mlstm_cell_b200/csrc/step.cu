// step.cu -- the recurrent decode step of the mLSTM cell (one token, state in place).
//
// "xLSTM Guide: Extended LSTM Architecture & Matrix Memory", "Recurrent
// Formulation (Inference Mode)" applied once per (batch, head):
//   m' = max(log f + m, i~),  f' = exp(log f + m - m'),  i' = exp(i~ - m')
//   C' = f' C + i' k v^T,     n' = f' n + i' k
//   h  = o * (C'^T qh) / max(|n' . qh|, exp(-m')),  qh = q / sqrt(DHQK)
//
// The step is bound by HBM: every byte of the fp32 state C is read once and
// written once, and nothing else is of comparable size.  The value columns of
// one head's state are split over a thread-block cluster of G CTAs (G = 1 when
// there are enough heads to fill the GPU).  In a CTA, threads form RG row
// groups of CW/4 threads (CW = DHV / G columns); a thread owns four consecutive
// columns of C (one 16-byte vector) and walks the rows i = g, g + RG, ... so
// that each iteration the CTA streams RG rows of its column slice.  Column sums
// stay in the thread and are combined over row groups through shared memory;
// each CTA then writes h for its own columns.  Every CTA forms n' and n' . qh
// itself (DHQK values); only the cluster's first CTA writes n' and m', after a
// cluster barrier has made sure that every CTA has read the old ones.  C is
// loaded and stored with the streaming (evict-first) cache hint since it is
// touched once per step.
#include "common.cuh"
#include "mlstm_internal.h"

namespace mlstm {

template <typename T, int UNROLL, int G>
__global__ void __launch_bounds__(512, 2)
step_kernel(float *__restrict__ C, float *__restrict__ n, float *__restrict__ m,
            const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
            const float *__restrict__ igate, const float *__restrict__ fgate,
            const T *__restrict__ ogate, int DHQK, int DHV, int RG, T *__restrict__ h)
{
    extern __shared__ float smem[];
    const int CW = DHV / G;           // value columns of this CTA
    float *qs = smem;                 // [DHQK] qh
    float *ks = qs + DHQK;            // [DHQK] k
    float *ns = ks + DHQK;            // [DHQK] n'
    float *part = ns + DHQK;          // [RG][CW] partial column sums
    __shared__ float red[32];

    const int bh = blockIdx.x / G;
    const int rank = blockIdx.x % G;  // rank in the cluster (the cluster spans G consecutive CTAs)
    const int tid = threadIdx.x;
    const int nthr = blockDim.x;
    const int tx = tid % (CW / 4);    // column group
    const int g = tid / (CW / 4);     // row group
    const int jl = tx * 4;            // first column of the thread in the CTA's slice
    const int j = rank * CW + jl;     // ... and in the head
    griddep_wait();
    griddep_launch_dependents();

    // the thread's first UNROLL rows of C and the small per-head inputs are requested together,
    // so that their latencies overlap (the remaining rows follow UNROLL at a time)
    float *Cb = C + (size_t)bh * DHQK * DHV + j;
    float4 c[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
        const int i = g + u * RG;
        if (i < DHQK) c[u] = __ldcs(reinterpret_cast<const float4 *>(Cb + (size_t)i * DHV));
    }
    const T *qb = q + (size_t)bh * DHQK;
    const T *kb = k + (size_t)bh * DHQK;
    float *nb = n + (size_t)bh * DHQK;
    const float fgv = fgate[bh], it = igate[bh], m_old = m[bh];
    float q0 = 0.f, k0 = 0.f, n0 = 0.f;
    if (tid < DHQK) {
        q0 = to_f32(qb[tid]);
        k0 = to_f32(kb[tid]);
        n0 = nb[tid];
    }
    const float4 v4 = load4(v + (size_t)bh * DHV + j);

    const float lf = log_sigmoid(fgv);
    const float m_new = fmaxf(lf + m_old, it);
    const float fp = expf(lf + m_old - m_new);
    const float ip = expf(it - m_new);
    const float scale = rsqrtf((float)DHQK);

    float den = 0.f;
    for (int i = tid; i < DHQK; i += nthr) {
        const bool first = (i == tid);
        const float qi = (first ? q0 : to_f32(qb[i])) * scale;
        const float ki = first ? k0 : to_f32(kb[i]);
        const float ni = fp * (first ? n0 : nb[i]) + ip * ki;
        ns[i] = ni;
        qs[i] = qi;
        ks[i] = ki;
        den += ni * qi;
    }
    den = warp_sum(den);
    if ((tid & 31) == 0) red[tid >> 5] = den;
    __syncthreads();
    if (tid < 32) {
        float x = tid < (nthr + 31) / 32 ? red[tid] : 0.f;
        x = warp_sum(x);
        if (tid == 0) red[0] = x;
    }

    const float4 iv = make_float4(ip * v4.x, ip * v4.y, ip * v4.z, ip * v4.w);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i0 = g; i0 < DHQK; i0 += UNROLL * RG) {
        if (i0 != g) {
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int i = i0 + u * RG;
                if (i < DHQK) c[u] = __ldcs(reinterpret_cast<const float4 *>(Cb + (size_t)i * DHV));
            }
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int i = i0 + u * RG;
            if (i < DHQK) {
                const float kk = ks[i], qq = qs[i];
                c[u].x = fmaf(fp, c[u].x, kk * iv.x);
                c[u].y = fmaf(fp, c[u].y, kk * iv.y);
                c[u].z = fmaf(fp, c[u].z, kk * iv.z);
                c[u].w = fmaf(fp, c[u].w, kk * iv.w);
                __stcs(reinterpret_cast<float4 *>(Cb + (size_t)i * DHV), c[u]);
                acc.x = fmaf(qq, c[u].x, acc.x);
                acc.y = fmaf(qq, c[u].y, acc.y);
                acc.z = fmaf(qq, c[u].z, acc.z);
                acc.w = fmaf(qq, c[u].w, acc.w);
            }
        }
    }
    *reinterpret_cast<float4 *>(part + (size_t)g * CW + jl) = acc;
    __syncthreads();
    if (g == 0) {   // this CTA's column sums over all rows: h for its columns
        for (int r = 1; r < RG; ++r) {
            const float4 pr = *reinterpret_cast<const float4 *>(part + (size_t)r * CW + jl);
            acc.x += pr.x; acc.y += pr.y; acc.z += pr.z; acc.w += pr.w;
        }
        float4 o4 = make_float4(1.f, 1.f, 1.f, 1.f);
        if (ogate) o4 = load4(ogate + (size_t)bh * DHV + j);
        const float inv = 1.f / fmaxf(fabsf(red[0]), expf(-m_new));
        store4(h + (size_t)bh * DHV + j,
               make_float4(o4.x * acc.x * inv, o4.y * acc.y * inv, o4.z * acc.z * inv, o4.w * acc.w * inv));
    }
    if constexpr (G > 1) {
        // every CTA of the head has read the old n and m (their values are consumed above, so the
        // loads are complete); a relaxed arrive does not wait for this CTA's stores of C to drain
        asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
        asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    }
    if (rank == 0) {
        for (int i = tid; i < DHQK; i += nthr) nb[i] = ns[i];
        if (tid == 0) m[bh] = m_new;
    }
}

template <typename T, int G>
static cudaError_t launch_step_g(const StepArgs &a, int RG, int threads, size_t smem)
{
    return launch_kernel(step_kernel<T, 8, G>, dim3(a.BH * G), dim3(threads), smem, a.stream, G, a.C, a.n, a.m,
                         (const T *)a.q, (const T *)a.k, (const T *)a.v, a.igate, a.fgate, (const T *)a.ogate, a.DHQK,
                         a.DHV, RG, (T *)a.h);
}

// Value columns of one head are split over G CTAs when there are too few heads for two waves of CTAs
// (each CTA keeps a multiple of four columns).
static int step_cluster_size(int BH, int DHV)
{
    int G = 1;
    while (G < 8 && (long long)BH * G < 2 * 148 && DHV % (8 * G) == 0) G *= 2;
    return G;
}

template <typename T>
static cudaError_t launch_step_t(const StepArgs &a)
{
    const int G = step_cluster_size(a.BH, a.DHV);
    const int tx = a.DHV / G / 4;
    int RG = 512 / tx;
    if (RG < 1) RG = 1;
    if (RG > a.DHQK) RG = a.DHQK;
    const int threads = tx * RG;
    const size_t smem = sizeof(float) * (3 * (size_t)a.DHQK + (size_t)RG * (a.DHV / G));
    if (smem > 48 * 1024) {
        cudaError_t e = ensure_dynamic_smem(G == 1 ? (const void *)step_kernel<T, 8, 1>
                                                   : G == 2 ? (const void *)step_kernel<T, 8, 2>
                                                   : G == 4 ? (const void *)step_kernel<T, 8, 4>
                                                            : (const void *)step_kernel<T, 8, 8>,
                                            (int)smem);
        if (e != cudaSuccess) return e;
    }
    switch (G) {
    case 1: return launch_step_g<T, 1>(a, RG, threads, smem);
    case 2: return launch_step_g<T, 2>(a, RG, threads, smem);
    case 4: return launch_step_g<T, 4>(a, RG, threads, smem);
    default: return launch_step_g<T, 8>(a, RG, threads, smem);
    }
}

cudaError_t launch_step(const StepArgs &a)
{
    return a.bf16 ? launch_step_t<__nv_bfloat16>(a) : launch_step_t<float>(a);
}

}  // namespace mlstm
