// step.cu -- the recurrent decode step of the mLSTM cell (one token, state in place).
//
// "xLSTM Guide: Extended LSTM Architecture & Matrix Memory", "Recurrent
// Formulation (Inference Mode)" applied once per (batch, head):
//   m' = max(log f + m, i~),  f' = exp(log f + m - m'),  i' = exp(i~ - m')
//   C' = f' C + i' k v^T,     n' = f' n + i' k
//   h  = o * (C'^T qh) / max(|n' . qh|, exp(-m')),  qh = q / sqrt(DHQK)
//
// The step is bound by HBM: every byte of the fp32 state C is read once and
// written once, and nothing else is of comparable size.  The rows of one head's
// state are split over a thread-block cluster of G CTAs (G = 1 when there are
// enough heads to fill the GPU).  In a CTA, threads form RG row groups of DHV/4
// threads; a thread owns four consecutive columns of C (one 16-byte vector)
// and walks the rows i = g, g + RG, ... of its CTA's share, so that each
// iteration the CTA streams RG whole rows, contiguous in memory.  Column sums
// stay in the thread, are combined over row groups through shared memory and,
// for G > 1, over the cluster through distributed shared memory by the
// cluster's first CTA, which also forms n' . qh and writes h.  C is loaded and
// stored with the streaming (evict-first) cache hint since it is touched once
// per step.
#include <cooperative_groups.h>

#include "common.cuh"
#include "mlstm_internal.h"

namespace cg = cooperative_groups;

namespace mlstm {

template <typename T, int UNROLL, int G>
__global__ void __launch_bounds__(512, 2)
step_kernel(float *__restrict__ C, float *__restrict__ n, float *__restrict__ m,
            const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
            const float *__restrict__ igate, const float *__restrict__ fgate,
            const T *__restrict__ ogate, int DHQK, int DHV, int RG, T *__restrict__ h)
{
    extern __shared__ float smem[];
    const int rows = DHQK / G;        // rows of C handled by this CTA
    float *qs = smem;                 // [rows] qh
    float *ks = qs + rows;            // [rows] k
    float *part = ks + rows;          // [RG][DHV] partial column sums
    __shared__ float red[32];

    const int bh = blockIdx.x / G;
    const int rank = blockIdx.x % G;  // rank in the cluster (the cluster spans G consecutive CTAs)
    const int r0 = rank * rows;
    const int tid = threadIdx.x;
    const int nthr = blockDim.x;
    const int tx = tid % (DHV / 4);   // column group
    const int g = tid / (DHV / 4);    // row group

    // the thread's first UNROLL rows of C are requested before the gate arithmetic, so that their
    // latency overlaps it (the rest follow UNROLL at a time)
    const int j = tx * 4;
    float *Cb = C + ((size_t)bh * DHQK + r0) * DHV + j;
    float4 c[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
        const int i = g + u * RG;
        if (i < rows) c[u] = __ldcs(reinterpret_cast<const float4 *>(Cb + (size_t)i * DHV));
    }

    const float lf = log_sigmoid(fgate[bh]);
    const float it = igate[bh];
    const float m_old = m[bh];
    const float m_new = fmaxf(lf + m_old, it);
    const float fp = expf(lf + m_old - m_new);
    const float ip = expf(it - m_new);
    const float scale = rsqrtf((float)DHQK);

    const T *qb = q + (size_t)bh * DHQK + r0;
    const T *kb = k + (size_t)bh * DHQK + r0;
    float *nb = n + (size_t)bh * DHQK + r0;
    float den = 0.f;
    for (int i = tid; i < rows; i += nthr) {
        const float qi = to_f32(qb[i]) * scale;
        const float ki = to_f32(kb[i]);
        const float ni = fp * nb[i] + ip * ki;
        nb[i] = ni;
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

    const float4 v4 = load4(v + (size_t)bh * DHV + j);
    const float4 iv = make_float4(ip * v4.x, ip * v4.y, ip * v4.z, ip * v4.w);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);

    // UNROLL rows in flight per thread: all loads of a group are issued before any is used
    for (int i0 = g; i0 < rows; i0 += UNROLL * RG) {
        if (i0 != g) {
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int i = i0 + u * RG;
                if (i < rows) c[u] = __ldcs(reinterpret_cast<const float4 *>(Cb + (size_t)i * DHV));
            }
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int i = i0 + u * RG;
            if (i < rows) {
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
    *reinterpret_cast<float4 *>(part + (size_t)g * DHV + j) = acc;
    __syncthreads();
    if (g == 0) {   // this CTA's column sums, left in row group 0 of `part`
        for (int r = 1; r < RG; ++r) {
            const float4 pr = *reinterpret_cast<const float4 *>(part + (size_t)r * DHV + j);
            acc.x += pr.x; acc.y += pr.y; acc.z += pr.z; acc.w += pr.w;
        }
        *reinterpret_cast<float4 *>(part + j) = acc;
    }
    float dtot = red[0];
    if constexpr (G > 1) {
        cg::cluster_group cluster = cg::this_cluster();
        cluster.sync();                             // every CTA's partial sums are in its shared memory
        if (rank == 0 && g == 0) {
            for (int r = 1; r < G; ++r) {
                const float *rp = cluster.map_shared_rank(part, r);
                const float *rr = cluster.map_shared_rank(red, r);
                const float4 pr = *reinterpret_cast<const float4 *>(rp + j);
                acc.x += pr.x; acc.y += pr.y; acc.z += pr.z; acc.w += pr.w;
                dtot += rr[0];
            }
        }
        cluster.sync();                             // the remote reads are done before any CTA exits
    }
    if (rank == 0 && g == 0) {
        const float inv = 1.f / fmaxf(fabsf(dtot), expf(-m_new));
        float4 o4 = make_float4(1.f, 1.f, 1.f, 1.f);
        if (ogate) o4 = load4(ogate + (size_t)bh * DHV + j);
        store4(h + (size_t)bh * DHV + j,
               make_float4(o4.x * acc.x * inv, o4.y * acc.y * inv, o4.z * acc.z * inv, o4.w * acc.w * inv));
        if (tid == 0) m[bh] = m_new;
    }
}

template <typename T, int G>
static cudaError_t launch_step_g(const StepArgs &a, int RG, int threads, size_t smem)
{
    auto kern = step_kernel<T, 8, G>;
    if (G == 1) {
        kern<<<a.BH, threads, smem, a.stream>>>(a.C, a.n, a.m, (const T *)a.q, (const T *)a.k, (const T *)a.v,
                                                a.igate, a.fgate, (const T *)a.ogate, a.DHQK, a.DHV, RG, (T *)a.h);
        return cudaGetLastError();
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.BH * G);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = a.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = G;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a.C, a.n, a.m, (const T *)a.q, (const T *)a.k, (const T *)a.v, a.igate,
                              a.fgate, (const T *)a.ogate, a.DHQK, a.DHV, RG, (T *)a.h);
}

// Rows of one head are split over G CTAs when there are too few heads for two waves of CTAs.
static int step_cluster_size(int BH, int DHQK)
{
    int G = 1;
    while (G < 8 && (long long)BH * G < 2 * 148 && DHQK / (2 * G) >= 8 && DHQK % (2 * G) == 0) G *= 2;
    return G;
}

template <typename T>
static cudaError_t launch_step_t(const StepArgs &a)
{
    const int G = step_cluster_size(a.BH, a.DHQK);
    const int rows = a.DHQK / G;
    const int tx = a.DHV / 4;
    int RG = 512 / tx;
    if (RG < 1) RG = 1;
    if (RG > rows) RG = rows;
    const int threads = tx * RG;
    const size_t smem = sizeof(float) * (2 * (size_t)rows + (size_t)RG * a.DHV);
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
