// seqpar.cu -- the pieces of a sequence-parallel forward pass: a sequence split into R
// consecutive slices, one per rank.
//
// The state after a slice is a linear function of the state before it.  With the slice's
// total log forget decay g = sum_t logsigmoid(f~_t) and its final state (C_r, n_r, m_r) from
// the zero state (m_0 = 0), the state (C, n, m) before the slice becomes
//   m' = max(m + g, m_r),
//   C' = exp(m + g - m') C + exp(m_r - m') C_r,   n' likewise,
// which is the recurrence of "Recurrent Formulation (Inference Mode)" (xLSTM Guide: Extended
// LSTM Architecture & Matrix Memory) applied token by token: the earlier state decays by the
// product of the slice's forget gates and the slice adds its own stabilized contribution
// (C' e^{m'} = e^g C e^{m} + C_r e^{m_r}).  Rank r composes the summaries of slices 0 .. r-1
// from the zero state to get its start state; the per-rank summaries are all-gathered between
// the two kernels by the caller (NCCL).  The m of the composed state can be above the one the
// token-by-token recurrence reaches (the zero-start slices take m_0 = 0); C and n are then
// scaled to match, so h and the unstabilized state are the same.
#include "mlstm.h"
#include "common.cuh"
#include "mlstm_internal.h"

namespace mlstm {

// g[bh] = sum over the S tokens of logsigmoid(f~): one CTA per head.
__global__ void __launch_bounds__(256)
log_decay_sum_kernel(const float *__restrict__ fgate, int S, float *__restrict__ g)
{
    griddep_wait();
    griddep_launch_dependents();
    __shared__ float red[8];
    const int bh = blockIdx.x;
    const float *f = fgate + (size_t)bh * S;
    float acc = 0.f;
    for (int t = threadIdx.x; t < S; t += blockDim.x) acc += log_sigmoid(f[t]);
    acc = warp_sum(acc);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x < 32) {
        float x = threadIdx.x < 8 ? red[threadIdx.x] : 0.f;
        x = warp_sum(x);
        if (threadIdx.x == 0) g[bh] = x;
    }
}

// The start state of slice `rank` from the gathered slice summaries ([R][BH][...] each): every
// thread composes its four consecutive state elements over slices 0 .. rank-1, forming the
// per-slice factors itself (rank scalars per head).
__global__ void __launch_bounds__(256)
state_prefix_kernel(const float *__restrict__ Cp, const float *__restrict__ np, const float *__restrict__ mp,
                    const float *__restrict__ gp, int rank, int BH, int DHQK, int DHV, float *__restrict__ C0,
                    float *__restrict__ n0, float *__restrict__ m0)
{
    griddep_wait();
    griddep_launch_dependents();
    const int bh = blockIdx.y;
    const size_t nquad = (size_t)DHQK * DHV / 4;
    const size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t head = (size_t)DHQK * DHV;
    float4 c = make_float4(0.f, 0.f, 0.f, 0.f);
    float m = 0.f;
    for (int r = 0; r < rank; ++r) {
        const float gr = gp[(size_t)r * BH + bh], mr = mp[(size_t)r * BH + bh];
        const float mn = fmaxf(m + gr, mr);
        const float a = expf(m + gr - mn), b = expf(mr - mn);
        if (e < nquad) {
            const float4 x = *reinterpret_cast<const float4 *>(Cp + ((size_t)r * BH + bh) * head + 4 * e);
            c = make_float4(a * c.x + b * x.x, a * c.y + b * x.y, a * c.z + b * x.z, a * c.w + b * x.w);
        }
        m = mn;
    }
    if (e < nquad) *reinterpret_cast<float4 *>(C0 + (size_t)bh * head + 4 * e) = c;
    if (blockIdx.x == 0) {   // n and m of the head
        for (int d = threadIdx.x; d < DHQK; d += blockDim.x) {
            float nv = 0.f, mm = 0.f;
            for (int r = 0; r < rank; ++r) {
                const float gr = gp[(size_t)r * BH + bh], mr = mp[(size_t)r * BH + bh];
                const float mn = fmaxf(mm + gr, mr);
                nv = expf(mm + gr - mn) * nv + expf(mr - mn) * np[((size_t)r * BH + bh) * DHQK + d];
                mm = mn;
            }
            n0[(size_t)bh * DHQK + d] = nv;
        }
        if (threadIdx.x == 0) m0[bh] = m;
    }
}

}  // namespace mlstm

using namespace mlstm;

extern "C" {

mlstm_status mlstm_log_decay_sum(const float *fgate, int B, int NH, int S, float *g_out, void *stream)
{
    if (B < 0 || NH < 0 || S < 0) return MLSTM_ERR_INVALID_ARG;
    const long long BH = (long long)B * NH;
    if (BH == 0) return MLSTM_OK;
    if (BH > (1LL << 30)) return MLSTM_ERR_UNSUPPORTED;
    if (!g_out || (S > 0 && !fgate)) return MLSTM_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = launch_kernel(log_decay_sum_kernel, dim3((unsigned)BH), dim3(256), 0, st, 1, fgate, S, g_out);
    return e == cudaSuccess ? MLSTM_OK : MLSTM_ERR_CUDA;
}

mlstm_status mlstm_state_prefix(const float *C_parts, const float *n_parts, const float *m_parts,
                                const float *g_parts, int R, int rank, int B, int NH, int DHQK, int DHV,
                                float *C0, float *n0, float *m0, void *stream)
{
    if (B < 0 || NH < 0 || R < 1 || rank < 0 || rank >= R) return MLSTM_ERR_INVALID_ARG;
    if (DHQK < 8 || DHQK > 512 || DHQK % 8 || DHV < 8 || DHV > 512 || DHV % 8) return MLSTM_ERR_UNSUPPORTED;
    const long long BH = (long long)B * NH;
    if (BH == 0) return MLSTM_OK;
    if (BH > 65535) return MLSTM_ERR_UNSUPPORTED;
    if (!C0 || !n0 || !m0) return MLSTM_ERR_INVALID_ARG;
    if (rank > 0 && (!C_parts || !n_parts || !m_parts || !g_parts)) return MLSTM_ERR_INVALID_ARG;
    const uintptr_t mis = reinterpret_cast<uintptr_t>(C_parts) | reinterpret_cast<uintptr_t>(C0);
    if (mis & 15u) return MLSTM_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int nquad = DHQK * DHV / 4;
    cudaError_t e = launch_kernel(state_prefix_kernel, dim3((nquad + 255) / 256, (unsigned)BH), dim3(256), 0, st, 1,
                                  C_parts, n_parts, m_parts, g_parts, rank, (int)BH, DHQK, DHV, C0, n0, m0);
    return e == cudaSuccess ? MLSTM_OK : MLSTM_ERR_CUDA;
}

}  // extern "C"
