// bwd_simt.cu -- chunkwise backward pass of the mLSTM cell on CUDA cores (fp32 arithmetic).
//
// Gradients of a loss L = sum_t dh_t . h_t with respect to q, k, v, the gate pre-activations
// i~, f~ and the output gate o, for the forward pass from the zero state (the training form of
// the xLSTM Guide's "The Dual Formulation: How mLSTM Enables Parallel GPU Training", taken
// chunkwise as in "Exploit Chunkwise Hardware Kernels for Production Training").
//
// Per chunk c of L tokens, with the gate preprocessing of gate_prep.cu (chunk-local cumulative
// log decay a, chunk-local prefix maximum p_t of i~ - a, chunk-start stabilizer m_c, per-token
// stabilizer m_t = a_t + max(m_c, p_t)) and the chunk-start state (C_c, n_c) of the forward carry,
// the forward read-out is
//   S_ts = qh_t . k_s,  D_ts = exp(a_t - a_s + i~_s - m_t) = exp(x_s - max(m_c, p_t)) (s <= t,
//   x_s = i~_s - a_s: a_t cancels before rounding),  A = D * S,
//   sc_t = exp(a_t + m_c - m_t) = exp(m_c - max(m_c, p_t)),
//   num_t = sc_t C_c^T qh_t + sum_s A_ts v_s,  den_t = sc_t n_c . qh_t + sum_s A_ts,
//   N_t = max(|den_t|, exp(-m_t)),  h_t = o_t * num_t / N_t.
// The stabilizer carries no gradient (h does not depend on it), so with hh_t = num_t / N_t:
//   do_t = dh_t * hh_t,  g_t = o_t * dh_t / N_t (the gradient of num_t),
//   dden_t = -(g_t . hh_t) sign(den_t) where |den_t| > exp(-m_t), else 0,
//   dA_ts = g_t . v_s + dden_t,  dS = dA * D,
//   the chunk's read-out adds  dC_c += sum_t sc_t qh_t g_t^T,  dn_c += sum_t sc_t dden_t qh_t,
// and the state gradients run backwards over the chunks,
//   G_c = dC_c + exp(g_c + m_c - m_{c+1}) G_{c+1},  G_NC = 0  (likewise for n),
// with G_{c+1} the gradient of the state at the end of chunk c.  Then, with
// w_s = exp(g_c - a_s + i~_s - m_{c+1}) the weight of token s in that state,
//   dqh_t = sum_s dS_ts k_s + sc_t (C_c g_t + dden_t n_c),
//   dk_s  = sum_t dS_ts qh_t + w_s (G_{c+1} v_s + dn_{c+1}),
//   dv_s  = sum_t A_ts g_t + w_s G_{c+1}^T k_s,          dq = dqh / sqrt(DHQK).
// Gate gradients.  h depends on the gates through the weights D_ts of the pairs s <= t (the
// unstabilized read-out weighs v_s for query t by exp(i~_s + sum_{s < u <= t} log f_u)); with
// R_ts = dL/dD_ts D_ts (inside a chunk dA_ts A_ts; for tokens of different chunks the same quantity,
// reached through the chunk's state) the gradients are
//   dL/di~_s = sum_{t >= s} R_ts = k_s . dk_s,
//   dL/dlog f_j = sum_{s < j <= t} R_ts,  dL/df~_j = dL/dlog f_j * sigmoid(-f~_j).
// For j in chunk c the pairs that straddle j fall into four disjoint groups, each summed on its own:
//   F_j = E_c + sum_{t in c, t >= j} q_t . dq^inter_t + sum_{s in c, s < j} k_s . dk^inter_s + RECT_j,
// E_c = exp(g_c + m_c - m_{c+1}) (<G_{c+1}, C_c> + <dn_{c+1}, n_c>) the pairs that skip chunk c (the
// gradient of the state at its end against the decayed state at its start), dq^inter and dk^inter the
// inter-chunk terms alone (q_t . dq^inter_t sums R_ts over the s before t's chunk, k_s . dk^inter_s over
// the t after s's chunk) and RECT_j the pairs inside the chunk, summed from R in the dS kernel.  The
// shorter form sum_{t >= j} (q_t . dq_t - k_t . dk_t) equals F_j, but every pair at or after j cancels
// there, the pairs s = t (the largest terms) among them, and with strongly forgetting gates the
// result was lost to fp32 rounding.
//
// Kernels, in launch order (after the gate preprocessing and the forward's fp32 carry that stores
// the chunk-start states): bwd_scores_kernel (A, den, N per chunk), bwd_num_kernel (the read-out
// numerator, g and do per chunk and 64 value columns), bwd_ds_kernel (dden, dS, dn of the read-out, RECT),
// bwd_dc_kernel (dC of the read-out per 64 x 64 state tile), bwd_state_scan_kernel (the reverse scan
// of the state gradients), bwd_skip_kernel (E_c), bwd_grad_kernel (dq, dk, dv per chunk and 64
// columns) and bwd_gate_kernel.  The per-chunk products run as 64 x 64 output tiles on the CUDA cores in fp32.
#include "bwd_tc.h"
#include "common.cuh"
#include "mlstm_internal.h"

namespace mlstm {
namespace bwd {

constexpr int NT = 256;   // threads of the chunk kernels

struct Params {
    int S, L, NC, DK, DV, NTK;
    const void *q, *k, *v, *o, *dh;
    const float *ig, *fg;
    const float *A, *P, *MC, *G;     // gate preprocessing
    float *CS, *NS;                  // chunk-start states [BH][NC][DK][DV], [BH][NC][DK]
    float *GS, *GN;                  // read-out state gradients, then chunk-end gradients (same layout)
    float *Gt;                       // g = o dh / N [BH][S][DV]
    float *DD;                       // dden [BH][S]
    float *DEN, *NRM;                // den and N = max(|den|, exp(-m)) [BH][S]
    float *DOTP;                     // partial row sums of g . hh per 64 value columns [BH][S][NJT]
    int NJT;                         // ceil(DV / 64)
    float *P2, *AI;                  // dS and A per chunk [BH][NC][L][L]
    // per 32 columns of dk: partial q . dq^inter, k . dk and k . dk^inter [BH][S][NTK] (^inter: the
    // inter-chunk term alone), and RECT [BH][S], the sum of dA_ts A_ts over the pairs s < j <= t of
    // token j's chunk (written by the dS kernels)
    float *QD, *KD, *KI, *RECT;
    float *EP;                       // partial sums of E_c [BH][NC][NEP] (the pairs that skip chunk c)
    int NEP;
    void *dq, *dk, *dv, *dog;
    float *dig, *dfg;
};

// Shared-memory floats of bwd_chunk_kernel and bwd_grad_kernel for chunk length L.

// Per-token gate terms of chunk c, in forms where the chunk-local cumulative log decay a_t
// cancels before rounding (m_t = a_t + max(m_c, p_t), so a_t - a_s + i~_s - m_t = x_s - mx_t):
//   xs[s] = i~_s - a_s (-inf past the end), mx[t] = max(m_c, p_t), sc[t] = exp(m_c - mx_t),
//   fl[t] = exp(-m_t) (the denominator's floor).
__device__ __forceinline__ void chunk_rows(const Params &p, int bh, int c, int t0, int len, float *xs, float *mx,
                                           float *fl, float *sc)
{
    const float mc = p.MC[(size_t)bh * (p.NC + 1) + c];
    for (int t = threadIdx.x; t < p.L; t += blockDim.x) {
        const bool ok = t < len;
        const size_t g = (size_t)bh * p.S + t0 + t;
        const float a = ok ? p.A[g] : 0.f;
        const float m = ok ? fmaxf(mc, p.P[g]) : 0.f;
        xs[t] = ok ? p.ig[g] - a : -INFINITY;
        mx[t] = m;
        fl[t] = ok ? expf(-(a + m)) : 1.f;
        sc[t] = ok ? expf(mc - m) : 0.f;
    }
}

// ---------------------------------------------------------------- per chunk: read-out recompute
// grid (BH, NC), NT threads.  Recomputes A, den, N and num of the chunk, writes do, g, dden, dS,
// A and the read-out's state gradients (dC_c, dn_c).
// ---------------------------------------------------------------- 64 x 64 tiles of the chunk products
// The per-chunk products (S = qh K^T, the read-out numerator, g V^T, the read-out's state gradient)
// run as tiles of 64 x 64 outputs per CTA of 256 threads, a 4 x 4 block per thread, the reduction
// in steps of 32 staged in shared memory k-major (As[k][m], Bs[k][n], rows padded to 68 floats so
// that a thread reads its four rows or columns with one 16-byte load).
constexpr int GM = 64, GK = 32, GSTR = 68;
static_assert(NT == 256, "the 64 x 64 tiles take 16 x 16 threads");

__device__ __forceinline__ void tile_mma(const float *As, const float *Bs, float (&acc)[4][4])
{
    const int tm = threadIdx.x >> 4, tn = threadIdx.x & 15;
#pragma unroll 8
    for (int k = 0; k < GK; ++k) {
        const float4 a = *reinterpret_cast<const float4 *>(As + k * GSTR + 4 * tm);
        const float4 b = *reinterpret_cast<const float4 *>(Bs + k * GSTR + 4 * tn);
        const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
}

// Runs `nsteps` reduction steps of 32 into acc.  A thread stages 8 elements of each tile per step:
// get(st, e, a, b) reads element e (0..2047) of step st's A and B tiles from global memory and
// put(st, e, a, b) stores them into As and Bs.  The next step's reads are issued before this step's
// products, so their latency overlaps the products.
template <typename Get, typename Put>
__device__ __forceinline__ void tile_gemm(int nsteps, Get get, Put put, const float *As, const float *Bs,
                                          float (&acc)[4][4])
{
    float ra[8], rb[8];
    if (nsteps > 0) {
#pragma unroll
        for (int u = 0; u < 8; ++u) get(0, threadIdx.x + u * NT, ra[u], rb[u]);
    }
    for (int st = 0; st < nsteps; ++st) {
        __syncthreads();   // the previous step's readers are done
#pragma unroll
        for (int u = 0; u < 8; ++u) put(st, threadIdx.x + u * NT, ra[u], rb[u]);
        __syncthreads();
        if (st + 1 < nsteps) {
#pragma unroll
            for (int u = 0; u < 8; ++u) get(st + 1, threadIdx.x + u * NT, ra[u], rb[u]);
        }
        tile_mma(As, Bs, acc);
    }
}

// Sum over the 16 threads that share a tile row block (tn = lane & 15).
__device__ __forceinline__ float sum16(float v)
{
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// ---------------------------------------------------------------- per chunk: scores and denominators
// grid (BH, NC): A = D * S with S = qh K^T on the causal triangle (-> AI), den_t = rowsum(A)_t +
// sc_t n_c . qh_t and N_t = max(|den_t|, exp(-m_t)) (-> DEN, NRM).
template <typename T>
__global__ void __launch_bounds__(NT) bwd_scores_kernel(Params p)
{
    griddep_wait();
    griddep_launch_dependents();
    __shared__ __align__(16) float As[GK * GSTR], Bs[GK * GSTR];
    __shared__ float xs_[128], mx[128], fl[128], sc[128], rsum[128];
    const int L = p.L, DK = p.DK;
    const int bh = blockIdx.x, c = blockIdx.y;
    const int t0 = c * L, len = min(L, p.S - t0);
    const int tid = threadIdx.x, tm = tid >> 4, tn = tid & 15, lane = tid & 31, warp = tid >> 5;
    const float scale = rsqrtf((float)DK);
    const T *qb = static_cast<const T *>(p.q) + ((size_t)bh * p.S + t0) * DK;
    const T *kb = static_cast<const T *>(p.k) + ((size_t)bh * p.S + t0) * DK;
    const float *nc = p.NS + ((size_t)bh * p.NC + c) * DK;
    float *AIg = p.AI + ((size_t)bh * p.NC + c) * L * L;

    chunk_rows(p, bh, c, t0, len, xs_, mx, fl, sc);
    for (int t = tid; t < L; t += NT) rsum[t] = 0.f;
    const int nmt = (L + GM - 1) / GM;
    for (int mt = 0; mt < nmt; ++mt)
        for (int nt = 0; nt <= mt; ++nt) {   // tiles on or below the diagonal
            float acc[4][4] = {};
            for (int d0 = 0; d0 < DK; d0 += GK) {   // (a small product: staged without prefetch)
                __syncthreads();
                for (int e = tid; e < GK * GM; e += NT) {
                    const int m = e >> 5, k = e & 31;   // consecutive threads: consecutive d
                    const int ta = mt * GM + m, tb = nt * GM + m;
                    As[k * GSTR + m] = (ta < len && d0 + k < DK) ? to_f32(qb[(size_t)ta * DK + d0 + k]) * scale : 0.f;
                    Bs[k * GSTR + m] = (tb < len && d0 + k < DK) ? to_f32(kb[(size_t)tb * DK + d0 + k]) : 0.f;
                }
                __syncthreads();
                tile_mma(As, Bs, acc);
            }
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int t = mt * GM + 4 * tm + a;
                float part = 0.f;
#pragma unroll
                for (int b2 = 0; b2 < 4; ++b2) {
                    const int s2 = nt * GM + 4 * tn + b2;
                    float av = 0.f;
                    if (s2 <= t && t < len) av = acc[a][b2] * expf(xs_[s2] - mx[t]);
                    if (t < L && s2 < L) AIg[(size_t)t * L + s2] = av;
                    part += av;
                }
                part = sum16(part);
                if (tn == 0 && t < L) atomicAdd(&rsum[t], part);
            }
            // tiles above the diagonal (s > t everywhere) hold zeros
            if (nt < mt) {
                for (int e = tid; e < GM * GM; e += NT) {
                    const int t = nt * GM + e / GM, s2 = mt * GM + e % GM;
                    if (t < L && s2 < L) AIg[(size_t)t * L + s2] = 0.f;
                }
            }
        }
    __syncthreads();
    // den and N: a warp per row, lanes over DK
    for (int t = warp; t < L; t += NT / 32) {
        float qn = 0.f;
        if (t < len)
            for (int d = lane; d < DK; d += 32) qn = fmaf(nc[d], to_f32(qb[(size_t)t * DK + d]), qn);
        qn = warp_sum(qn);
        if (lane == 0 && t < len) {
            const float den = rsum[t] + qn * scale * sc[t];
            p.DEN[(size_t)bh * p.S + t0 + t] = den;
            p.NRM[(size_t)bh * p.S + t0 + t] = fmaxf(fabsf(den), fl[t]);
        }
    }
}

// ---------------------------------------------------------------- per chunk and 64 value columns: the read-out
// grid (BH, NC, NJT): num = sc qh C_c + A V (one product over [sc qh | A] and [C_c ; V], K = DK + L),
// hh = num / N, do = dh hh, g = o dh / N (-> Gt) and the partial row sums of g . hh (-> DOTP).
template <typename T>
__global__ void __launch_bounds__(NT) bwd_num_kernel(Params p)
{
    griddep_wait();
    griddep_launch_dependents();
    __shared__ __align__(16) float As[GK * GSTR], Bs[GK * GSTR];
    __shared__ float sc[128], xs_[128], mx[128], fl[128];
    const int L = p.L, DK = p.DK, DV = p.DV;
    const int bh = blockIdx.x, c = blockIdx.y, jt = blockIdx.z, j0 = jt * GM;
    const int t0 = c * L, len = min(L, p.S - t0);
    const int tid = threadIdx.x, tm = tid >> 4, tn = tid & 15;
    const float scale = rsqrtf((float)DK);
    const T *qb = static_cast<const T *>(p.q) + ((size_t)bh * p.S + t0) * DK;
    const T *vb = static_cast<const T *>(p.v) + ((size_t)bh * p.S + t0) * DV;
    const T *ob = p.o ? static_cast<const T *>(p.o) + ((size_t)bh * p.S + t0) * DV : nullptr;
    const T *dhb = static_cast<const T *>(p.dh) + ((size_t)bh * p.S + t0) * DV;
    T *dob = p.dog ? static_cast<T *>(p.dog) + ((size_t)bh * p.S + t0) * DV : nullptr;
    float *gtb = p.Gt + ((size_t)bh * p.S + t0) * DV;
    const float *Cc = p.CS + ((size_t)bh * p.NC + c) * DK * DV;
    const float *AIg = p.AI + ((size_t)bh * p.NC + c) * L * L;
    const float *nrm = p.NRM + (size_t)bh * p.S + t0;

    chunk_rows(p, bh, c, t0, len, xs_, mx, fl, sc);
    __syncthreads();   // sc is read by the tile loads
    const int nmt = (L + GM - 1) / GM;
    for (int mt = 0; mt < nmt; ++mt) {
        float acc[4][4] = {};
        for (int d0 = 0; d0 < DK; d0 += GK) {   // sc qh C_c
            __syncthreads();
            for (int e = tid; e < GK * GM; e += NT) {
                const int m = e >> 5, k = e & 31;
                const int t = mt * GM + m;
                As[k * GSTR + m] = (t < len && d0 + k < DK) ? to_f32(qb[(size_t)t * DK + d0 + k]) * scale * sc[t] : 0.f;
                const int kk = e >> 6, n = e & 63;   // consecutive threads: consecutive value columns
                Bs[kk * GSTR + n] = (d0 + kk < DK && j0 + n < DV) ? Cc[(size_t)(d0 + kk) * DV + j0 + n] : 0.f;
            }
            __syncthreads();
            tile_mma(As, Bs, acc);
        }
        for (int s0 = 0; s0 < L; s0 += GK) {    // A V (A is zero past the end and above the diagonal)
            __syncthreads();
            for (int e = tid; e < GK * GM; e += NT) {
                const int m = e >> 5, k = e & 31;
                const int t = mt * GM + m;
                As[k * GSTR + m] = (t < L && s0 + k < L) ? AIg[(size_t)t * L + s0 + k] : 0.f;
                const int kk = e >> 6, n = e & 63;
                Bs[kk * GSTR + n] = (s0 + kk < len && j0 + n < DV) ? to_f32(vb[(size_t)(s0 + kk) * DV + j0 + n]) : 0.f;
            }
            __syncthreads();
            tile_mma(As, Bs, acc);
        }
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const int t = mt * GM + 4 * tm + a;
            float part = 0.f;
            if (t < len) {
                const float N = nrm[t];
#pragma unroll
                for (int b2 = 0; b2 < 4; ++b2) {
                    const int j = j0 + 4 * tn + b2;
                    if (j < DV) {
                        const size_t off = (size_t)t * DV + j;
                        const float hh = acc[a][b2] / N;
                        const float dhv = to_f32(dhb[off]);
                        const float ov = ob ? to_f32(ob[off]) : 1.f;
                        if (dob) dob[off] = from_f32<T>(dhv * hh);
                        const float g = ov * dhv / N;
                        gtb[off] = g;
                        part = fmaf(g, hh, part);
                    }
                }
            }
            part = sum16(part);
            if (tn == 0 && t < len) p.DOTP[((size_t)bh * p.S + t0 + t) * p.NJT + jt] = part;
        }
    }
}

// ---------------------------------------------------------------- per chunk: dden and dS
// grid (BH, NC): dden_t = -(g_t . hh_t) sign(den_t) where the floor does not bind (-> DD),
// dS = (g V^T + dden) * D on the causal triangle (-> P2), and the read-out's normalizer gradient
// dn_c = sum_t sc_t dden_t qh_t (-> GN).
template <typename T>
__global__ void __launch_bounds__(NT) bwd_ds_kernel(Params p)
{
    griddep_wait();
    griddep_launch_dependents();
    __shared__ __align__(16) float As[GK * GSTR], Bs[GK * GSTR];
    __shared__ float xs_[128], mx[128], fl[128], sc[128], dd[128];
    __shared__ float rowl[128], colb[128], cpart[NT / 32][GM];   // sums of R by row and column
    const int L = p.L, DK = p.DK, DV = p.DV;
    const int bh = blockIdx.x, c = blockIdx.y;
    const int t0 = c * L, len = min(L, p.S - t0);
    const int tid = threadIdx.x, tm = tid >> 4, tn = tid & 15;
    const float scale = rsqrtf((float)DK);
    const T *qb = static_cast<const T *>(p.q) + ((size_t)bh * p.S + t0) * DK;
    const T *vb = static_cast<const T *>(p.v) + ((size_t)bh * p.S + t0) * DV;
    const float *gtb = p.Gt + ((size_t)bh * p.S + t0) * DV;
    float *P2g = p.P2 + ((size_t)bh * p.NC + c) * L * L;
    const float *AIg = p.AI + ((size_t)bh * p.NC + c) * L * L;

    chunk_rows(p, bh, c, t0, len, xs_, mx, fl, sc);
    for (int t = tid; t < 128; t += NT) rowl[t] = colb[t] = 0.f;
    for (int t = tid; t < L; t += NT) {
        float v = 0.f;
        if (t < len) {
            const size_t r = (size_t)bh * p.S + t0 + t;
            float dot = 0.f;
            for (int u = 0; u < p.NJT; ++u) dot += p.DOTP[r * p.NJT + u];
            const float den = p.DEN[r];
            if (fabsf(den) > fl[t]) v = -dot * copysignf(1.f, den);
            p.DD[r] = v;
        }
        dd[t] = v;
    }
    const int nmt = (L + GM - 1) / GM;
    for (int mt = 0; mt < nmt; ++mt)
        for (int nt = 0; nt < nmt; ++nt) {
            if (nt > mt) {   // above the diagonal: zeros
                for (int e = tid; e < GM * GM; e += NT) {
                    const int t = mt * GM + e / GM, s2 = nt * GM + e % GM;
                    if (t < L && s2 < L) P2g[(size_t)t * L + s2] = 0.f;
                }
                continue;
            }
            float acc[4][4] = {};
            tile_gemm((DV + GK - 1) / GK,   // g V^T
                      [&](int st, int e, float &av, float &bv) {
                          const int m = e >> 5, k = e & 31, j = st * GK + k;
                          const int ta = mt * GM + m, tb = nt * GM + m;
                          av = (ta < len && j < DV) ? gtb[(size_t)ta * DV + j] : 0.f;
                          bv = (tb < len && j < DV) ? to_f32(vb[(size_t)tb * DV + j]) : 0.f;
                      },
                      [&](int, int e, float av, float bv) {
                          As[(e & 31) * GSTR + (e >> 5)] = av;
                          Bs[(e & 31) * GSTR + (e >> 5)] = bv;
                      },
                      As, Bs, acc);
            // dS, and R_ts = dA_ts A_ts of the pairs s < t (the derivative of the loss by the log decay
            // between them): its sums along the rows (left of the diagonal) and columns (below it)
            float cp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int t = mt * GM + 4 * tm + a;
                float rp = 0.f;
#pragma unroll
                for (int b2 = 0; b2 < 4; ++b2) {
                    const int s2 = nt * GM + 4 * tn + b2;
                    float pv = 0.f;
                    if (s2 <= t && t < len) {
                        const float da = acc[a][b2] + dd[t];
                        pv = da * expf(xs_[s2] - mx[t]);
                        if (s2 < t) {
                            const float rv = da * AIg[(size_t)t * L + s2];
                            rp += rv;
                            cp[b2] += rv;
                        }
                    }
                    if (t < L && s2 < L) P2g[(size_t)t * L + s2] = pv;
                }
                rp = sum16(rp);
                if (tn == 0 && t < L) rowl[t] += rp;   // one thread per row: tiles in order
            }
#pragma unroll
            for (int b2 = 0; b2 < 4; ++b2) {
                cp[b2] += __shfl_xor_sync(0xffffffffu, cp[b2], 16);
                if (tm % 2 == 0) cpart[tid >> 5][4 * tn + b2] = cp[b2];
            }
            __syncthreads();
            if (tid < GM && nt * GM + tid < L) {
                float v = 0.f;
                for (int w2 = 0; w2 < NT / 32; ++w2) v += cpart[w2][tid];
                colb[nt * GM + tid] += v;
            }
        }
    __syncthreads();
    if (tid < 32) {   // RECT_j = sum_{s < j} (colb_s - rowl_s) over the chunk (a warp scan in fp64)
        const int per = (L + 31) / 32, sb = tid * per;
        double loc = 0.0;
        for (int u = sb; u < min(sb + per, len); ++u) loc += (double)colb[u] - (double)rowl[u];
        double inc = loc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double y = __shfl_up_sync(0xffffffffu, inc, o);
            if (tid >= o) inc += y;
        }
        double run = inc - loc;
        for (int u = sb; u < min(sb + per, len); ++u) {
            p.RECT[(size_t)bh * p.S + t0 + u] = (float)run;
            run += (double)colb[u] - (double)rowl[u];
        }
    }
    float *GNc = p.GN + ((size_t)bh * p.NC + c) * DK;
    for (int i = tid; i < DK; i += NT) {
        float a2 = 0.f;
        for (int t = 0; t < len; ++t) a2 = fmaf(sc[t] * dd[t], to_f32(qb[(size_t)t * DK + i]) * scale, a2);
        GNc[i] = a2;
    }
}

// ---------------------------------------------------------------- per chunk and 64 x 64 state tile: dC of the read-out
// grid (BH NC, ceil(DK / 64), NJT): GS[i][j] = sum_t sc_t qh_t[i] g_t[j].
template <typename T>
__global__ void __launch_bounds__(NT) bwd_dc_kernel(Params p)
{
    griddep_wait();
    griddep_launch_dependents();
    __shared__ __align__(16) float As[GK * GSTR], Bs[GK * GSTR];
    __shared__ float xs_[128], mx[128], fl[128], sc[128];
    const int L = p.L, DK = p.DK, DV = p.DV;
    const int bh = blockIdx.x / p.NC, c = blockIdx.x % p.NC;
    const int i0 = blockIdx.y * GM, j0 = blockIdx.z * GM;
    const int t0 = c * L, len = min(L, p.S - t0);
    const int tid = threadIdx.x, tm = tid >> 4, tn = tid & 15;
    const float scale = rsqrtf((float)DK);
    const T *qb = static_cast<const T *>(p.q) + ((size_t)bh * p.S + t0) * DK;
    const float *gtb = p.Gt + ((size_t)bh * p.S + t0) * DV;
    float *GSc = p.GS + ((size_t)bh * p.NC + c) * DK * DV;

    chunk_rows(p, bh, c, t0, len, xs_, mx, fl, sc);
    __syncthreads();   // sc is read by the tile loads
    float acc[4][4] = {};
    for (int k0 = 0; k0 < L; k0 += GK) {
        __syncthreads();
        for (int e = tid; e < GK * GM; e += NT) {
            const int k = e >> 6, m = e & 63;   // consecutive threads: consecutive columns
            const int t = k0 + k;
            As[k * GSTR + m] = (t < len && i0 + m < DK) ? to_f32(qb[(size_t)t * DK + i0 + m]) * scale * sc[t] : 0.f;
            Bs[k * GSTR + m] = (t < len && j0 + m < DV) ? gtb[(size_t)t * DV + j0 + m] : 0.f;
        }
        __syncthreads();
        tile_mma(As, Bs, acc);
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int i = i0 + 4 * tm + a;
        if (i < DK) {
#pragma unroll
            for (int b2 = 0; b2 < 4; ++b2) {
                const int j = j0 + 4 * tn + b2;
                if (j < DV) GSc[(size_t)i * DV + j] = acc[a][b2];
            }
        }
    }
}

// ---------------------------------------------------------------- reverse scan of the state gradients
// grid (ceil(DK * DV / 1024), BH): each thread four state elements; G_c = dC_c + decay_c G_{c+1}, the
// slot of chunk c then holds G_{c+1} (the gradient of the state at the chunk's end).
__global__ void __launch_bounds__(256) bwd_state_scan_kernel(Params p)
{
    griddep_wait();
    griddep_launch_dependents();
    constexpr int SCAN_CHUNKS = 256;                   // decay factors staged per pass
    __shared__ float decay[SCAN_CHUNKS];
    const int bh = blockIdx.y;
    const float *MCb = p.MC + (size_t)bh * (p.NC + 1);
    const float *Gb = p.G + (size_t)bh * p.NC;
    const size_t nstate = (size_t)p.DK * p.DV;
    const size_t nq = nstate / 4;                      // DK DV is a multiple of 4 (DK % 8 == 0)
    const size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x;   // a quad of state elements
    float4 *slot = reinterpret_cast<float4 *>(p.GS + (size_t)bh * p.NC * nstate) + e;
    float4 G = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c0 = p.NC; c0 > 0; c0 -= SCAN_CHUNKS) {
        // the decay factors of chunks cb .. c0 - 1, once per CTA
        const int cb = max(0, c0 - SCAN_CHUNKS);
        __syncthreads();
        for (int c = cb + threadIdx.x; c < c0; c += blockDim.x) decay[c - cb] = expf(Gb[c] + MCb[c] - MCb[c + 1]);
        __syncthreads();
        if (e < nq) {
            constexpr int BATCH = 8;
            for (int c1 = c0; c1 > cb; c1 -= BATCH) {   // chunks c1 - 1 down to c1 - BATCH, loads first
                float4 d[BATCH];
#pragma unroll
                for (int u = 0; u < BATCH; ++u)
                    if (c1 - 1 - u >= cb) d[u] = __ldcg(slot + (size_t)(c1 - 1 - u) * nq);
#pragma unroll
                for (int u = 0; u < BATCH; ++u) {
                    const int c = c1 - 1 - u;
                    if (c >= cb) {
                        slot[(size_t)c * nq] = G;
                        const float f = decay[c - cb];
                        G = make_float4(d[u].x + f * G.x, d[u].y + f * G.y, d[u].z + f * G.z, d[u].w + f * G.w);
                    }
                }
            }
        }
    }
    if (blockIdx.x == 0) {
        for (int i = threadIdx.x; i < p.DK; i += blockDim.x) {
            float *slot = p.GN + (size_t)bh * p.NC * p.DK + i;
            float G = 0.f;
            for (int c = p.NC - 1; c >= 0; --c) {
                const float d = slot[(size_t)c * p.DK];
                slot[(size_t)c * p.DK] = G;
                G = d + expf(Gb[c] + MCb[c] - MCb[c + 1]) * G;
            }
        }
    }
}

// ---------------------------------------------------------------- per chunk and 64 columns: dq, dk, dv
// grid (BH, NC, tiles): KIND 0 computes dq over ceil(DK / 64) tiles, KIND 1 dk over as many, KIND 2
// dv over NJT tiles, each a product of 64 x 64 outputs with the chunk-local and the inter-chunk
// terms stacked along the reduction:
//   dqh = [dS | sc g] [K ; C_c^T] + sc dden n_c,          K = L + DV,
//   dk  = [dS^T | w v] [qh ; G_end^T] + w dn_end,         K = L + DV,
//   dv  = [A^T | w k] [g ; G_end],                        K = L + DK,
// with w_s = exp(g_c - a_s + i~_s - m_{c+1}) the weight of token s in the state at the chunk's end.
// The dq and dk tiles also leave, for the gate gradients, the partial row sums of their two 32-column
// halves: q . dq^inter (QD), k . dk^inter (KI) of the inter-chunk term alone, and k . dk (KD).
template <typename T, int KIND>
__global__ void __launch_bounds__(NT, 2) bwd_grad_kernel(Params p)
{
    griddep_wait();
    griddep_launch_dependents();
    __shared__ __align__(16) float As[GK * GSTR], Bs[GK * GSTR];
    __shared__ float xs_[128], mx[128], fl[128], sc[128], wt[128], dd[128];
    const int L = p.L, DK = p.DK, DV = p.DV;
    const int bh = blockIdx.x, c = blockIdx.y, z = blockIdx.z;
    const int t0 = c * L, len = min(L, p.S - t0);
    const int tid = threadIdx.x, tm = tid >> 4, tn = tid & 15;
    const float scale = rsqrtf((float)DK);
    const T *qb = static_cast<const T *>(p.q) + ((size_t)bh * p.S + t0) * DK;
    const T *kb = static_cast<const T *>(p.k) + ((size_t)bh * p.S + t0) * DK;
    const T *vb = static_cast<const T *>(p.v) + ((size_t)bh * p.S + t0) * DV;
    const float *gtb = p.Gt + ((size_t)bh * p.S + t0) * DV;
    const float *Cc = p.CS + ((size_t)bh * p.NC + c) * DK * DV;
    const float *nc = p.NS + ((size_t)bh * p.NC + c) * DK;
    const float *Ge = p.GS + ((size_t)bh * p.NC + c) * DK * DV;   // gradient of the state at the chunk's end
    const float *ge = p.GN + ((size_t)bh * p.NC + c) * DK;
    const float *P2g = p.P2 + ((size_t)bh * p.NC + c) * L * L;
    const float *AIg = p.AI + ((size_t)bh * p.NC + c) * L * L;

    chunk_rows(p, bh, c, t0, len, xs_, mx, fl, sc);
    {
        const float gm = p.G[(size_t)bh * p.NC + c] - p.MC[(size_t)bh * (p.NC + 1) + c + 1];
        for (int t = tid; t < L; t += NT) {
            wt[t] = t < len ? expf(xs_[t] + gm) : 0.f;
            dd[t] = t < len ? p.DD[(size_t)bh * p.S + t0 + t] : 0.f;
        }
    }
    __syncthreads();   // sc, wt and dd are read by the tile loads
    constexpr int kind = KIND;                 // dq, dk, dv
    const int c0 = z * GM;                     // first output column
    const int NC_ = kind == 2 ? DV : DK;       // output columns
    const int nmt = (L + GM - 1) / GM;
    for (int mt = 0; mt < nmt; ++mt) {
        float acc[4][4] = {};
        // steps 0 .. nloc - 1: the chunk-local term (reduction over the chunk's tokens); from nloc: the
        // inter-chunk term (over DV for dq and dk, over DK for dv)
        const int KI = kind == 2 ? DK : DV;
        const int nloc = (L + GK - 1) / GK, ninter = (KI + GK - 1) / GK;
        auto get = [&](int st, int e, float &av, float &bv) {
            if (st < nloc) {
                const int k0 = st * GK;
                if (kind == 0) {          // As[u][t] = dS[t][u]
                    const int m = e >> 5, k = e & 31, t = mt * GM + m;
                    av = (t < L && k0 + k < L) ? P2g[(size_t)t * L + k0 + k] : 0.f;
                } else {                  // As[u][s] = dS[u][s] or A[u][s]
                    const int k = e >> 6, m = e & 63, s2 = mt * GM + m;
                    av = (s2 < L && k0 + k < L) ? (kind == 1 ? P2g : AIg)[(size_t)(k0 + k) * L + s2] : 0.f;
                }
                const int kk = e >> 6, n = e & 63, u = k0 + kk;   // Bs[u][col]: k, qh or g
                bv = 0.f;
                if (u < len && c0 + n < NC_) {
                    if (kind == 0) bv = to_f32(kb[(size_t)u * DK + c0 + n]);
                    else if (kind == 1) bv = to_f32(qb[(size_t)u * DK + c0 + n]) * scale;
                    else bv = gtb[(size_t)u * DV + c0 + n];
                }
            } else {
                const int k0 = (st - nloc) * GK;
                const int m = e >> 5, k = e & 31, r = mt * GM + m;   // row r of the output tile
                av = 0.f;
                if (r < len && k0 + k < KI) {
                    if (kind == 0) av = sc[r] * gtb[(size_t)r * DV + k0 + k];
                    else if (kind == 1) av = wt[r] * to_f32(vb[(size_t)r * DV + k0 + k]);
                    else av = wt[r] * to_f32(kb[(size_t)r * DK + k0 + k]);
                }
                if (kind == 2) {           // Bs[i][j] = G_end[i][j]
                    const int kk = e >> 6, n = e & 63;
                    bv = (k0 + kk < DK && c0 + n < DV) ? Ge[(size_t)(k0 + kk) * DV + c0 + n] : 0.f;
                } else {                   // Bs[j][i] = C_c[i][j] or G_end[i][j]
                    const int n = e >> 5, kk = e & 31;
                    bv = (c0 + n < DK && k0 + kk < DV) ? (kind == 0 ? Cc : Ge)[(size_t)(c0 + n) * DV + k0 + kk] : 0.f;
                }
            }
        };
        auto put = [&](int st, int e, float av, float bv) {
            if (st < nloc) {
                if (kind == 0) As[(e & 31) * GSTR + (e >> 5)] = av;
                else As[(e >> 6) * GSTR + (e & 63)] = av;
                Bs[(e >> 6) * GSTR + (e & 63)] = bv;
            } else {
                As[(e & 31) * GSTR + (e >> 5)] = av;
                if (kind == 2) Bs[(e >> 6) * GSTR + (e & 63)] = bv;
                else Bs[(e & 31) * GSTR + (e >> 5)] = bv;
            }
        };
        // the inter-chunk term first: for dq and dk its own row sums q . dq^inter, k . dk^inter (the
        // pairs of tokens in different chunks, for the forget-gate gradients) are taken before the
        // chunk-local term joins the accumulator
        tile_gemm(ninter, [&](int st, int e, float &av, float &bv) { get(nloc + st, e, av, bv); },
                  [&](int st, int e, float av, float bv) { put(nloc + st, e, av, bv); }, As, Bs, acc);
        auto row_parts = [&](int a, float part, float *dst) {   // the tile's two 32-column halves
#pragma unroll
            for (int o = 4; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
            const int r = mt * GM + 4 * tm + a, half = (c0 >> 5) + (tn >> 3);
            if ((tn & 7) == 0 && r < len && half * 32 < DK) dst[((size_t)bh * p.S + t0 + r) * p.NTK + half] = part;
        };
        if (kind < 2) {
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int r = mt * GM + 4 * tm + a;
                float part = 0.f;
#pragma unroll
                for (int b2 = 0; b2 < 4; ++b2) {
                    const int col = c0 + 4 * tn + b2;
                    if (r < len && col < NC_) {
                        if (kind == 0)
                            part = fmaf(to_f32(qb[(size_t)r * DK + col]) * scale, acc[a][b2] + sc[r] * dd[r] * nc[col], part);
                        else
                            part = fmaf(to_f32(kb[(size_t)r * DK + col]), acc[a][b2] + wt[r] * ge[col], part);
                    }
                }
                row_parts(a, part, kind == 0 ? p.QD : p.KI);
            }
        }
        tile_gemm(nloc, get, put, As, Bs, acc);
        // epilogue
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const int r = mt * GM + 4 * tm + a;
            float part = 0.f;
            if (r < len) {
#pragma unroll
                for (int b2 = 0; b2 < 4; ++b2) {
                    const int col = c0 + 4 * tn + b2;
                    if (col < NC_) {
                        if (kind == 0) {
                            const float dqh = acc[a][b2] + sc[r] * dd[r] * nc[col];
                            static_cast<T *>(p.dq)[((size_t)bh * p.S + t0 + r) * DK + col] = from_f32<T>(dqh * scale);
                        } else if (kind == 1) {
                            const float dkv = acc[a][b2] + wt[r] * ge[col];
                            static_cast<T *>(p.dk)[((size_t)bh * p.S + t0 + r) * DK + col] = from_f32<T>(dkv);
                            part = fmaf(to_f32(kb[(size_t)r * DK + col]), dkv, part);
                        } else {
                            static_cast<T *>(p.dv)[((size_t)bh * p.S + t0 + r) * DV + col] = from_f32<T>(acc[a][b2]);
                        }
                    }
                }
            }
            if (kind == 1) row_parts(a, part, p.KD);   // k . dk (the input-gate gradient)
        }
    }
}

// ---------------------------------------------------------------- gate gradients
// grid (BH, ceil(NC / 8)), 256 threads, a warp per chunk (a lane takes L / 32 consecutive tokens):
// dL/di~_t = k_t . dk_t and dL/df~_j = sigmoid(-f~_j) F_j with, for j in chunk c,
//   F_j = E_c + sum_{t in c, t >= j} q_t . dq^inter_t + sum_{s in c, s < j} k_s . dk^inter_s + RECT_j,
// the four disjoint sets of the pairs s < j <= t, summed in fp64 (E_c from its NEP partial sums).
constexpr int GT = 256;

__device__ __forceinline__ double warp_scan_incl(double v, int lane)   // sum over lanes <= lane
{
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += y;
    }
    return v;
}

__global__ void __launch_bounds__(GT) bwd_gate_kernel(Params p)
{
    griddep_wait();
    griddep_launch_dependents();
    const int bh = blockIdx.x, lane = threadIdx.x & 31;
    const int c = blockIdx.y * (GT / 32) + (threadIdx.x >> 5);
    if (c >= p.NC) return;                       // (whole warps)
    const int t0 = c * p.L, len = min(p.L, p.S - t0);
    constexpr int MAXPER = 4;                    // chunk <= 128
    const int per = (p.L + 31) / 32;
    double e = 0.0;                              // E_c: the pairs that skip the chunk
    for (int z = lane; z < p.NEP; z += 32) e += (double)p.EP[((size_t)bh * p.NC + c) * p.NEP + z];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) e += __shfl_xor_sync(0xffffffffu, e, o);
    double ki[MAXPER], qi[MAXPER], kd[MAXPER];
    double lk = 0.0, lq = 0.0;
#pragma unroll
    for (int u = 0; u < MAXPER; ++u) {
        ki[u] = qi[u] = kd[u] = 0.0;
        const int tl = lane * per + u;
        if (u < per && tl < len) {
            const size_t r = ((size_t)bh * p.S + t0 + tl) * p.NTK;
            for (int z = 0; z < p.NTK; ++z) {
                ki[u] += (double)p.KI[r + z];
                qi[u] += (double)p.QD[r + z];
                kd[u] += (double)p.KD[r + z];
            }
        }
        lk += ki[u];
        lq += qi[u];
    }
    // k . dk^inter over the chunk's tokens before this lane's, q . dq^inter over those from it on
    double kpre = warp_scan_incl(lk, lane) - lk;
    double qtot = lq;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) qtot += __shfl_xor_sync(0xffffffffu, qtot, o);
    double qsuf = qtot - (warp_scan_incl(lq, lane) - lq);
#pragma unroll
    for (int u = 0; u < MAXPER; ++u) {
        const int tl = lane * per + u;
        if (u < per && tl < len) {
            const size_t g = (size_t)bh * p.S + t0 + tl;
            p.dig[g] = (float)kd[u];
            const float f = p.fg[g];
            const float sgm = f >= 0.f ? expf(-f) / (1.f + expf(-f)) : 1.f / (1.f + expf(f));   // sigmoid(-f)
            p.dfg[g] = (float)(e + qsuf + kpre + (double)p.RECT[g]) * sgm;
        }
        kpre += ki[u];
        qsuf -= qi[u];
    }
}

// ---------------------------------------------------------------- the pairs that skip a chunk
// grid (BH, NC), 256 threads: EP[c] = E_c = exp(g_c + m_c - m_{c+1}) (<G_end, C_c> + <dn_end, n_c>), the
// gradient of the state at chunk c's end against the decayed state at its start (fp32 arrays).
__global__ void __launch_bounds__(NT) bwd_skip_kernel(Params p)
{
    griddep_wait();
    griddep_launch_dependents();
    __shared__ double wsum[NT / 32];
    const int bh = blockIdx.x, c = blockIdx.y, tid = threadIdx.x;
    const size_t nstate = (size_t)p.DK * p.DV, zc = (size_t)bh * p.NC + c;
    const float4 *ge = reinterpret_cast<const float4 *>(p.GS + zc * nstate);
    const float4 *cs = reinterpret_cast<const float4 *>(p.CS + zc * nstate);
    float acc = 0.f;
    for (size_t e = tid; e < nstate / 4; e += NT) {
        const float4 a = ge[e], b = cs[e];
        acc = fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, fmaf(a.w, b.w, acc))));
    }
    for (int d = tid; d < p.DK; d += NT) acc = fmaf(p.GN[zc * p.DK + d], p.NS[zc * p.DK + d], acc);
    double v = acc;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((tid & 31) == 0) wsum[tid >> 5] = v;
    __syncthreads();
    if (tid == 0) {
        double t = 0.0;
        for (int w = 0; w < NT / 32; ++w) t += wsum[w];
        const float decay = expf(p.G[zc] + p.MC[(size_t)bh * (p.NC + 1) + c] - p.MC[(size_t)bh * (p.NC + 1) + c + 1]);
        p.EP[zc] = (float)t * decay;
    }
}

template <typename T>
cudaError_t launch_t(const Params &p, int BH, cudaStream_t st, const bwdtc::Args *tc)
{
    cudaError_t e;
    e = tc ? bwdtc::launch_scores(*tc) : launch_kernel(bwd_scores_kernel<T>, dim3(BH, p.NC), dim3(NT), 0, st, 1, p);
    if (e != cudaSuccess) return e;
    e = tc ? bwdtc::launch_num(*tc) : launch_kernel(bwd_num_kernel<T>, dim3(BH, p.NC, p.NJT), dim3(NT), 0, st, 1, p);
    if (e != cudaSuccess) return e;
    e = tc ? bwdtc::launch_ds(*tc) : launch_kernel(bwd_ds_kernel<T>, dim3(BH, p.NC), dim3(NT), 0, st, 1, p);
    if (e != cudaSuccess) return e;
    if (tc) {   // the read-out's state gradients and their reverse scan in one walk
        e = bwdtc::launch_gstate(*tc);
    } else {
        e = launch_kernel(bwd_dc_kernel<T>, dim3(BH * p.NC, (p.DK + GM - 1) / GM, p.NJT), dim3(NT), 0, st, 1, p);
        if (e != cudaSuccess) return e;
        e = launch_kernel(bwd_state_scan_kernel, dim3((p.DK * p.DV / 4 + 255) / 256, BH), dim3(256), 0, st, 1, p);
        if (e == cudaSuccess) e = launch_kernel(bwd_skip_kernel, dim3(BH, p.NC), dim3(NT), 0, st, 1, p);
    }
    if (e != cudaSuccess) return e;
    if (tc) {   // dq, dk, dv on the tensor cores
        if ((e = bwdtc::launch(*tc)) != cudaSuccess) return e;
        return launch_kernel(bwd_gate_kernel, dim3(BH, (p.NC + GT / 32 - 1) / (GT / 32)), dim3(GT), 0, st, 1, p);
    }
    const int nk = (p.DK + GM - 1) / GM;
    if ((e = launch_kernel(bwd_grad_kernel<T, 0>, dim3(BH, p.NC, nk), dim3(NT), 0, st, 1, p)) != cudaSuccess) return e;
    if ((e = launch_kernel(bwd_grad_kernel<T, 1>, dim3(BH, p.NC, nk), dim3(NT), 0, st, 1, p)) != cudaSuccess) return e;
    if ((e = launch_kernel(bwd_grad_kernel<T, 2>, dim3(BH, p.NC, p.NJT), dim3(NT), 0, st, 1, p)) != cudaSuccess) return e;
    return launch_kernel(bwd_gate_kernel, dim3(BH, (p.NC + GT / 32 - 1) / (GT / 32)), dim3(GT), 0, st, 1, p);
}

}  // namespace bwd

cudaError_t launch_bwd(const BwdArgs &a, const BwdWorkspace &w)
{
    bwd::Params p;
    p.S = a.S; p.L = a.chunk; p.NC = w.NC; p.DK = a.DHQK; p.DV = a.DHV; p.NTK = (a.DHQK + 31) / 32;
    p.q = a.q; p.k = a.k; p.v = a.v; p.o = a.ogate; p.dh = a.dh; p.ig = a.igate; p.fg = a.fgate;
    p.A = w.A; p.P = w.M; p.MC = w.MC; p.G = w.G; p.CS = w.CS; p.NS = w.NS;
    p.GS = w.GS; p.GN = w.GN; p.Gt = w.Gt; p.DD = w.DD; p.P2 = w.P2; p.AI = w.AI; p.QD = w.QD; p.KD = w.KD;
    p.KI = w.KI; p.RECT = w.RECT; p.EP = w.EP; p.NEP = w.NEP; p.DEN = w.DEN; p.NRM = w.NRM; p.DOTP = w.DOTP; p.NJT = (a.DHV + 63) / 64;
    p.dq = a.dq; p.dk = a.dk; p.dv = a.dv; p.dog = a.ogate ? a.dogate : nullptr; p.dig = a.digate; p.dfg = a.dfgate;
    if (!a.bf16) return bwd::launch_t<float>(p, a.BH, a.stream, nullptr);
    if (!w.tc) return bwd::launch_t<__nv_bfloat16>(p, a.BH, a.stream, nullptr);
    using bf = __nv_bfloat16;
    bwdtc::Args t;
    t.BH = a.BH; t.S = a.S; t.L = a.chunk; t.NC = w.NC; t.DK = a.DHQK; t.DV = a.DHV; t.NTK = p.NTK;
    t.A = w.A; t.P = w.M; t.MC = w.MC; t.G = w.G; t.ig = a.igate; t.DD = w.DD; t.NS = w.NS; t.GN = w.GN;
    t.q = static_cast<const bf *>(a.q); t.k = static_cast<const bf *>(a.k); t.v = static_cast<const bf *>(a.v);
    t.C16 = w.CS16; t.G16 = w.GS16; t.g16 = w.Gt16; t.dS16 = w.P216; t.A16 = w.AI16;
    t.dq = static_cast<bf *>(a.dq); t.dk = static_cast<bf *>(a.dk); t.dv = static_cast<bf *>(a.dv);
    t.QD = w.QD; t.KD = w.KD; t.KI = w.KI; t.RECTw = w.RECT; t.EPw = w.EP; t.NEP = w.NEP; t.status = w.status; t.stream = a.stream;
    t.dh = static_cast<const bf *>(a.dh); t.o = static_cast<const bf *>(a.ogate); t.NRM = w.NRM;
    t.DOTP = w.DOTP; t.g16w = w.Gt16; t.dog = a.ogate ? static_cast<bf *>(a.dogate) : nullptr;
    t.NJT = p.NJT; t.sg16 = w.SG16; t.G16w = w.GS16;
    t.wk16 = w.WK16; t.C16w = w.CS16; t.NSw = w.NS;
    t.DENw = w.DEN; t.NRMw = w.NRM; t.DDw = w.DD; t.GNw = w.GN; t.A16w = w.AI16; t.dS16w = w.P216;
    cudaError_t e = bwdtc::launch_carry(t);   // the chunk-start states
    if (e != cudaSuccess) return e;
    return bwd::launch_t<bf>(p, a.BH, a.stream, &t);
}

bool bwd_tc_path(bool bf16, int BH, int S, int DHQK, int DHV, int chunk)
{
    // (tensor-map extents are 32-bit: the chunk-start states' two parts span 2 BH NC boxes, the
    // scores' two parts 2 NC chunk rows; the grids take NC chunks in y)
    const long long NC = (S + (long long)chunk - 1) / chunk;
    return bf16 && bwdtc::supported(DHQK, DHV, chunk) && 2LL * BH * NC < (1LL << 31) &&
           2LL * NC * chunk < (1LL << 31) && NC <= 65535;
}

}  // namespace mlstm
