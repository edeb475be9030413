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
// Gate gradients: h depends on the global cumulative log decay A_t only through exp(A_t) qh_t
// and exp(i~_s - A_s) k_s (the unstabilized read-out), so
//   dL/di~_t = k_t . dk_t,  dL/dA_t = q_t . dq_t - k_t . dk_t,
//   dL/dlog f_j = sum_{t >= j} dL/dA_t,  dL/df~_j = dL/dlog f_j * sigmoid(-f~_j),
// a reverse cumulative sum over the sequence (accumulated in fp64).
#include "common.cuh"
#include "mlstm_internal.h"

namespace mlstm {
namespace bwd {

constexpr int NT = 256;   // threads of the chunk kernels
constexpr int TW = 32;    // column tile

struct Params {
    int S, L, NC, DK, DV, NTK;
    const void *q, *k, *v, *o, *dh;
    const float *ig, *fg;
    const float *A, *P, *MC, *G;     // gate preprocessing
    const float *CS, *NS;            // chunk-start states [BH][NC][DK][DV], [BH][NC][DK]
    float *GS, *GN;                  // read-out state gradients, then chunk-end gradients (same layout)
    float *Gt;                       // g = o dh / N [BH][S][DV]
    float *DD;                       // dden [BH][S]
    float *P2, *AI;                  // dS and A per chunk [BH][NC][L][L]
    float *QD, *KD;                  // per dk tile partial q . dq and k . dk [BH][S][NTK]
    void *dq, *dk, *dv, *dog;
    float *dig, *dfg;
};

// Shared-memory floats of bwd_chunk_kernel and bwd_grad_kernel for chunk length L.
__host__ __device__ constexpr int chunk_smem_floats(int L) { return 2 * L * (L + 1) + 3 * L * 33 + 32 * 33 + 8 * L; }
__host__ __device__ constexpr int grad_smem_floats(int L) { return L * (L + 1) + 2 * L * 36 + 2 * 32 * 36 + 4 * L; }

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
template <typename T>
__global__ void __launch_bounds__(NT, 3) bwd_chunk_kernel(Params p)
{
    griddep_wait();
    griddep_launch_dependents();
    extern __shared__ float sm[];
    const int L = p.L, LP = L + 1, DK = p.DK, DV = p.DV;
    float *Sm = sm;               // [L][LP]: S, then A = D * S
    float *dAg = Sm + L * LP;     // [L][LP]: g v^T over the value tiles
    float *qs = dAg + L * LP;     // [L][33]
    float *xs = qs + L * 33;      // [L][33]: k slice, then v tile
    float *gs = xs + L * 33;      // [L][33]: g tile
    float *cs = gs + L * 33;      // [32][33]: slice of C_c
    float *xs_ = cs + 32 * 33, *mx = xs_ + L, *fl = mx + L, *sc = fl + L;
    float *den = sc + L, *nrm = den + L, *dot = nrm + L, *dd = dot + L;

    const int bh = blockIdx.x, c = blockIdx.y;
    const int t0 = c * L, len = min(L, p.S - t0);
    const int tid = threadIdx.x, x = tid & 31, ty = tid >> 5;
    const float scale = rsqrtf((float)DK);
    const T *qb = static_cast<const T *>(p.q) + ((size_t)bh * p.S + t0) * DK;
    const T *kb = static_cast<const T *>(p.k) + ((size_t)bh * p.S + t0) * DK;
    const T *vb = static_cast<const T *>(p.v) + ((size_t)bh * p.S + t0) * DV;
    const T *ob = p.o ? static_cast<const T *>(p.o) + ((size_t)bh * p.S + t0) * DV : nullptr;
    const T *dhb = static_cast<const T *>(p.dh) + ((size_t)bh * p.S + t0) * DV;
    T *dob = p.dog ? static_cast<T *>(p.dog) + ((size_t)bh * p.S + t0) * DV : nullptr;
    float *gtb = p.Gt + ((size_t)bh * p.S + t0) * DV;
    const float *Cc = p.CS + ((size_t)bh * p.NC + c) * DK * DV;
    const float *nc = p.NS + ((size_t)bh * p.NC + c) * DK;

    chunk_rows(p, bh, c, t0, len, xs_, mx, fl, sc);
    for (int t = tid; t < L; t += NT) dot[t] = 0.f;
    for (int e = tid; e < L * LP; e += NT) {
        Sm[e] = 0.f;
        dAg[e] = 0.f;
    }
    __syncthreads();

    // S = qh K^T over slices of 32 of DK (lower triangle)
    for (int d0 = 0; d0 < DK; d0 += 32) {
        for (int e = tid; e < L * 32; e += NT) {
            const int t = e >> 5, xx = e & 31;
            const bool ok = t < len && d0 + xx < DK;
            qs[t * 33 + xx] = ok ? to_f32(qb[(size_t)t * DK + d0 + xx]) * scale : 0.f;
            xs[t * 33 + xx] = ok ? to_f32(kb[(size_t)t * DK + d0 + xx]) : 0.f;
        }
        __syncthreads();
        for (int e = tid; e < L * L; e += NT) {
            const int t = e / L, s = e % L;
            if (s <= t) {
                float acc = Sm[t * LP + s];
#pragma unroll 8
                for (int xx = 0; xx < 32; ++xx) acc = fmaf(qs[t * 33 + xx], xs[s * 33 + xx], acc);
                Sm[t * LP + s] = acc;
            }
        }
        __syncthreads();
    }
    // A = D * S on the causal triangle (zero elsewhere and past the end of the sequence)
    for (int e = tid; e < L * L; e += NT) {
        const int t = e / L, s = e % L;
        Sm[t * LP + s] = (s <= t && t < len) ? Sm[t * LP + s] * expf(xs_[s] - mx[t]) : 0.f;
    }
    __syncthreads();
    // den and the normalizer N
    for (int t = tid; t < L; t += NT) {
        float r = 0.f;
        for (int s = 0; s <= t; ++s) r += Sm[t * LP + s];
        float qn = 0.f;
        if (t < len) {
            for (int d = 0; d < DK; ++d) qn = fmaf(nc[d], to_f32(qb[(size_t)t * DK + d]), qn);
            qn *= scale * sc[t];
        }
        den[t] = r + qn;
        nrm[t] = t < len ? fmaxf(fabsf(r + qn), fl[t]) : 1.f;
    }
    __syncthreads();

    // value tiles of 32 columns: num, hh = num / N, do, g; sum of g . hh per row; g v^T
    const int RPT = L / 8;   // rows per thread: t = ty + 8 r
    for (int j0 = 0; j0 < DV; j0 += 32) {
        float acc[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) acc[r] = 0.f;
        for (int d0 = 0; d0 < DK; d0 += 32) {
            for (int e = tid; e < L * 32; e += NT) {
                const int t = e >> 5, xx = e & 31;
                qs[t * 33 + xx] = (t < len && d0 + xx < DK) ? to_f32(qb[(size_t)t * DK + d0 + xx]) * scale : 0.f;
            }
            for (int e = tid; e < 32 * 32; e += NT) {
                const int d = e >> 5, xx = e & 31;
                cs[d * 33 + xx] = (d0 + d < DK && j0 + xx < DV) ? Cc[(size_t)(d0 + d) * DV + j0 + xx] : 0.f;
            }
            __syncthreads();
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                const int t = ty + 8 * r;
                if (r < RPT) {
                    float a2 = 0.f;
#pragma unroll 8
                    for (int d = 0; d < 32; ++d) a2 = fmaf(qs[t * 33 + d], cs[d * 33 + x], a2);
                    acc[r] = fmaf(sc[t], a2, acc[r]);
                }
            }
            __syncthreads();
        }
        for (int e = tid; e < L * 32; e += NT) {
            const int s = e >> 5, xx = e & 31;
            xs[s * 33 + xx] = (s < len && j0 + xx < DV) ? to_f32(vb[(size_t)s * DV + j0 + xx]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const int t = ty + 8 * r;
            if (r < RPT) {
                float a2 = 0.f;
                for (int s = 0; s <= t; ++s) a2 = fmaf(Sm[t * LP + s], xs[s * 33 + x], a2);
                acc[r] += a2;
            }
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const int t = ty + 8 * r;
            if (r < RPT) {
                const int j = j0 + x;
                float g = 0.f, hh = 0.f;
                if (t < len && j < DV) {
                    const size_t off = (size_t)t * DV + j;
                    hh = acc[r] / nrm[t];
                    const float dhv = to_f32(dhb[off]);
                    const float ov = ob ? to_f32(ob[off]) : 1.f;
                    if (dob) dob[off] = from_f32<T>(dhv * hh);
                    g = ov * dhv / nrm[t];
                    gtb[off] = g;
                }
                gs[t * 33 + x] = g;
                const float pr = warp_sum(g * hh);   // the warp holds one row t
                if (x == 0) dot[t] += pr;
            }
        }
        __syncthreads();
        for (int e = tid; e < L * L; e += NT) {
            const int t = e / L, s = e % L;
            if (s <= t && t < len) {
                float a2 = dAg[t * LP + s];
#pragma unroll 8
                for (int xx = 0; xx < 32; ++xx) a2 = fmaf(gs[t * 33 + xx], xs[s * 33 + xx], a2);
                dAg[t * LP + s] = a2;
            }
        }
        __syncthreads();
    }

    // dden (the branch of the max that the forward pass took), then dS = (g v^T + dden) * D and A
    for (int t = tid; t < L; t += NT) {
        const bool live = t < len && fabsf(den[t]) > fl[t];
        dd[t] = live ? -dot[t] * copysignf(1.f, den[t]) : 0.f;
        if (t < len) p.DD[(size_t)bh * p.S + t0 + t] = dd[t];
    }
    __syncthreads();
    float *P2g = p.P2 + ((size_t)bh * p.NC + c) * L * L;
    float *AIg = p.AI + ((size_t)bh * p.NC + c) * L * L;
    for (int e = tid; e < L * L; e += NT) {
        const int t = e / L, s = e % L;
        float pv = 0.f;
        if (s <= t && t < len) pv = (dAg[t * LP + s] + dd[t]) * expf(xs_[s] - mx[t]);
        P2g[e] = pv;
        AIg[e] = Sm[t * LP + s];
    }

    // the read-out's state gradients: dC[i][j] = sum_t sc_t qh_t[i] g_t[j], dn[i] = sum_t sc_t dd_t qh_t[i]
    float *GSc = p.GS + ((size_t)bh * p.NC + c) * DK * DV;
    float *GNc = p.GN + ((size_t)bh * p.NC + c) * DK;
    for (int i0 = 0; i0 < DK; i0 += 32) {
        __syncthreads();
        for (int e = tid; e < L * 32; e += NT) {
            const int t = e >> 5, xx = e & 31;
            qs[t * 33 + xx] = (t < len && i0 + xx < DK) ? sc[t] * to_f32(qb[(size_t)t * DK + i0 + xx]) * scale : 0.f;
        }
        __syncthreads();
        if (tid < 32 && i0 + tid < DK) {
            float a2 = 0.f;
            for (int t = 0; t < len; ++t) a2 = fmaf(qs[t * 33 + tid], dd[t], a2);
            GNc[i0 + tid] = a2;
        }
        for (int j0 = 0; j0 < DV; j0 += 32) {
            for (int e = tid; e < L * 32; e += NT) {
                const int t = e >> 5, xx = e & 31;
                gs[t * 33 + xx] = (t < len && j0 + xx < DV) ? __ldcg(gtb + (size_t)t * DV + j0 + xx) : 0.f;
            }
            __syncthreads();
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int i = ty + 8 * r;
                float a2 = 0.f;
                for (int t = 0; t < len; ++t) a2 = fmaf(qs[t * 33 + i], gs[t * 33 + x], a2);
                if (i0 + i < DK && j0 + x < DV) GSc[(size_t)(i0 + i) * DV + j0 + x] = a2;
            }
            __syncthreads();
        }
    }
}

// ---------------------------------------------------------------- reverse scan of the state gradients
// grid (ceil(DK * DV / 256), BH): each thread one state element; G_c = dC_c + decay_c G_{c+1}, the
// slot of chunk c then holds G_{c+1} (the gradient of the state at the chunk's end).
__global__ void __launch_bounds__(256) bwd_state_scan_kernel(Params p)
{
    griddep_wait();
    griddep_launch_dependents();
    const int bh = blockIdx.y;
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    const float *MCb = p.MC + (size_t)bh * (p.NC + 1);
    const float *Gb = p.G + (size_t)bh * p.NC;
    const size_t nstate = (size_t)p.DK * p.DV;
    if (e < p.DK * p.DV) {
        float *slot = p.GS + (size_t)bh * p.NC * nstate + e;
        float G = 0.f;
        constexpr int BATCH = 8;
        for (int c1 = p.NC; c1 > 0; c1 -= BATCH) {   // chunks c1 - 1 down to c1 - BATCH, loads first
            float d[BATCH];
#pragma unroll
            for (int u = 0; u < BATCH; ++u)
                if (c1 - 1 - u >= 0) d[u] = __ldcg(slot + (size_t)(c1 - 1 - u) * nstate);
#pragma unroll
            for (int u = 0; u < BATCH; ++u) {
                const int c = c1 - 1 - u;
                if (c >= 0) {
                    slot[(size_t)c * nstate] = G;
                    G = d[u] + expf(Gb[c] + MCb[c] - MCb[c + 1]) * G;
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

// ---------------------------------------------------------------- per chunk and column tile: dq, dk, dv
// grid (BH, NC, NTK + NTV), NT threads.  Tiles z < NTK: 32 columns of DK (dq and dk); the rest:
// 32 columns of DV (dv).  A thread owns column x of the tile for the rows ty + 8 r; the products
// run with the reduction index outermost, so that a shared value read by the whole warp (a row of
// the left factor) and one per lane (the lane's column of the right factor) feed the warp's rows,
// four reduction steps per 16-byte load where the layout allows.
constexpr int TS = 36;    // row stride of the 32-column tiles (16-byte aligned rows, no bank conflicts)

template <typename T>
__global__ void __launch_bounds__(NT) bwd_grad_kernel(Params p)
{
    griddep_wait();
    griddep_launch_dependents();
    extern __shared__ float sm[];
    const int L = p.L, LP = L + 1, DK = p.DK, DV = p.DV;
    float *Ms = sm;               // [L][LP]: dS (key tiles) or A (value tiles)
    float *as_ = Ms + L * LP;     // [L][TS]
    float *bs = as_ + L * TS;     // [L][TS]
    float *cs = bs + L * TS;      // [32][TS]
    float *cs2 = cs + 32 * TS;    // [32][TS]
    float *xs_ = cs2 + 32 * TS, *mx = xs_ + L, *fl = mx + L, *sc = fl + L;

    const int bh = blockIdx.x, c = blockIdx.y, z = blockIdx.z;
    const int t0 = c * L, len = min(L, p.S - t0);
    const int tid = threadIdx.x, x = tid & 31, ty = tid >> 5;
    const float scale = rsqrtf((float)DK);
    const T *qb = static_cast<const T *>(p.q) + ((size_t)bh * p.S + t0) * DK;
    const T *kb = static_cast<const T *>(p.k) + ((size_t)bh * p.S + t0) * DK;
    const T *vb = static_cast<const T *>(p.v) + ((size_t)bh * p.S + t0) * DV;
    const float *gtb = p.Gt + ((size_t)bh * p.S + t0) * DV;
    const float *Cc = p.CS + ((size_t)bh * p.NC + c) * DK * DV;
    const float *nc = p.NS + ((size_t)bh * p.NC + c) * DK;
    const float *Ge = p.GS + ((size_t)bh * p.NC + c) * DK * DV;   // gradient of the state at the chunk's end
    const float *ge = p.GN + ((size_t)bh * p.NC + c) * DK;
    const float *ddb = p.DD + (size_t)bh * p.S + t0;
    const float gc = p.G[(size_t)bh * p.NC + c], mn = p.MC[(size_t)bh * (p.NC + 1) + c + 1];
    const int RPT = L / 8;

    chunk_rows(p, bh, c, t0, len, xs_, mx, fl, sc);
    const float *Mg = (z < p.NTK ? p.P2 : p.AI) + ((size_t)bh * p.NC + c) * L * L;
    for (int e = tid; e < L * L; e += NT) Ms[(e / L) * LP + e % L] = Mg[e];
    __syncthreads();
    // w_s = exp(g_c - a_s + i~_s - m_{c+1}): weight of token s in the state at the chunk's end
    const float gm = gc - mn;
    auto wtok = [&](int s) { return s < len ? expf(xs_[s] + gm) : 0.f; };

    if (z < p.NTK) {
        const int i0 = z * 32;
        const int i = i0 + x;
        for (int e = tid; e < L * 32; e += NT) {
            const int t = e >> 5, xx = e & 31;
            const bool ok = t < len && i0 + xx < DK;
            as_[t * TS + xx] = ok ? to_f32(kb[(size_t)t * DK + i0 + xx]) : 0.f;
            bs[t * TS + xx] = ok ? to_f32(qb[(size_t)t * DK + i0 + xx]) * scale : 0.f;
        }
        __syncthreads();
        float aq[16], ak[16], iq[16], ik[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) aq[r] = ak[r] = iq[r] = ik[r] = 0.f;
        // dS K (row t: sum_s dS_ts k_s) and dS^T qh (row t: sum_u dS_ut qh_u); dS is zero above the
        // diagonal and past the end of the sequence
        for (int s = 0; s < L; ++s) {
            const float ks = as_[s * TS + x], qs = bs[s * TS + x];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                if (r < RPT) {
                    const int t = ty + 8 * r;
                    aq[r] = fmaf(Ms[t * LP + s], ks, aq[r]);
                    ak[r] = fmaf(Ms[s * LP + t], qs, ak[r]);
                }
            }
        }
        // inter-chunk parts over slices of 32 of DV: g C_c^T (rows t) and V G_end^T (rows s)
        for (int j0 = 0; j0 < DV; j0 += 32) {
            __syncthreads();
            for (int e = tid; e < L * 32; e += NT) {
                const int t = e >> 5, xx = e & 31;
                const bool ok = t < len && j0 + xx < DV;
                as_[t * TS + xx] = ok ? gtb[(size_t)t * DV + j0 + xx] : 0.f;
                bs[t * TS + xx] = ok ? to_f32(vb[(size_t)t * DV + j0 + xx]) : 0.f;
            }
            for (int e = tid; e < 32 * 32; e += NT) {
                const int ii = e >> 5, xx = e & 31;
                const bool ok = i0 + ii < DK && j0 + xx < DV;
                cs[ii * TS + xx] = ok ? Cc[(size_t)(i0 + ii) * DV + j0 + xx] : 0.f;
                cs2[ii * TS + xx] = ok ? Ge[(size_t)(i0 + ii) * DV + j0 + xx] : 0.f;
            }
            __syncthreads();
#pragma unroll 2
            for (int jj = 0; jj < 32; jj += 4) {
                const float4 c4 = *reinterpret_cast<const float4 *>(cs + x * TS + jj);
                const float4 e4 = *reinterpret_cast<const float4 *>(cs2 + x * TS + jj);
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    if (r < RPT) {
                        const int t = ty + 8 * r;
                        const float4 g4 = *reinterpret_cast<const float4 *>(as_ + t * TS + jj);
                        const float4 v4 = *reinterpret_cast<const float4 *>(bs + t * TS + jj);
                        iq[r] = fmaf(g4.x, c4.x, fmaf(g4.y, c4.y, fmaf(g4.z, c4.z, fmaf(g4.w, c4.w, iq[r]))));
                        ik[r] = fmaf(v4.x, e4.x, fmaf(v4.y, e4.y, fmaf(v4.z, e4.z, fmaf(v4.w, e4.w, ik[r]))));
                    }
                }
            }
        }
        const float ncx = i < DK ? nc[i] : 0.f, gex = i < DK ? ge[i] : 0.f;
        T *dqb = static_cast<T *>(p.dq) + ((size_t)bh * p.S + t0) * DK;
        T *dkb = static_cast<T *>(p.dk) + ((size_t)bh * p.S + t0) * DK;
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const int t = ty + 8 * r;
            if (r < RPT) {
                float qdq = 0.f, kdk = 0.f;
                if (t < len && i < DK) {
                    const float dqh = aq[r] + sc[t] * (iq[r] + ddb[t] * ncx);
                    const float dkv = ak[r] + wtok(t) * (ik[r] + gex);
                    const float qh = to_f32(qb[(size_t)t * DK + i]) * scale;
                    const float kv = to_f32(kb[(size_t)t * DK + i]);
                    dqb[(size_t)t * DK + i] = from_f32<T>(dqh * scale);
                    dkb[(size_t)t * DK + i] = from_f32<T>(dkv);
                    qdq = qh * dqh;
                    kdk = kv * dkv;
                }
                qdq = warp_sum(qdq);
                kdk = warp_sum(kdk);
                if (x == 0 && t < len) {
                    p.QD[((size_t)bh * p.S + t0 + t) * p.NTK + z] = qdq;
                    p.KD[((size_t)bh * p.S + t0 + t) * p.NTK + z] = kdk;
                }
            }
        }
    } else {
        const int j0 = (z - p.NTK) * 32;
        const int j = j0 + x;
        for (int e = tid; e < L * 32; e += NT) {
            const int t = e >> 5, xx = e & 31;
            as_[t * TS + xx] = (t < len && j0 + xx < DV) ? gtb[(size_t)t * DV + j0 + xx] : 0.f;
        }
        __syncthreads();
        float av[16], iv[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) av[r] = iv[r] = 0.f;
        // A^T g (row s: sum_u A_us g_u); A is zero above the diagonal and past the end
        for (int u = 0; u < L; ++u) {
            const float gu = as_[u * TS + x];
#pragma unroll
            for (int r = 0; r < 16; ++r)
                if (r < RPT) av[r] = fmaf(Ms[u * LP + ty + 8 * r], gu, av[r]);
        }
        // K G_end over slices of 32 of DK; the slice of G_end transposed ([value column][DK]) so that
        // a lane reads its column's four DK entries at once
        float *gT = cs2;
        for (int i0 = 0; i0 < DK; i0 += 32) {
            __syncthreads();
            for (int e = tid; e < L * 32; e += NT) {
                const int t = e >> 5, xx = e & 31;
                bs[t * TS + xx] = (t < len && i0 + xx < DK) ? to_f32(kb[(size_t)t * DK + i0 + xx]) : 0.f;
            }
            for (int e = tid; e < 32 * 32; e += NT) {
                const int ii = e >> 5, xx = e & 31;
                gT[xx * TS + ii] = (i0 + ii < DK && j0 + xx < DV) ? Ge[(size_t)(i0 + ii) * DV + j0 + xx] : 0.f;
            }
            __syncthreads();
#pragma unroll 2
            for (int ii = 0; ii < 32; ii += 4) {
                const float4 e4 = *reinterpret_cast<const float4 *>(gT + x * TS + ii);
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    if (r < RPT) {
                        const float4 k4 = *reinterpret_cast<const float4 *>(bs + (ty + 8 * r) * TS + ii);
                        iv[r] = fmaf(k4.x, e4.x, fmaf(k4.y, e4.y, fmaf(k4.z, e4.z, fmaf(k4.w, e4.w, iv[r]))));
                    }
                }
            }
        }
        T *dvb = static_cast<T *>(p.dv) + ((size_t)bh * p.S + t0) * DV;
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const int s = ty + 8 * r;
            if (r < RPT && s < len && j < DV) dvb[(size_t)s * DV + j] = from_f32<T>(av[r] + wtok(s) * iv[r]);
        }
    }
}

// ---------------------------------------------------------------- gate gradients
// grid (BH), 1024 threads: dL/di~_t = k_t . dk_t; dL/df~_j = sigmoid(-f~_j) sum_{t >= j} (q_t . dq_t - k_t . dk_t).
constexpr int GT = 1024;

__global__ void __launch_bounds__(GT) bwd_gate_kernel(Params p)
{
    griddep_wait();
    griddep_launch_dependents();
    __shared__ double wsum[GT / 32];
    const int bh = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (p.S + GT - 1) / GT;
    const int tb = min(tid * per, p.S), te = min(tb + per, p.S);
    const float *qd = p.QD + (size_t)bh * p.S * p.NTK;
    const float *kd = p.KD + (size_t)bh * p.S * p.NTK;
    auto da = [&](int t, double *kdk) {
        double a = 0.0, b = 0.0;
        for (int z = 0; z < p.NTK; ++z) {
            a += (double)qd[(size_t)t * p.NTK + z];
            b += (double)kd[(size_t)t * p.NTK + z];
        }
        *kdk = b;
        return a - b;
    };
    double loc = 0.0, kk;
    for (int t = tb; t < te; ++t) loc += da(t, &kk);
    // exclusive suffix sum over the threads after this one (the tokens after this thread's range)
    double inc = loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double y = __shfl_down_sync(0xffffffffu, inc, o);
        if (lane + o < 32) inc += y;
    }
    if (lane == 0) wsum[warp] = inc;   // the warp's total
    __syncthreads();
    double after = inc - loc;           // later lanes of this warp
    for (int w2 = warp + 1; w2 < GT / 32; ++w2) after += wsum[w2];
    double run = after;
    for (int t = te - 1; t >= tb; --t) {
        run += da(t, &kk);
        const size_t g = (size_t)bh * p.S + t;
        p.dig[g] = (float)kk;
        const float f = p.fg[g];
        const float sgm = f >= 0.f ? expf(-f) / (1.f + expf(-f)) : 1.f / (1.f + expf(f));   // sigmoid(-f)
        p.dfg[g] = (float)run * sgm;
    }
}

template <typename T>
cudaError_t launch_t(const Params &p, int BH, cudaStream_t st)
{
    const int ntv = (p.DV + TW - 1) / TW;
    const size_t sm1 = sizeof(float) * chunk_smem_floats(p.L);
    const size_t sm2 = sizeof(float) * grad_smem_floats(p.L);
    cudaError_t e;
    if ((e = ensure_dynamic_smem((const void *)bwd_chunk_kernel<T>, (int)sm1)) != cudaSuccess) return e;
    if ((e = ensure_dynamic_smem((const void *)bwd_grad_kernel<T>, (int)sm2)) != cudaSuccess) return e;
    e = launch_kernel(bwd_chunk_kernel<T>, dim3(BH, p.NC), dim3(NT), sm1, st, 1, p);
    if (e != cudaSuccess) return e;
    e = launch_kernel(bwd_state_scan_kernel, dim3((p.DK * p.DV + 255) / 256, BH), dim3(256), 0, st, 1, p);
    if (e != cudaSuccess) return e;
    e = launch_kernel(bwd_grad_kernel<T>, dim3(BH, p.NC, p.NTK + ntv), dim3(NT), sm2, st, 1, p);
    if (e != cudaSuccess) return e;
    return launch_kernel(bwd_gate_kernel, dim3(BH), dim3(GT), 0, st, 1, p);
}

}  // namespace bwd

cudaError_t launch_bwd(const BwdArgs &a, const BwdWorkspace &w)
{
    bwd::Params p;
    p.S = a.S; p.L = a.chunk; p.NC = w.NC; p.DK = a.DHQK; p.DV = a.DHV; p.NTK = (a.DHQK + 31) / 32;
    p.q = a.q; p.k = a.k; p.v = a.v; p.o = a.ogate; p.dh = a.dh; p.ig = a.igate; p.fg = a.fgate;
    p.A = w.A; p.P = w.M; p.MC = w.MC; p.G = w.G; p.CS = w.CS; p.NS = w.NS;
    p.GS = w.GS; p.GN = w.GN; p.Gt = w.Gt; p.DD = w.DD; p.P2 = w.P2; p.AI = w.AI; p.QD = w.QD; p.KD = w.KD;
    p.dq = a.dq; p.dk = a.dk; p.dv = a.dv; p.dog = a.ogate ? a.dogate : nullptr; p.dig = a.digate; p.dfg = a.dfgate;
    return a.bf16 ? bwd::launch_t<__nv_bfloat16>(p, a.BH, a.stream) : bwd::launch_t<float>(p, a.BH, a.stream);
}

}  // namespace mlstm
