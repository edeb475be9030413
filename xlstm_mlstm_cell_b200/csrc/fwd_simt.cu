// fwd_simt.cu -- chunkwise forward pass on CUDA cores in fp32 (no tensor cores).
//
// This path serves float32 inputs (where bf16 tensor-core operands cannot meet
// an fp32 error budget) and the shapes the tensor-core path does not take
// (small head dimensions, chunks of 16 or 32).  It computes the same chunkwise
// decomposition as the tensor-core path, with every product in fp32 FMAs:
//
// Carry ("inter-chunk states via a scan", xLSTM Guide, "Exploit Chunkwise
// Hardware Kernels for Production Training"), per chunk c with the gate
// preprocessing a, g, m of gate_prep.cu:
//   w_s     = exp(g_c - a_s + i~_s - m_{c+1})              (<= 1)
//   C_{c+1} = exp(g_c + m_c - m_{c+1}) C_c + sum_s w_s k_s v_s^T
//   n_{c+1} = exp(g_c + m_c - m_{c+1}) n_c + sum_s w_s k_s
//
// Output (the causal decay matrix of "The Dual Formulation", restricted to a
// chunk, plus the state of the chunk start), for token tau of chunk c:
//   D_{tau,s} = exp(a_tau - a_s + i~_s - m_tau)  for s <= tau, else 0     (<= 1)
//   sc_tau    = exp(a_tau + m_c - m_tau)                                  (<= 1)
//   num_tau   = sc_tau C_c^T qh_tau + sum_s D_{tau,s} (qh_tau . k_s) v_s
//   den_tau   = sc_tau n_c . qh_tau + sum_s D_{tau,s} (qh_tau . k_s)
//   h_tau     = o_tau * num_tau / max(|den_tau|, exp(-m_tau))
// In exact arithmetic this equals the token-by-token recurrence.
#include "common.cuh"
#include "mlstm_internal.h"

namespace mlstm {

constexpr int ST = 32;   // state tile edge (rows of C and columns of C / h)

// ---------------------------------------------------------------- carry
// grid (BH, ceil(DHQK/64), ceil(DHV/64)), 256 threads; thread (tx, ty) = (tid % 16, tid / 16)
// owns rows 4 ty .. 4 ty + 3 and columns 4 tx .. 4 tx + 3 of a 64 x 64 tile of C, and in the tiles
// of columns 0..63 threads 0..63 own n of their row.  Walks all chunks of its head in order,
// storing the state at every chunk start (CS, or its two bf16 parts CS16 when given; NS) and the
// final state.  A chunk's k (fp32) and
// w_s v_s are staged in shared memory, so that a step of the reduction over the chunk's tokens is
// two 16-byte loads and 16 FMAs per thread; the next chunk's k, v and gates are loaded into
// registers while the current chunk's steps run.  Every state element takes the operations of a
// token-by-token fp32 update in their order: C <- decay C, then C += k_s (w_s v_s) for s
// ascending (n <- decay n, then n += w_s k_s).
constexpr int CT = 64;         // state tile edge of the carry
constexpr int CKS = CT + 4;    // row stride (floats) of the staged tiles: rows 16 bytes apart in the banks

// Eight consecutive elements of a k or v row as loaded (16-byte aligned), converted on staging.
template <typename T> struct Seg8;
template <> struct Seg8<float> {
    float4 a, b;
    MLSTM_DEVINL void load(const float *p)
    {
        a = *reinterpret_cast<const float4 *>(p);
        b = *reinterpret_cast<const float4 *>(p + 4);
    }
    MLSTM_DEVINL void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
    MLSTM_DEVINL void get(float (&f)[8]) const
    {
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
        f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    }
};
template <> struct Seg8<__nv_bfloat16> {
    uint4 u;
    MLSTM_DEVINL void load(const __nv_bfloat16 *p) { u = *reinterpret_cast<const uint4 *>(p); }
    MLSTM_DEVINL void zero() { u = make_uint4(0u, 0u, 0u, 0u); }
    MLSTM_DEVINL void get(float (&f)[8]) const
    {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int z = 0; z < 4; ++z) {   // bf16 -> fp32 is exact: the 16 bits are the high half
            f[2 * z] = __uint_as_float(w[z] << 16);
            f[2 * z + 1] = __uint_as_float(w[z] & 0xffff0000u);
        }
    }
};

template <typename T>
__global__ void __launch_bounds__(256, 2)
carry_simt_kernel(const T *__restrict__ k, const T *__restrict__ v, const float *__restrict__ igate,
                  const float *__restrict__ A, const float *__restrict__ G, const float *__restrict__ MC,
                  int S, int L, int NC, int DHQK, int DHV,
                  float *__restrict__ CS, float *__restrict__ NS, __nv_bfloat16 *__restrict__ CS16,
                  float *C_final, float *n_final, float *__restrict__ m_final, const float *C0, const float *n0)
{
    griddep_wait();
    griddep_launch_dependents();
    extern __shared__ float sm[];
    float *ks = sm;                    // [L][CKS] k_s, this tile's rows
    float *wvs = ks + L * CKS;         // [L][CKS] w_s v_s, this tile's columns
    float *wsb = wvs + L * CKS;        // [L] w_s
    const int bh = blockIdx.x, i0 = blockIdx.y * CT, j0 = blockIdx.z * CT;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const bool n_warp = blockIdx.z == 0 && tid < CT;            // warps 0 and 1 of column tile 0
    const T *kb = k + (size_t)bh * S * DHQK;
    const T *vb = v + (size_t)bh * S * DHV;
    const float *igb = igate + (size_t)bh * S;
    const float *Ab = A + (size_t)bh * S;
    const float *MCb = MC + (size_t)bh * (NC + 1);
    const float *Gb = G + (size_t)bh * NC;
    // the state elements of this thread: rows ri + r, columns cj .. cj + 3 (a group of four columns
    // lies wholly inside or outside DHV, which is a multiple of 8)
    const int ri = i0 + 4 * ty, cj = j0 + 4 * tx;
    const bool cols_in = cj < DHV;

    // initial state (zero when C0 is NULL); C_final may alias C0: every element is read here, by the
    // thread that writes it at the end
    float c[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        float4 x4 = make_float4(0.f, 0.f, 0.f, 0.f);
        if (C0 && cols_in && ri + r < DHQK) x4 = *reinterpret_cast<const float4 *>(C0 + ((size_t)bh * DHQK + ri + r) * DHV + cj);
        c[r][0] = x4.x; c[r][1] = x4.y; c[r][2] = x4.z; c[r][3] = x4.w;
    }
    float nn = 0.f;
    if (n0 && n_warp && i0 + tid < DHQK) nn = n0[(size_t)bh * DHQK + i0 + tid];

    // staging: thread tid takes row tid / 4 (and tid / 4 + 64 when L = 128) and the 16 columns
    // 16 (tid % 4) .. of the k and v tiles, as two 8-element halves (each wholly inside or outside
    // DHQK / DHV)
    const int sl = tid >> 2, xp = (tid & 3) * 16;
    Seg8<T> pk[2][2], pv[2][2];
    float pa[2] = {0.f, 0.f}, pig[2] = {0.f, 0.f};
    auto load_chunk = [&](int ch) {
        const int t0 = ch * L, len = min(L, S - t0);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int s = sl + 64 * u;
            const bool valid = s < len;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int xk = i0 + xp + 8 * h, xv = j0 + xp + 8 * h;
                if (valid && xk < DHQK) pk[u][h].load(kb + (size_t)(t0 + s) * DHQK + xk);
                else pk[u][h].zero();
                if (valid && xv < DHV) pv[u][h].load(vb + (size_t)(t0 + s) * DHV + xv);
                else pv[u][h].zero();
            }
            if (valid) {
                pa[u] = Ab[t0 + s];
                pig[u] = igb[t0 + s];
            }
        }
    };
    if (NC > 0) load_chunk(0);

    for (int ch = 0; ch < NC; ++ch) {
        const int t0 = ch * L, len = min(L, S - t0);
        // state at the chunk start
        const size_t cso = ((size_t)bh * NC + ch) * DHQK * DHV;
        if (cols_in) {
#pragma unroll
            for (int r = 0; r < 4; ++r)
                if (ri + r < DHQK) {
                    const size_t o = cso + (size_t)(ri + r) * DHV + cj;
                    if (!CS16) {
                        *reinterpret_cast<float4 *>(CS + o) = make_float4(c[r][0], c[r][1], c[r][2], c[r][3]);
                    } else {   // only the two bf16 parts, which the backward's tensor-core products read
                        __nv_bfloat16 hi[4], lo[4];
#pragma unroll
                        for (int x = 0; x < 4; ++x) bf16_parts(c[r][x], hi[x], lo[x]);
                        const size_t o16 = 2 * cso + (size_t)(ri + r) * DHV + cj;
                        *reinterpret_cast<uint2 *>(CS16 + o16) = *reinterpret_cast<const uint2 *>(hi);
                        *reinterpret_cast<uint2 *>(CS16 + o16 + (size_t)DHQK * DHV) = *reinterpret_cast<const uint2 *>(lo);
                    }
                }
        }
        if (n_warp && i0 + tid < DHQK) NS[((size_t)bh * NC + ch) * DHQK + i0 + tid] = nn;

        const float mc = MCb[ch], mn = MCb[ch + 1];
        const float g = Gb[ch];
        const float decay = expf(g + mc - mn);
        __syncthreads();   // the previous chunk's steps have read the staged tiles
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int s = sl + 64 * u;
            if (s < L) {
                const float w = s < len ? expf(g - pa[u] + pig[u] - mn) : 0.f;
                if ((tid & 3) == 0) wsb[s] = w;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float f[8];
                    pk[u][h].get(f);
                    float *kd = ks + s * CKS + xp + 8 * h;
                    *reinterpret_cast<float4 *>(kd) = make_float4(f[0], f[1], f[2], f[3]);
                    *reinterpret_cast<float4 *>(kd + 4) = make_float4(f[4], f[5], f[6], f[7]);
                    pv[u][h].get(f);
                    float *vd = wvs + s * CKS + xp + 8 * h;
                    *reinterpret_cast<float4 *>(vd) = make_float4(w * f[0], w * f[1], w * f[2], w * f[3]);
                    *reinterpret_cast<float4 *>(vd + 4) = make_float4(w * f[4], w * f[5], w * f[6], w * f[7]);
                }
            }
        }
        __syncthreads();
        if (ch + 1 < NC) load_chunk(ch + 1);   // lands while the steps below run

#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int x = 0; x < 4; ++x) c[r][x] *= decay;
        nn *= decay;
        if (n_warp) {
            for (int s = 0; s < len; ++s) {
                const float4 kk = *reinterpret_cast<const float4 *>(ks + s * CKS + 4 * ty);
                const float4 vv = *reinterpret_cast<const float4 *>(wvs + s * CKS + 4 * tx);
                const float kr[4] = {kk.x, kk.y, kk.z, kk.w}, vr[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int x = 0; x < 4; ++x) c[r][x] = fmaf(kr[r], vr[x], c[r][x]);
                nn = fmaf(wsb[s], ks[s * CKS + tid], nn);
            }
        } else {
            for (int s = 0; s < len; ++s) {
                const float4 kk = *reinterpret_cast<const float4 *>(ks + s * CKS + 4 * ty);
                const float4 vv = *reinterpret_cast<const float4 *>(wvs + s * CKS + 4 * tx);
                const float kr[4] = {kk.x, kk.y, kk.z, kk.w}, vr[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int x = 0; x < 4; ++x) c[r][x] = fmaf(kr[r], vr[x], c[r][x]);
            }
        }
    }
    if (C_final && cols_in) {
#pragma unroll
        for (int r = 0; r < 4; ++r)
            if (ri + r < DHQK)
                *reinterpret_cast<float4 *>(C_final + ((size_t)bh * DHQK + ri + r) * DHV + cj) =
                    make_float4(c[r][0], c[r][1], c[r][2], c[r][3]);
    }
    if (n_final && n_warp && i0 + tid < DHQK) n_final[(size_t)bh * DHQK + i0 + tid] = nn;
    if (m_final && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0) m_final[bh] = MCb[NC];
}

// ---------------------------------------------------------------- output
// grid (BH, NC, ceil(DHV/32)), 256 threads.  Shared: P [L][L+1], q/k slices
// [L][33], v tile [L][33], C slice [32][33], per-row scalars.
template <typename T>
__global__ void __launch_bounds__(256)
output_simt_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                   const float *__restrict__ igate, const T *__restrict__ ogate,
                   const float *__restrict__ A, const float *__restrict__ Mtok, const float *__restrict__ MC,
                   const float *__restrict__ CS, const float *__restrict__ NS,
                   int S, int L, int NC, int DHQK, int DHV, T *__restrict__ h)
{
    griddep_wait();
    griddep_launch_dependents();
    extern __shared__ float sm[];
    const int LP = L + 1;
    float *P = sm;                       // [L][L+1]
    float *qs = P + L * LP;              // [L][33]
    float *ks2 = qs + L * 33;            // [L][33]   (k slice, later the v tile)
    float *cs = ks2 + L * 33;            // [32][33]
    float *ar = cs + 32 * 33;            // [L] a
    float *mr = ar + L;                  // [L] m
    float *ir = mr + L;                  // [L] i~
    float *sc = ir + L;                  // [L] sc
    float *den = sc + L;                 // [L]

    const int bh = blockIdx.x, ch = blockIdx.y, j0 = blockIdx.z * ST;
    const int t0 = ch * L, len = min(L, S - t0);
    const int tid = threadIdx.x;
    const float scale = rsqrtf((float)DHQK);
    const T *qb = q + ((size_t)bh * S + t0) * DHQK;
    const T *kb = k + ((size_t)bh * S + t0) * DHQK;
    const T *vb = v + ((size_t)bh * S + t0) * DHV;
    const float mc = MC[(size_t)bh * (NC + 1) + ch];

    for (int t = tid; t < L; t += blockDim.x) {
        const bool ok = t < len;
        ar[t] = ok ? A[(size_t)bh * S + t0 + t] : 0.f;
        mr[t] = ok ? ar[t] + fmaxf(mc, Mtok[(size_t)bh * S + t0 + t]) : 0.f;   // m = a + max(m_c, p)
        ir[t] = ok ? igate[(size_t)bh * S + t0 + t] : -INFINITY;
        sc[t] = ok ? expf(ar[t] + mc - mr[t]) : 0.f;
    }
    for (int e = tid; e < L * LP; e += blockDim.x) P[e] = 0.f;
    __syncthreads();

    // S = qh K^T over DHQK slices of 32
    for (int d0 = 0; d0 < DHQK; d0 += 32) {
        for (int e = tid; e < L * 32; e += blockDim.x) {
            const int t = e / 32, x = e % 32;
            const bool ok = t < len && d0 + x < DHQK;
            qs[t * 33 + x] = ok ? to_f32(qb[(size_t)t * DHQK + d0 + x]) * scale : 0.f;
            ks2[t * 33 + x] = ok ? to_f32(kb[(size_t)t * DHQK + d0 + x]) : 0.f;
        }
        __syncthreads();
        for (int e = tid; e < L * L; e += blockDim.x) {
            const int t = e / L, s = e % L;
            if (s <= t) {
                float acc = P[t * LP + s];
#pragma unroll 8
                for (int x = 0; x < 32; ++x) acc = fmaf(qs[t * 33 + x], ks2[s * 33 + x], acc);
                P[t * LP + s] = acc;
            }
        }
        __syncthreads();
    }
    // P = S * D, row sums
    for (int e = tid; e < L * L; e += blockDim.x) {
        const int t = e / L, s = e % L;
        if (s <= t && t < len) P[t * LP + s] *= expf(ar[t] - ar[s] + ir[s] - mr[t]);
        else P[t * LP + s] = 0.f;
    }
    __syncthreads();
    for (int t = tid; t < L; t += blockDim.x) {
        float r = 0.f;
        for (int s = 0; s <= t; ++s) r += P[t * LP + s];
        // inter-chunk normalizer term sc * n_c . qh
        float dn = 0.f;
        if (t < len) {
            const float *nc = NS + ((size_t)bh * NC + ch) * DHQK;
            for (int d = 0; d < DHQK; ++d) dn = fmaf(nc[d], to_f32(qb[(size_t)t * DHQK + d]), dn);
            dn *= scale * sc[t];
        }
        den[t] = r + dn;
    }
    __syncthreads();

    // num = sc * qh C_c + P V over the 32 columns of this tile.  Thread layout:
    // column x = tid % 32, rows t = tid / 32 + 8 r.
    const int x = tid & 31, ty = tid >> 5;
    const int RPT = (L + 7) / 8;     // rows per thread (L <= 128 -> <= 16)
    float acc[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) acc[r] = 0.f;
    const float *Cc = CS + ((size_t)bh * NC + ch) * DHQK * DHV;
    for (int d0 = 0; d0 < DHQK; d0 += 32) {
        for (int e = tid; e < L * 32; e += blockDim.x) {
            const int t = e / 32, xx = e % 32;
            const bool ok = t < len && d0 + xx < DHQK;
            qs[t * 33 + xx] = ok ? to_f32(qb[(size_t)t * DHQK + d0 + xx]) * scale : 0.f;
        }
        for (int e = tid; e < 32 * 32; e += blockDim.x) {
            const int d = e / 32, xx = e % 32;
            cs[d * 33 + xx] = (d0 + d < DHQK && j0 + xx < DHV) ? Cc[(size_t)(d0 + d) * DHV + j0 + xx] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const int t = ty + 8 * r;
            if (r < RPT && t < L) {
                float a2 = 0.f;
#pragma unroll 8
                for (int d = 0; d < 32; ++d) a2 = fmaf(qs[t * 33 + d], cs[d * 33 + x], a2);
                acc[r] = fmaf(sc[t], a2, acc[r]);
            }
        }
        __syncthreads();
    }
    for (int e = tid; e < L * 32; e += blockDim.x) {
        const int s = e / 32, xx = e % 32;
        ks2[s * 33 + xx] = (s < len && j0 + xx < DHV) ? to_f32(vb[(size_t)s * DHV + j0 + xx]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        const int t = ty + 8 * r;
        if (r < RPT && t < L) {
            float a2 = 0.f;
            for (int s = 0; s <= t; ++s) a2 = fmaf(P[t * LP + s], ks2[s * 33 + x], a2);
            acc[r] += a2;
        }
    }
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        const int t = ty + 8 * r;
        if (r < RPT && t < len && j0 + x < DHV) {
            const size_t off = ((size_t)bh * S + t0 + t) * DHV + j0 + x;
            const float o = ogate ? to_f32(ogate[off]) : 1.f;
            h[off] = from_f32<T>(o * acc[r] / fmaxf(fabsf(den[t]), expf(-mr[t])));
        }
    }
}

template <typename T>
static cudaError_t launch_fwd_simt_t(const FwdArgs &a, const FwdWorkspace &w, const PhaseMark &mark)
{
    const int L = a.chunk;
    dim3 g1(a.BH, (a.DHQK + CT - 1) / CT, (a.DHV + CT - 1) / CT);
    const size_t sm1 = sizeof(float) * (2 * (size_t)L * CKS + L);
    cudaError_t e = cudaSuccess;
    if (sm1 > 48 * 1024 && (e = ensure_dynamic_smem((const void *)carry_simt_kernel<T>, (int)sm1)) != cudaSuccess)
        return e;
    e = launch_kernel(carry_simt_kernel<T>, g1, dim3(256), sm1, a.stream, 1, (const T *)a.k, (const T *)a.v, a.igate,
                      w.A, w.G, w.MC, a.S, L, w.NC, a.DHQK, a.DHV, w.CS, w.NS, w.CS16, a.C_final, a.n_final,
                      a.m_final, a.C0, a.n0);
    if (e != cudaSuccess) return e;
    if ((e = mark(2)) != cudaSuccess) return e;   // the chunk scan is fused into the carry walk
    if ((e = mark(3)) != cudaSuccess) return e;
    if (!a.outputs) return cudaSuccess;   // the final state is complete after the carry walk
    dim3 g2(a.BH, w.NC, (a.DHV + ST - 1) / ST);
    const size_t sm2 = sizeof(float) * ((size_t)L * (L + 1) + 2 * (size_t)L * 33 + 32 * 33 + 5 * (size_t)L);
    if (sm2 > 48 * 1024 && (e = ensure_dynamic_smem((const void *)output_simt_kernel<T>, (int)sm2)) != cudaSuccess)
        return e;
    return launch_kernel(output_simt_kernel<T>, g2, dim3(256), sm2, a.stream, 1, (const T *)a.q, (const T *)a.k,
                         (const T *)a.v, a.igate, (const T *)a.ogate, w.A, w.M, w.MC, w.CS, w.NS, a.S, L, w.NC,
                         a.DHQK, a.DHV, (T *)a.h);
}

cudaError_t launch_fwd_simt(const FwdArgs &a, const FwdWorkspace &w, const PhaseMark &mark)
{
    return a.bf16 ? launch_fwd_simt_t<__nv_bfloat16>(a, w, mark) : launch_fwd_simt_t<float>(a, w, mark);
}

size_t simt_state_bytes(int BH, int NC, int DHQK, int DHV)
{
    return sizeof(float) * ((size_t)BH * NC * DHQK * DHV + (size_t)BH * NC * DHQK);
}

}  // namespace mlstm
