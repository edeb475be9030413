// bwd_tc.h -- the gradient products of the backward pass on the tensor cores (bwd_tc.cu): what the
// CUDA-core backward (bwd_simt.cu) hands them.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mlstm {
namespace bwdtc {

struct Args {
    int BH, S, L, NC, DK, DV, NTK;
    // gate preprocessing [BH][S] (A: chunk-local cumulative log decay, P: chunk-local prefix maximum
    // of i~ - A), chunk stabilizers MC [BH][NC + 1] and log decay sums G [BH][NC]; i~ [BH][S]
    const float *A, *P, *MC, *G, *ig;
    const float *DD;                        // gradient of the denominator [BH][S]
    const float *NS, *GN;                   // n at the chunk starts, gradient of n at the chunk ends [BH][NC][DK]
    const __nv_bfloat16 *q, *k, *v;         // inputs [BH][S][DK | DV]
    // bf16 copies of the fp32 intermediates: chunk-start states C16 [BH][NC][2][DK][DV], scores
    // A16 [BH][NC][2][L][L] and the read-out numerator's gradient g16 [BH][2][S][DV] as two parts
    // each (the bf16 value and the bf16 of its rounding residue: together about 16 significant
    // bits; products that need only the value read part 0), chunk-end state gradients G16
    // [BH][NC][DK][DV] and dS16 [BH][NC][L][L]
    const __nv_bfloat16 *C16, *G16, *g16, *dS16, *A16;
    __nv_bfloat16 *dq, *dk, *dv;            // outputs [BH][S][DK | DV]
    // partial q . dq^inter (the inter-chunk term alone), k . dk and k . dk^inter per 32 columns
    // [BH][S][NTK], for the gate gradients
    float *QD, *KD, *KI;
    // the read-out numerator: dh, o (NULL without an output gate) [BH][S][DV], N = max(|den|,
    // exp(-m)) [BH][S]; writes g (its two bf16 parts, g16w), do (when o is given) and the partial
    // row sums of g . hh per 64 value columns DOTP [BH][S][NJT]
    const __nv_bfloat16 *dh, *o;
    const float *NRM;
    float *DOTP;
    __nv_bfloat16 *g16w, *dog;
    int NJT;
    // sc_t g_t as two bf16 parts [BH][2][S][DV] (written by the numerator's epilogue, read by the
    // state-gradient walk), and that walk's output, the chunk-end state gradients (the array G16)
    __nv_bfloat16 *sg16, *G16w;
    // the forward carry (launch_carry): w_s k_s as two bf16 parts [BH][2][S][DK] (written, then
    // read), and its outputs, the chunk-start states as two bf16 parts (the array C16 above) and n
    __nv_bfloat16 *wk16, *C16w;
    float *NSw;
    // the scores and dS (launch_scores, launch_ds): write DEN, NRM [BH][S] and A16 (two parts);
    // DD [BH][S], dS16 and the read-out's dn_c GNw [BH][NC][DK]
    float *DENw, *NRMw, *DDw, *GNw;
    // dS also writes RECT [BH][S]: sum of dA_ts A_ts over the pairs s < j <= t of token j's chunk;
    // the state-gradient walk writes the partial sums of E_c = exp(g_c + m_c - m_{c+1})
    // (<G_end, C_c> + <dn_end, n_c>) [BH][NC][NEP], NEP = 4 (DK / 128) (DV / 64) (a warp of each tile)
    float *RECTw, *EPw;
    int NEP;
    __nv_bfloat16 *A16w, *dS16w;
    uint32_t *status;
    cudaStream_t stream;
};

// bf16 inputs with chunk 64 or 128 and head sizes that are multiples of 128.
bool supported(int DK, int DV, int L);
// The dq, dk and dv products of every chunk (three launches on a.stream).
cudaError_t launch(const Args &a);
// The read-out numerator of every chunk, num = sc qh C_c + A V, and what follows from it (one launch).
cudaError_t launch_num(const Args &a);
// The state gradients at the chunk ends, G_end (bf16), from the read-out's dC_c = (sc qh)^T g of every
// chunk, and the normalizer's in GN (in place: dn_c in, the chunk-end gradient out), by a reverse walk
// over the chunks per state tile with dC_c on tcgen05 (one launch).
cudaError_t launch_gstate(const Args &a);
// The chunk's scores A = D * (qh K^T) (two bf16 parts), den and N (one launch).
cudaError_t launch_scores(const Args &a);
// dden, dS = (g V^T + dden) * D (bf16) and the read-out's dn_c (one launch; after the numerator).
cudaError_t launch_ds(const Args &a);
// The forward pass's chunk-start states C_c (as two bf16 parts) and n_c from the zero state: w_s k_s
// as two bf16 parts, then a walk over the chunks per state tile with each chunk's contribution
// sum_s (w_s k_s) v_s^T on tcgen05 and the fp32 state in registers (two launches).
cudaError_t launch_carry(const Args &a);

}  // namespace bwdtc
}  // namespace mlstm
