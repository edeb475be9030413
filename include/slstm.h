/* slstm.h -- C ABI of the sLSTM recurrence in libmlstm (sm_100a).
 *
 * The sLSTM cell ("xLSTM Guide: Extended LSTM Architecture & Matrix Memory",
 * section "The Twin Cells: sLSTM and mLSTM Mathematical Formulations", part 1,
 * the step-by-step recurrent equations) keeps one scalar memory c, normalizer n
 * and stabilizer m per cell and mixes the cells of a head through recurrent
 * matrices R.  Heads do not mix (the hu-po summary "Introduction to xLSTM
 * architecture", section "xLSTM Architecture Design": the gates pass through a
 * block-diagonal layer whose diagonal blocks, the heads, keep connectivity inside
 * a head), so R is block-diagonal: one DH x DH block per head and gate.
 *
 * Per batch item b, head e and cell j, at every step t:
 *   x~[g][j] = wx[b][t][g][e][j] + sum_k R[e][g][j][k] h[k]     (g = i, f, z, o; h = h_{t-1} of head e)
 *   lf       = f~                  (forget_sigmoid == 0: exponential forget gate)
 *            = log sigmoid(f~)     (forget_sigmoid != 0: sigmoid forget gate)
 *   m'  = max(lf + m, i~)
 *   c'  = exp(lf + m - m') c + exp(i~ - m') tanh(z~)
 *   n'  = exp(lf + m - m') n + exp(i~ - m')
 *   h'  = sigmoid(o~) c' / n'
 *
 * The input projection W x_t + b is not part of the recurrence: callers pass its
 * result as wx (one GEMM over the whole sequence, outside this call).
 */
#ifndef SLSTM_H
#define SLSTM_H

#include <stddef.h>

#include "mlstm.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Runs S steps of the recurrence for every batch item and head, starting from
 * the state (c, n, m, h) and leaving the state after the last step in place.
 *
 *   wx      [B][S][4][NH][DH] device, dtype dt: gate pre-activations W x_t + b,
 *           gate order i, f, z, o; aligned to its element size.
 *   R       [NH][4][DH][DH] device, dtype dt: recurrent weights, R[e][g] @ h_{t-1}
 *           (row j feeds cell j); 16-byte aligned.
 *   c, n, m, h  [B][NH][DH] device fp32 state, read at the start and overwritten
 *           with the state after step S (m is per cell).  A fresh sequence starts
 *           from all zeros.  4-byte aligned.
 *   h_out   [B][S][NH][DH] device, dtype dt: h of every step, or NULL (state only).
 *   DH      32, 64, 128, 192 or 256 (the cells of one head are spread over a thread-
 *           block cluster of DH / 32 CTAs).
 *   status  device uint32 or NULL, 4-byte aligned: set to MLSTM_ERR_TIMEOUT if one of the
 *           kernel's bounded waits (2 s each, for the other CTAs' h of a step) gave up; the
 *           outputs are then not valid.  The call never clears it.
 *   stream  cudaStream_t, or NULL for the default stream.  Asynchronous.
 *
 * Arithmetic is fp32 (bf16 inputs are widened exactly; h_out is rounded to dt).
 * All pointers are caller-owned; nothing is allocated.  Errors: invalid pointers,
 * sizes or alignment return MLSTM_ERR_INVALID_ARG, an unsupported DH or dtype
 * MLSTM_ERR_UNSUPPORTED, a failed launch MLSTM_ERR_CUDA, all before or at launch.
 * B == 0 or S == 0 returns MLSTM_OK without a launch (and without looking at the
 * pointers); the state is left as it is.
 */
mlstm_status slstm_fwd(const void *wx, const void *R, mlstm_dtype dt, int B, int S, int NH, int DH,
                       int forget_sigmoid, float *c, float *n, float *m, float *h, void *h_out,
                       unsigned int *status, void *stream);

/* The batch items one cluster carries through the recurrence for this shape on
 * the current device (1, 2, 4 or 8), or 0 for an unsupported shape: the launch
 * uses NH * ceil(B / that) clusters of DH / 32 CTAs. */
int slstm_batch_per_cluster(int B, int NH, int DH, mlstm_dtype dt);

#ifdef __cplusplus
}
#endif

#endif /* SLSTM_H */
