// tc_fwd.h -- what the kernels of the tensor-core forward pass share: their launch parameters and
// the host-side launchers of the walk over CTA pairs.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace mlstm {
namespace tcfwd {

struct Params {
    int S, L, NC, R, NSEG, DK, DV, BH;
    const float *A, *Mtok, *ig, *MC, *G, *GP, *SGb;
    float *DC, *DN;
    const __nv_bfloat16 *o;
    __nv_bfloat16 *h;
    uint32_t *status;
};

// [BH][S][D] bf16 tensor map with boxes of 64 columns x `rows` tokens x 1 head, 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *base, int D, int S, int BH, int rows);

// The walk over CTA pairs (walk_pair.cu): taken for these head sizes and chunk length.
bool walk_pair_supported(int DK, int DV, int L);
// Launches it; q, k, v the bf16 inputs [BH][S][DK | DV].
cudaError_t launch_walk_pair(const Params &p, const void *q, const void *k, const void *v, cudaStream_t stream);

}  // namespace tcfwd
}  // namespace mlstm
