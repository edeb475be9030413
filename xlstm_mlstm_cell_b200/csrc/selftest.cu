// selftest.cu -- a self-test of the library's failure detection.
//
// Every wait of the tensor-core kernels on an mbarrier is bounded: after
// WAIT_LIMIT_NS it gives up, sets the call's status word to a timeout and the CTA
// leaves through its normal teardown, so a stalled pipeline ends the call with
// MLSTM_ERR_TIMEOUT (read back by mlstm_fwd_status) instead of hanging the GPU.
// The kernel here exercises exactly that path on purpose: one CTA waits, through
// the same bounded wait, on a barrier that nothing ever completes.
#include "mlstm.h"
#include "common.cuh"
#include "tc_common.cuh"

namespace mlstm {
using namespace tc;

__global__ void __launch_bounds__(32) selftest_wait_timeout_kernel(uint32_t *status)
{
    __shared__ uint64_t bar;
    __shared__ uint32_t abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);          // one arrival expected, none will come
        abort_flag = 0u;
        *status = 0u;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        WaitCtx wc{&abort_flag, status};
        mbar_wait(&bar, 0u, wc);     // gives up after WAIT_LIMIT_NS and records the timeout
    }
}

}  // namespace mlstm

extern "C" mlstm_status mlstm_selftest_wait_timeout(void *workspace, void *stream)
{
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MLSTM_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    mlstm::selftest_wait_timeout_kernel<<<1, 32, 0, st>>>(static_cast<uint32_t *>(workspace));
    return cudaGetLastError() == cudaSuccess ? MLSTM_OK : MLSTM_ERR_CUDA;
}
