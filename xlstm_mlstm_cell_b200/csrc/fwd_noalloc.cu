// fwd_noalloc.cu -- mlstm_fwd for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc or any allocating routine: code that runs
// inside a host framework which owns all device memory and hands out none for
// scratch (plugin and extension interfaces), and latency-critical paths where an
// allocation's implicit device synchronization is not acceptable.  For them this
// file keeps the forward pass's scratch memory in one statically sized device
// array that the library itself carries.  The caller still provides inputs and
// outputs; only the workspace comes from here.
//
// The array lives in the module image as an uninitialized __device__ variable:
// every GPU on which the library's module is loaded holds it until the process
// exits.  In host code its name only stands for the device variable (using it as
// an address would be wrong), so its device address is looked up with
// cudaGetSymbolAddress, once per device, with that device current, and handed to
// the kernels like any caller-owned workspace.
#include "mlstm.h"
#include "mlstm_internal.h"

#include <mutex>

namespace {

constexpr size_t kScratchBytes = (size_t)MLSTM_FWD_NOALLOC_MAX_BYTES;

__device__ __align__(256) unsigned char g_fwd_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void *g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_lock;

// Device address of the scratch array on the current device (looked up once per device).
cudaError_t scratch_address(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> guard(g_scratch_lock);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_fwd_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" mlstm_status mlstm_fwd_noalloc(const void *q, const void *k, const void *v, const float *igate,
                                          const float *fgate, const void *ogate, mlstm_dtype dt, int B, int NH,
                                          int S, int DHQK, int DHV, int chunk, void *h_out, float *C_final,
                                          float *n_final, float *m_final, void *stream)
{
    if (B < 0 || NH < 0 || S < 0) return MLSTM_ERR_INVALID_ARG;
    const size_t need = mlstm_fwd_workspace_size(B, NH, S, DHQK, DHV, chunk, dt);
    if (need == 0) return MLSTM_ERR_UNSUPPORTED;
    if (need > kScratchBytes) return MLSTM_ERR_WORKSPACE;   // larger than the built-in scratch
    void *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return MLSTM_ERR_CUDA;
    return mlstm_fwd(q, k, v, igate, fgate, ogate, dt, B, NH, S, DHQK, DHV, chunk, h_out, C_final, n_final,
                     m_final, scratch, kScratchBytes, stream);
}
