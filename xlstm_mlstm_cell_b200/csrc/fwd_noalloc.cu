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

#include <cudaTypedefs.h>

#include <mutex>

namespace {

constexpr size_t kScratchBytes = (size_t)MLSTM_FWD_NOALLOC_MAX_BYTES;

__device__ __align__(256) unsigned char g_fwd_scratch[kScratchBytes];

// The array's device address per device, with the identity of the context it was looked up in:
// after the primary context is destroyed and created again (cudaDeviceReset), the module is
// loaded anew and the address is looked up again.
struct Slot {
    void *ptr = nullptr;
    unsigned long long ctx = 0;
    bool ctx_known = false;
};
constexpr int kMaxDevices = 64;
Slot g_slots[kMaxDevices];
std::mutex g_scratch_lock;

// Unique id of the context current on this thread (false when none is current or the driver
// does not offer the query).
bool current_context_id(unsigned long long *id)
{
    static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static bool looked_up = false;
    if (!looked_up) {   // under g_scratch_lock
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
        looked_up = true;
    }
    if (!get_current || !get_id) return false;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the scratch array on the current device: looked up with
// cudaGetSymbolAddress the first time on a device (and again if that device's context has been
// replaced since), then taken from the cache.
cudaError_t scratch_address(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> guard(g_scratch_lock);
    Slot &s = g_slots[dev];
    unsigned long long id = 0;
    const bool have_id = current_context_id(&id);
    if (s.ptr && s.ctx_known && have_id && s.ctx == id) {
        *out = s.ptr;
        return cudaSuccess;
    }
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_fwd_scratch);   // creates the device's primary context if needed
    if (e != cudaSuccess) {
        s = Slot();
        return e;
    }
    s.ptr = p;
    s.ctx_known = current_context_id(&s.ctx);
    *out = p;
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

extern "C" mlstm_status mlstm_fwd_noalloc_status(void *stream)
{
    void *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return MLSTM_ERR_CUDA;
    return mlstm_fwd_status(scratch, stream);
}
