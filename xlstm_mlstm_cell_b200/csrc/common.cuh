// common.cuh -- small device helpers shared by the libmlstm kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#define MLSTM_DEVINL __device__ __forceinline__

namespace mlstm {

// Element loads/stores for the two supported element types of q, k, v, o and h.
MLSTM_DEVINL float to_f32(float x) { return x; }
MLSTM_DEVINL float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> MLSTM_DEVINL T from_f32(float x);
template <> MLSTM_DEVINL float from_f32<float>(float x) { return x; }
template <> MLSTM_DEVINL __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Two floats rounded to bf16 (nearest even) as one 32-bit word, the first in the low half.
MLSTM_DEVINL uint32_t bf16x2_bits(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// A float as two bf16: its rounding and the rounding of the residue (about 16 significant bits).
MLSTM_DEVINL void bf16_parts(float x, __nv_bfloat16 &hi, __nv_bfloat16 &lo)
{
    hi = __float2bfloat16_rn(x);
    lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}

// Four consecutive elements as float (16-byte aligned for float, 8 for bf16).
MLSTM_DEVINL float4 load4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
MLSTM_DEVINL float4 load4(const __nv_bfloat16 *p)
{
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(&u.x);
    __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&u.y);
    float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    return make_float4(fa.x, fa.y, fb.x, fb.y);
}
MLSTM_DEVINL void store4(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }
MLSTM_DEVINL void store4(__nv_bfloat16 *p, float4 v)
{
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
    __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t *>(&a);
    u.y = *reinterpret_cast<uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(p) = u;
}

// logsigmoid(x) = -log(1 + exp(-x)) without overflow, through CUDA's own expf/log1pf.
MLSTM_DEVINL float log_sigmoid(float x)
{
    return x >= 0.f ? -log1pf(expf(-x)) : x - log1pf(expf(x));
}

MLSTM_DEVINL float warp_sum(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Programmatic dependent launch.  Every kernel of the library is launched with programmatic
// stream serialization, so that its launch and its prologue (barrier set-up, TMEM allocation,
// descriptor prefetch: nothing that touches global memory) overlap the tail of the kernel before
// it.  griddep_wait() returns once the preceding grid has completed and its memory is visible;
// it must come before the kernel's first global load or store.  griddep_launch_dependents()
// lets the next kernel in the stream start launching (it still waits for this one to finish).
// Both are no-ops for a kernel launched without the attribute.
MLSTM_DEVINL void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
MLSTM_DEVINL void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" :::); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                                 int cluster_x, Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    int na = 0;
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
    if (cluster_x > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = (unsigned)cluster_x;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = (unsigned)na;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// One lock for the library's host-side caches (the per-kernel shared-memory limits set so far,
// the sLSTM kernel's cluster capacity, the tensor-map encoder), so that host threads may call the
// library at the same time.  An inline function's static is one object across translation units.
inline std::mutex &host_cache_mutex()
{
    static std::mutex m;
    return m;
}

// Raises a kernel's dynamic shared-memory limit once per (kernel, device), so that
// launches stay free of attribute calls after the first one.  Thread-safe.
inline cudaError_t ensure_dynamic_smem(const void *kernel, int bytes)
{
    struct Entry { const void *fn; int dev; int bytes; };
    static Entry reg[128];
    static int used = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
    std::lock_guard<std::mutex> guard(host_cache_mutex());
    for (int i = 0; i < used; ++i)
        if (reg[i].fn == kernel && reg[i].dev == dev && reg[i].bytes >= bytes) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    for (int i = 0; i < used; ++i)
        if (reg[i].fn == kernel && reg[i].dev == dev) { reg[i].bytes = bytes; return cudaSuccess; }
    if (used < 128) reg[used++] = Entry{kernel, dev, bytes};
    return cudaSuccess;
}

// The SM count of the current device, looked up once per device.  Thread-safe.
inline cudaError_t sm_count(int *n)
{
    static int cached[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> guard(host_cache_mutex());
    if (dev >= 0 && dev < 64 && cached[dev] > 0) {
        *n = cached[dev];
        return cudaSuccess;
    }
    if ((e = cudaDeviceGetAttribute(n, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) cached[dev] = *n;
    return cudaSuccess;
}

}  // namespace mlstm
