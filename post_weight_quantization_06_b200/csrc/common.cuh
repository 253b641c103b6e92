// Shared device helpers of libgptq: the sticky status word, launch checks, small math.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <math.h>

#include <atomic>

#include "gptq.h"

namespace gptq {

// ---------------------------------------------------------------------------------------
// Sticky device status word: the first device-side error wins; read and cleared by
// gptq_sync_status(). One copy per device (a __device__ variable lives in every context).
// ---------------------------------------------------------------------------------------
struct DevStatus {
    int code;
    int pad;
    long long info;
};

__device__ DevStatus g_status;

__device__ __forceinline__ void report(int code, long long info) {
    if (atomicCAS(&g_status.code, 0, code) == 0) {
        atomicExch(reinterpret_cast<unsigned long long *>(&g_status.info),
                   static_cast<unsigned long long>(info));
    }
}

__device__ __forceinline__ bool finitef(float x) { return isfinite(x); }

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

inline int ceil_div(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }

// Multiprocessor count of the current device, looked up once per device.
inline int device_sm_count() {
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int v = cache[dev].load(std::memory_order_relaxed);
    if (v > 0) return v;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v < 1)
        v = 148;
    cache[dev].store(v, std::memory_order_relaxed);
    return v;
}

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current device unless this
// call site already set at least that much there (`set_bytes` holds the value per device).
template <typename K>
inline void smem_limit_once(K *kernel, int bytes, std::atomic<int> *set_bytes) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    if (set_bytes[dev].load(std::memory_order_acquire) >= bytes) return;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) ==
        cudaSuccess) {
        int prev = set_bytes[dev].load();
        while (prev < bytes && !set_bytes[dev].compare_exchange_weak(prev, bytes)) {}
    }
}
#define GPTQ_SMEM_LIMIT(kernel, bytes)                                  \
    do {                                                                \
        static std::atomic<int> gptq_smem_set_[64];                     \
        ::gptq::smem_limit_once(kernel, (int)(bytes), gptq_smem_set_);  \
    } while (0)

// Every kernel launch of the library is followed by launch_status(), which also counts it
// (read with gptq_launch_count()).
inline std::atomic<unsigned long long> &launch_counter() {
    static std::atomic<unsigned long long> c{0};
    return c;
}

inline int launch_status() {
    launch_counter().fetch_add(1, std::memory_order_relaxed);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

// Programmatic dependent launch: a kernel launched with `pdl` may start while the previous
// kernel of its stream is still running; it must call pdl_wait_prev() before touching what
// that kernel writes. pdl_launch_next() lets the next such kernel start. Both are no-ops for a
// kernel launched without the attribute.
__device__ __forceinline__ void pdl_launch_next() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait_prev() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline int launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                         cudaStream_t s, bool pdl, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
    const int st = launch_status();
    return e == cudaSuccess ? st : GPTQ_ERR_CUDA;
}

#define GPTQ_CHECK_LAUNCH()                  \
    do {                                     \
        int _s = ::gptq::launch_status();    \
        if (_s != GPTQ_OK) return _s;        \
    } while (0)

}  // namespace gptq
