// Shared device helpers for the KDA kernels (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "kda.h"

namespace kda {

// Device status word: the first error recorded since the last
// kda_check_device_status() (0 = none). One per device (module global).
__device__ unsigned int g_status;

__device__ __forceinline__ void record_status(unsigned int code) {
    atomicCAS(&g_status, 0u, code);
}

// Text behind the most recent KDA_ERR_CUDA (static storage), read by kda_last_cuda_error.
inline std::atomic<const char *> &last_error_text() {
    static std::atomic<const char *> text{"no error"};
    return text;
}
// Record a failed CUDA call (or another failure reported as KDA_ERR_CUDA) and return it.
inline kda_status fail_cuda(cudaError_t e) {
    last_error_text().store(cudaGetErrorString(e));
    return KDA_ERR_CUDA;
}
inline kda_status fail_text(const char *msg) {
    last_error_text().store(msg);
    return KDA_ERR_CUDA;
}
// Status of the launch just issued.
inline kda_status launch_result() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? KDA_OK : fail_cuda(e);
}

// Raise a kernel's dynamic shared-memory limit (and prefer the largest shared
// memory carveout) on the current device once.
// The attribute is per device, so a process that drives several GPUs keeps one
// bit per device ordinal in `done` (ordinals >= 64 set it on every call).
inline kda_status set_smem_limit_once(const void *fn, int bytes, std::atomic<unsigned long long> &done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail_cuda(e);
    const unsigned long long bit = dev < 64 ? (1ull << dev) : 0ull;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return KDA_OK;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return fail_cuda(e);
    done.fetch_or(bit, std::memory_order_release);
    return KDA_OK;
}

// Element type traits for the q/k/v/o arrays.
template <typename T> struct IO;
template <> struct IO<float> {
    static __device__ __forceinline__ float ld(const float *p) { return *p; }
    static __device__ __forceinline__ void st(float *p, float x) { *p = x; }
    // four consecutive elements
    static __device__ __forceinline__ float4 ld4(const float *p) {
        return *reinterpret_cast<const float4 *>(p);
    }
    static __device__ __forceinline__ void st4(float *p, float4 x) {
        *reinterpret_cast<float4 *>(p) = x;
    }
};
template <> struct IO<__nv_bfloat16> {
    static __device__ __forceinline__ float ld(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ void st(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }
    static __device__ __forceinline__ float4 ld4(const __nv_bfloat16 *p) {
        uint2 u = *reinterpret_cast<const uint2 *>(p);
        __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162 *>(&u.x);
        __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162 *>(&u.y);
        float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
        return make_float4(fa.x, fa.y, fb.x, fb.y);
    }
    static __device__ __forceinline__ void st4(__nv_bfloat16 *p, float4 x) {
        __nv_bfloat162 a = __floats2bfloat162_rn(x.x, x.y);
        __nv_bfloat162 b = __floats2bfloat162_rn(x.z, x.w);
        uint2 u;
        u.x = *reinterpret_cast<uint32_t *>(&a);
        u.y = *reinterpret_cast<uint32_t *>(&b);
        *reinterpret_cast<uint2 *>(p) = u;
    }
};

// Streaming 128-bit global accesses for state tiles that are touched once.
__device__ __forceinline__ float4 ld_stream(const float *p) {
    float4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
                 : "l"(p));
    return r;
}
__device__ __forceinline__ float4 ld_plain(const float *p) {
    return *reinterpret_cast<const float4 *>(p);
}
__device__ __forceinline__ void st_stream(float *p, float4 v) {
    asm volatile("st.global.cs.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(p), "f"(v.x), "f"(v.y),
                 "f"(v.z), "f"(v.w)
                 : "memory");
}

}  // namespace kda
