// Element-type helpers for the kernels: loads and stores of q/k/v/out in fp32
// or bf16, always computing in fp32.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace rda {

template <typename T> struct Io;

template <> struct Io<float> {
    static __device__ __forceinline__ float ld(const float *p) { return *p; }
    static __device__ __forceinline__ void st(float *p, float x) { *p = x; }
    // four consecutive elements (16-byte aligned for fp32)
    static __device__ __forceinline__ float4 ld4(const float *p) {
        return *reinterpret_cast<const float4 *>(p);
    }
    static __device__ __forceinline__ void st4(float *p, float4 x) {
        *reinterpret_cast<float4 *>(p) = x;
    }
};

template <> struct Io<__nv_bfloat16> {
    static __device__ __forceinline__ float ld(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ void st(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }
    // four consecutive elements (8-byte aligned for bf16)
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

// Asynchronous global -> shared copies (cp.async), completed by a hardware
// wait (cp.async.wait_group): no spin loop.  16-byte copies need 16-byte
// aligned addresses on both sides.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

}  // namespace rda
