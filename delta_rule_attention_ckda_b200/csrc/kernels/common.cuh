// Shared device helpers for the CKDA kernels (sm_100a).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace ckda {

// Device error word of this GPU. Bit 0: a bounded wait ran out.
// Written by kernels with atomicOr, read and cleared by ckda_get_device_error.
__device__ unsigned int g_error_word = 0;
constexpr unsigned int kErrTimeout = 1u;

__device__ __forceinline__ void report_error(unsigned int bits) {
    atomicOr(&g_error_word, bits);
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ float ld_in(const T* p) { return to_f32(__ldg(p)); }

// Four consecutive input elements starting at a 4-element-aligned index.
__device__ __forceinline__ float4 ld_in4(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }
__device__ __forceinline__ float4 ld_in4(const __nv_bfloat16* p) {
    uint2 raw = __ldg(reinterpret_cast<const uint2*>(p));
    __nv_bfloat162 lo = *reinterpret_cast<__nv_bfloat162*>(&raw.x);
    __nv_bfloat162 hi = *reinterpret_cast<__nv_bfloat162*>(&raw.y);
    float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
    return make_float4(a.x, a.y, b.x, b.y);
}

}  // namespace ckda
