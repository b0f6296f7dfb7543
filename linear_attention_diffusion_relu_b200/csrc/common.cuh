// Shared device helpers for the linear-attention kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sana {

// phi = ReLU on a packed pair of bf16 values. max(x, 0) is exact in bf16, so
// the feature map never rounds ("08_sana高效高分辨率生成", "Linear Attention 的原理").
__device__ __forceinline__ uint32_t relu_bf16x2(uint32_t packed) {
    __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&packed);
    __nv_bfloat162 z = __float2bfloat162_rn(0.0f);
    __nv_bfloat162 r = __hmax2(v, z);
    return *reinterpret_cast<uint32_t*>(&r);
}

__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t packed) {
    __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&packed);
    return __bfloat1622float2(v);
}

__device__ __forceinline__ uint32_t float2_to_bf16x2(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
}

// streaming 16-byte global load that bypasses L1 allocation (inputs are read once)
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

__device__ __forceinline__ void stg_stream(void* p, uint4 v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};"
                 :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

}  // namespace sana
