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

// Feature maps phi ("08_sana高效高分辨率生成", "Linear Attention 的原理": ReLU, with
// ELU+1 and cos named as alternatives). ELU is taken with alpha = 1.
enum : int { kFeatureRelu = 0, kFeatureElu1 = 1, kFeatureCos = 2 };

// cos(x) for moderate |x|: Cody-Waite additive range reduction (W. J. Cody and
// W. Waite, "Software Manual for the Elementary Functions", 1980) by the
// nearest multiple of 2*pi, with 2*pi carried as a float head plus a float
// tail and both products folded in by fma, then the hardware cosine
// (__cosf), whose error bound holds on [-pi, pi]. Inputs are bf16 activations
// (|x| of order 10 at most), where the reduced argument is accurate to a few
// float ulps.
__device__ __forceinline__ float cos_reduced(float x) {
    constexpr float kInv2Pi = 0.159154943091895336f;          // 1 / (2 pi), rounded
    constexpr float k2PiHi = 6.28318548202514648f;            // float(2 pi)
    constexpr float k2PiLo = -1.74845553146951880e-07f;       // 2 pi - float(2 pi)
    const float k = rintf(x * kInv2Pi);
    float r = fmaf(-k, k2PiHi, x);
    r = fmaf(-k, k2PiLo, r);
    return __cosf(r);
}

// ELU+1 uses the hardware exponential (__expf) on x <= 0, where its relative
// error is far below the bf16 hi/lo split's.
template <int FM>
__device__ __forceinline__ float feature_f32(float x) {
    if constexpr (FM == kFeatureElu1) return x > 0.0f ? x + 1.0f : __expf(x);
    else if constexpr (FM == kFeatureCos) return cos_reduced(x);
    else return fmaxf(x, 0.0f);
}

// phi of a packed bf16 pair, split into bf16 hi and lo parts: hi = bf16(phi),
// lo = bf16(phi - hi), so hi + lo carries phi to ~2^-17 relative and products
// on the tensor cores keep fp32-grade accuracy (ReLU needs no split: it is
// exact in bf16).
template <int FM>
__device__ __forceinline__ void feature_split_bf16x2(uint32_t packed, uint32_t& hi, uint32_t& lo) {
    const float2 x = bf16x2_to_float2(packed);
    const float a = feature_f32<FM>(x.x);
    const float b = feature_f32<FM>(x.y);
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    const float2 hf = __bfloat1622float2(h);
    __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
    hi = *reinterpret_cast<uint32_t*>(&h);
    lo = *reinterpret_cast<uint32_t*>(&l);
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
