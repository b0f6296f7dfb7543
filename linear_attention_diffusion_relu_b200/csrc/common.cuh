// Shared device helpers for the linear-attention kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ptx.cuh"

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

// phi on a pair of values, with packed fp32x2 arithmetic where a step allows.
// ELU+1 = max(x, 0) + e^min(x, 0): x + 1 above zero, e^x at or below, with
// e^y = 2^(y log2 e) on the special-function unit (its relative error is far
// below the bf16 hi/lo split's). cos: Cody-Waite additive range reduction
// (W. J. Cody and W. Waite, "Software Manual for the Elementary Functions",
// 1980) by the nearest multiple of 2*pi, with 2*pi carried as a float head
// plus a float tail and both products folded in by fma, then the hardware
// cosine (__cosf), whose error bound holds on [-pi, pi]. Inputs are bf16
// activations (|x| of order 10 at most), where the reduced argument is
// accurate to a few float ulps.
template <int FM>
__device__ __forceinline__ float2 feature_f32x2(float2 x) {
    if constexpr (FM == kFeatureElu1) {
        constexpr float kLog2e = 1.4426950408889634f;
        const float2 t = __fmul2_rn(make_float2(fminf(x.x, 0.0f), fminf(x.y, 0.0f)), make_float2(kLog2e, kLog2e));
        return __fadd2_rn(make_float2(fmaxf(x.x, 0.0f), fmaxf(x.y, 0.0f)),
                          make_float2(ptx::ex2_approx(t.x), ptx::ex2_approx(t.y)));
    } else if constexpr (FM == kFeatureCos) {
        constexpr float kInv2Pi = 0.159154943091895336f;          // 1 / (2 pi), rounded
        constexpr float k2PiHi = 6.28318548202514648f;            // float(2 pi)
        constexpr float k2PiLo = -1.74845553146951880e-07f;       // 2 pi - float(2 pi)
        // k = nearest integer to x / (2 pi): adding and subtracting 1.5 * 2^23
        // rounds any |q| < 2^22 to an integer (ties to even) on the FMA pipe
        constexpr float kRound = 12582912.0f;                     // 1.5 * 2^23
        const float2 q = __fmul2_rn(x, make_float2(kInv2Pi, kInv2Pi));
        const float2 k = __fadd2_rn(__fadd2_rn(q, make_float2(kRound, kRound)), make_float2(-kRound, -kRound));
        float2 r = __ffma2_rn(k, make_float2(-k2PiHi, -k2PiHi), x);   // x - k * head
        r = __ffma2_rn(k, make_float2(-k2PiLo, -k2PiLo), r);          // ... - k * tail
        return make_float2(__cosf(r.x), __cosf(r.y));
    } else {
        return make_float2(fmaxf(x.x, 0.0f), fmaxf(x.y, 0.0f));
    }
}

// phi of a packed bf16 pair, split into bf16 hi and lo parts: hi = bf16(phi),
// lo = bf16(phi - hi), so hi + lo carries phi to ~2^-17 relative and products
// on the tensor cores keep fp32-grade accuracy (ReLU needs no split: it is
// exact in bf16). phi - hi is exact in fp32 and comes from one packed fma.
template <int FM>
__device__ __forceinline__ void feature_split_bf16x2(uint32_t packed, uint32_t& hi, uint32_t& lo) {
    const float2 p = feature_f32x2<FM>(bf16x2_to_float2(packed));
    __nv_bfloat162 h = __floats2bfloat162_rn(p.x, p.y);
    const float2 d = __ffma2_rn(__bfloat1622float2(h), make_float2(-1.0f, -1.0f), p);
    __nv_bfloat162 l = __floats2bfloat162_rn(d.x, d.y);
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
