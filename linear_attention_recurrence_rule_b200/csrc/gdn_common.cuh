// Small device helpers shared by the library's kernels (not by the oracle).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Four consecutive elements starting at a 4-element-aligned address, as fp32.
__device__ __forceinline__ float4 load4(const float *p) {
    return *reinterpret_cast<const float4 *>(p);
}
__device__ __forceinline__ float4 load4(const __nv_bfloat16 *p) {
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(&u.x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&u.y);
    const float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
    return make_float4(a.x, a.y, b.x, b.y);
}

__device__ __forceinline__ float dot4(float4 a, float4 b) {
    return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
}

// d = a * b + c on two fp32 lanes at once (sm_100 packed FMA), each lane rounded
// as a scalar fmaf
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    unsigned long long ua, ub, uc, ud;
    memcpy(&ua, &a, 8);
    memcpy(&ub, &b, 8);
    memcpy(&uc, &c, 8);
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(ud) : "l"(ua), "l"(ub), "l"(uc));
    float2 d;
    memcpy(&d, &ud, 8);
    return d;
}

__device__ __forceinline__ float4 scale4(float4 a, float s) {
    return make_float4(a.x * s, a.y * s, a.z * s, a.w * s);
}

// Input prologue (the layer steps just before the rule): 1 / max(|x|, 1e-12)
// for an L2-normalised row with squared norm ss, and the sigmoid gates.
__device__ __forceinline__ float inv_l2norm(float ss) { return 1.f / fmaxf(sqrtf(ss), 1e-12f); }
__device__ __forceinline__ float gate_sigmoid(float x) { return 1.f / (1.f + expf(-x)); }
// Sigmoid of the layer steps (output gate, SiLU after the short convolution):
// hardware exponential and reciprocal, relative error ~1e-6 -- far inside the
// bf16 and fp32 output tolerances -- at a few instructions, so these steps stay
// memory-bound.  x is clamped at -80 so the reciprocal never sees an infinity.
__device__ __forceinline__ float layer_sigmoid(float x) {
    return __fdividef(1.f, 1.f + __expf(-fmaxf(x, -80.f)));
}
// log sigmoid(x) = min(x, 0) - log(1 + e^-|x|): finite at both ends
__device__ __forceinline__ float gate_log_sigmoid(float x) {
    return fminf(x, 0.f) - log1pf(expf(-fabsf(x)));
}

}  // namespace gdn
