// Device helpers shared by the tensor-core prefill kernels: TMEM row loads and
// stores, bf16 hi/lo operand splitting, and the chunk-local decay scan.
#pragma once

#include "tc_primitives.cuh"

namespace gdn {
namespace tcc {

using namespace tc;

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float *v) {
    float a[16], b[16];
    tmem_ld16(taddr, a);
    tmem_ld16(taddr + 16, b);
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        v[j] = a[j];
        v[16 + j] = b[j];
    }
}
__device__ __forceinline__ void tmem_st16w(uint32_t taddr, const uint32_t (&w)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 "
        "[%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]),
        "r"(w[8]), "r"(w[9]), "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]),
        "r"(w[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st32f(uint32_t taddr, const float *v) {
    float a[16], b[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        a[j] = v[j];
        b[j] = v[16 + j];
    }
    tmem_st16(taddr, a);
    tmem_st16(taddr + 16, b);
}
// 32 floats -> hi and lo bf16 words (16 each), packed in element order.
__device__ __forceinline__ void split_pack32(const float *f, uint32_t (&hi)[16],
                                             uint32_t (&lo)[16]) {
#pragma unroll
    for (int w = 0; w < 16; ++w) {
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(f[2 * w], f[2 * w + 1]);
        const float2 hf = __bfloat1622float2(h2);
        hi[w] = *reinterpret_cast<const uint32_t *>(&h2);
        lo[w] = pack_bf16x2(f[2 * w] - hf.x, f[2 * w + 1] - hf.y);
    }
}
// 8 floats -> hi chunk (bf16(x)) and lo chunk (bf16(x - hi)) at two shared addresses.
__device__ __forceinline__ void st_chunk_hilo(uint32_t hi_addr, uint32_t lo_addr, const float *f) {
    float hi[8], lo[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        hi[e] = __bfloat162float(__float2bfloat16_rn(f[e]));
        lo[e] = f[e] - hi[e];
    }
    st_shared_bf16x8(hi_addr, hi);
    st_shared_bf16x8(lo_addr, lo);
}

// Chunk-local running sum of g over 64 tokens by one warp: lane l owns
// tokens 2l and 2l+1 (rows >= L count as g = 0).  Inputs are the two g values
// of the lane; returns G(2l), G(2l+1).
__device__ __forceinline__ float2 warp_decay_scan(float g0, float g1) {
    const int lane = threadIdx.x & 31;
    float x = g0 + g1;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    return make_float2(x - g1, x);
}
__device__ __forceinline__ float2 load_g_pair(const float *g, int64_t s0, int L, int HV, int h) {
    const int lane = threadIdx.x & 31;
    const int t0 = 2 * lane, t1 = 2 * lane + 1;
    return make_float2(t0 < L ? g[(s0 + t0) * HV + h] : 0.f, t1 < L ? g[(s0 + t1) * HV + h] : 0.f);
}

}  // namespace tcc
}  // namespace gdn
