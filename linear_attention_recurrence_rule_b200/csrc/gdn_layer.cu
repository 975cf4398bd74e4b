// The layer steps around the rule: a short causal convolution on the values
// before it and a sigmoid gate on its read-out after it ("Qwen3-Next 80B-A3B --
// The Evolving Transformer", llamasearch.dev, section 01 GatedDeltaNet, names
// both: a one-dimensional convolution gives the values local context, and a
// gate sets how much of the rule's read-out reaches the output).  The page gives neither the width nor the
// gate's form; the library reads them as
//   y_t[c] = act(bias[c] + sum_{j<W} w[c][j] x_{t-(W-1)+j}[c])   (W = 2..8)
// per value channel c = h * dv + i, causal within each sequence, the inputs
// before a sequence's first token taken from a carried state of its last W-1
// inputs (zero without one), act = identity or SiLU; and o <- o * sigmoid(z)
// elementwise.
//
// All three kernels are single streaming passes over HBM:
//  * conv_kernel: a thread owns 16 bytes of channels (8 bf16 / 4 fp32) for one
//    contiguous segment of tokens (one segment per SM and channel block), with
//    its weights loaded once.  Its inputs come through a private ring of
//    kConvStages tiles of kConvTile tokens in shared memory, filled by cp.async
//    kConvStages - 1 tiles ahead (each thread reads back only what it copied,
//    so no barrier is involved and 96 KB per SM stay in flight: the load
//    depth an HBM stream needs), and it slides a window of the previous W-1
//    inputs in registers.  Each input is read from DRAM once; the W-1 halo rows
//    before a segment are re-read from L2.  A sequence start inside a segment
//    resets the window from the carried state.  For the layer prefill (GZ) the
//    same threads also turn the gate logits z of their tokens and channels (z has
//    v's layout) into the factors sigmoid(z): a second stream through the ring,
//    one launch for both passes.
//  * conv_state_kernel (launched after it on the same stream): each
//    sequence's new carried state, its last W-1 inputs (from the old state
//    where the sequence is shorter than W-1).  A launch of its own, so that
//    every read of the old state is over before it is overwritten in place.
//  * gate_kernel: o <- o * sigmoid(z), 16-byte vectors, grid-stride.
//  * gate_factor_kernel: sigmoid(z) -- fp16 (relative error <= 2^-12) for bf16
//    calls, fp32 for fp32 calls -- the factors the layer prefill's read-out
//    multiplies by, computed here on every SM at streaming speed rather than on
//    the prefill's chain SMs, where the special function unit would sit on the
//    critical path.
#include <cuda_fp16.h>

#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kConvThreads = 512;  // 16 warps per SM: the per-token arithmetic needs the latency hiding
constexpr int kConvTile = 4;     // tokens per tile
// tiles in a thread's ring: 4 (three in flight) for the values alone, 3 when the
// gate logits stream through the same ring
template <bool GZ>
__host__ __device__ constexpr int conv_stages() { return GZ ? 3 : 4; }
// bf16 widths 6..8 keep their weights and window in 256 threads' registers
template <typename T, int W>
__host__ __device__ constexpr int conv_threads() { return (sizeof(T) == 2 && W >= 6) ? 256 : kConvThreads; }
template <typename T, int W, bool GZ>
__host__ __device__ constexpr size_t conv_smem() {
    return (size_t)conv_stages<GZ>() * kConvTile * conv_threads<T, W>() * 16 * (GZ ? 2 : 1);
}
constexpr int kGateThreads = 256;

// 16 bytes of one dtype as raw words and as floats
template <typename T> struct Vec16;
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int n = 8;
    __device__ static void to_float(const uint4 &u, float (&f)[8]) {
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 t = __bfloat1622float2(h[i]);
            f[2 * i] = t.x;
            f[2 * i + 1] = t.y;
        }
    }
    __device__ static uint4 from_float(const float (&f)[8]) {
        uint4 u;
        uint32_t *w = reinterpret_cast<uint32_t *>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t *>(&h);
        }
        return u;
    }
};
template <> struct Vec16<float> {
    static constexpr int n = 4;
    __device__ static void to_float(const uint4 &u, float (&f)[4]) {
        f[0] = __uint_as_float(u.x);
        f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z);
        f[3] = __uint_as_float(u.w);
    }
    __device__ static uint4 from_float(const float (&f)[4]) {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                          __float_as_uint(f[3]));
    }
};

template <typename T>
__device__ __forceinline__ uint4 ld16(const T *p) { return *reinterpret_cast<const uint4 *>(p); }
template <typename T>
__device__ __forceinline__ void st16(T *p, uint4 v) { *reinterpret_cast<uint4 *>(p) = v; }

// bounds of sequence n
__device__ __forceinline__ void seq_bounds(const int32_t *cu, int64_t T_per, int n, int64_t &bos,
                                           int64_t &eos) {
    if (cu) {
        bos = cu[n];
        eos = cu[n + 1];
    } else {
        bos = (int64_t)n * T_per;
        eos = bos + T_per;
    }
}

__device__ __forceinline__ void conv_cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src)
                 : "memory");
}

template <typename T, int W, bool GZ>
__global__ void __launch_bounds__(conv_threads<T, W>(), 1)
conv_kernel(const T *__restrict__ x, const float *__restrict__ w, const float *__restrict__ bias,
            const T *__restrict__ cstate, const int32_t *__restrict__ cu, int N, int64_t T_per,
            int64_t Ttot, int C, int cblocks, int64_t seg_len, bool silu, T *__restrict__ y,
            T *__restrict__ y_lo, const T *__restrict__ z, void *__restrict__ fz) {
    constexpr int VN = Vec16<T>::n;
    constexpr int NT = conv_threads<T, W>();
    constexpr int NS = conv_stages<GZ>();
    constexpr int ZOFF = NS * kConvTile * NT;   // the z stream's part of the ring
    extern __shared__ uint4 ring[];   // [stage][token of the tile][thread] (values, then z)
    const int seg = (int)(blockIdx.x / cblocks);
    const int c0 = ((int)(blockIdx.x - seg * cblocks) * NT + threadIdx.x) * VN;
    if (c0 >= C) return;   // (no barrier below: every thread works on its own)
    const int64_t t0 = (int64_t)seg * seg_len;
    const int64_t t1 = t0 + seg_len < Ttot ? t0 + seg_len : Ttot;
    if (t0 >= t1) return;
    // the sequence holding token t0: the last n with start <= t0 (empty sequences skipped)
    int n;
    if (cu) {
        int lo = 0, hi = N - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (cu[mid] <= t0) lo = mid;
            else hi = mid - 1;
        }
        n = lo;
    } else {
        n = (int)(t0 / T_per);
    }
    int64_t bos, eos;
    seq_bounds(cu, T_per, n, bos, eos);

    // the ring: tile k of the segment into stage k % NS, this thread's 16 bytes of
    // each token; a commit group per tile (empty past the segment's end)
    const int ntiles = (int)((t1 - t0 + kConvTile - 1) / kConvTile);
    auto issue = [&](int k) {
        const int64_t tb = t0 + (int64_t)k * kConvTile;
        uint4 *dst = ring + (size_t)(k % NS) * kConvTile * NT + threadIdx.x;
        if (k < ntiles) {
#pragma unroll
            for (int r = 0; r < kConvTile; ++r)
                if (tb + r < t1) {
                    conv_cp_async16(dst + r * NT, x + (tb + r) * C + c0);
                    if (GZ) conv_cp_async16(dst + ZOFF + r * NT, z + (tb + r) * C + c0);
                }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
#pragma unroll
    for (int k = 0; k < NS - 1; ++k) issue(k);

    // this thread's VN x W weights are contiguous (16-byte aligned: c0 is a multiple of 4)
    // weights and bias as channel pairs (the arithmetic runs on packed fp32 pairs)
    constexpr int VP = VN / 2;
    float2 wt[W][VP], b[VP];
    {
        float flat[VN * W];
        const float4 *w4 = reinterpret_cast<const float4 *>(w + (size_t)c0 * W);
#pragma unroll
        for (int i = 0; i < VN * W / 4; ++i) {
            const float4 f = __ldg(w4 + i);
            flat[4 * i] = f.x;
            flat[4 * i + 1] = f.y;
            flat[4 * i + 2] = f.z;
            flat[4 * i + 3] = f.w;
        }
#pragma unroll
        for (int e = 0; e < VP; ++e)
#pragma unroll
            for (int j = 0; j < W; ++j) wt[j][e] = make_float2(flat[2 * e * W + j], flat[(2 * e + 1) * W + j]);
#pragma unroll
        for (int e = 0; e < VP; ++e)
            b[e] = bias ? make_float2(__ldg(bias + c0 + 2 * e), __ldg(bias + c0 + 2 * e + 1))
                        : make_float2(0.f, 0.f);
    }
    // window: win[m] = the input at token t - (W-1) + m, m < W-1, as fp32 pairs
    // (converted once, when it enters)
    float2 win[W - 1][VP];
    auto to_pairs = [](const uint4 &u, float2 (&f)[VP]) {
        float tmp[VN];
        Vec16<T>::to_float(u, tmp);
#pragma unroll
        for (int e = 0; e < VP; ++e) f[e] = make_float2(tmp[2 * e], tmp[2 * e + 1]);
    };
#pragma unroll
    for (int m = 0; m < W - 1; ++m) {
        const int64_t s = t0 - (W - 1) + m;
        uint4 raw = make_uint4(0u, 0u, 0u, 0u);   // +0.0 in both dtypes
        if (s >= bos)
            raw = ld16(x + s * C + c0);
        else if (cstate)
            raw = ld16(cstate + ((size_t)n * (W - 1) + (size_t)(s - bos + W - 1)) * C + c0);
        to_pairs(raw, win[m]);
    }
    for (int k = 0; k < ntiles; ++k) {
        issue(k + NS - 1);
        // all but the NS - 1 newest groups are complete: tile k has landed
        asm volatile("cp.async.wait_group %0;" ::"n"(NS - 1) : "memory");
        const uint4 *src = ring + (size_t)(k % NS) * kConvTile * NT + threadIdx.x;
        const int64_t tb = t0 + (int64_t)k * kConvTile;
#pragma unroll
        for (int u = 0; u < kConvTile; ++u) {
            const int64_t t = tb + u;
            if (t >= t1) break;
            const uint4 cur = src[u * NT];
            if (t >= eos) {
                // a new sequence starts at t (after any empty ones): window from its state
                do {
                    ++n;
                    seq_bounds(cu, T_per, n, bos, eos);
                } while (eos <= t);
#pragma unroll
                for (int m = 0; m < W - 1; ++m)
                    to_pairs(cstate ? ld16(cstate + ((size_t)n * (W - 1) + m) * C + c0)
                                    : make_uint4(0u, 0u, 0u, 0u),
                             win[m]);
            }
            float2 cf[VP], acc[VP];
            to_pairs(cur, cf);
#pragma unroll
            for (int e = 0; e < VP; ++e) {
                float2 a = b[e];
#pragma unroll
                for (int m = 0; m < W - 1; ++m) a = fma2(wt[m][e], win[m][e], a);
                a = fma2(wt[W - 1][e], cf[e], a);
                acc[e] = silu ? make_float2(a.x * layer_sigmoid(a.x), a.y * layer_sigmoid(a.y)) : a;
            }
            float af[VN];
#pragma unroll
            for (int e = 0; e < VP; ++e) {
                af[2 * e] = acc[e].x;
                af[2 * e + 1] = acc[e].y;
            }
            const uint4 yv = Vec16<T>::from_float(af);
            st16(y + t * C + c0, yv);
            if (y_lo) {
                // the remainder acc - y (exact in fp32) as a second output: the bf16
                // pair y + y_lo carries the convolved value to ~2^-17 relative
                float r[VN];
                Vec16<T>::to_float(yv, r);
#pragma unroll
                for (int e = 0; e < VN; ++e) r[e] = af[e] - r[e];
                st16(y_lo + t * C + c0, Vec16<T>::from_float(r));
            }
#pragma unroll
            for (int m = 0; m + 1 < W - 1; ++m)
#pragma unroll
                for (int e = 0; e < VP; ++e) win[m][e] = win[m + 1][e];
#pragma unroll
            for (int e = 0; e < VP; ++e) win[W - 2][e] = cf[e];
            if (GZ) {
                // gate factors sigmoid(z): fp16 for bf16 logits, fp32 for fp32 ones
                float zf[VN];
                Vec16<T>::to_float(src[ZOFF + u * NT], zf);
                uint4 fv;
                if constexpr (VN == 8) {
                    __half2 hh[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        hh[e] = __floats2half2_rn(layer_sigmoid(zf[2 * e]), layer_sigmoid(zf[2 * e + 1]));
                    fv = *reinterpret_cast<const uint4 *>(hh);
                } else {
                    fv = make_uint4(__float_as_uint(layer_sigmoid(zf[0])), __float_as_uint(layer_sigmoid(zf[1])),
                                    __float_as_uint(layer_sigmoid(zf[2])), __float_as_uint(layer_sigmoid(zf[3])));
                }
                *reinterpret_cast<uint4 *>(static_cast<uint8_t *>(fz) + ((size_t)t * C + c0) * sizeof(T)) = fv;
            }
        }
    }
    // (every group still pending is empty: tiles past the end issue no copy)
}

// new carried state of sequence blockIdx.x: its last W-1 inputs (raw copies)
template <typename T, int W>
__global__ void __launch_bounds__(kConvThreads)
conv_state_kernel(const T *__restrict__ x, T *cstate, const int32_t *__restrict__ cu, int64_t T_per,
                  int C) {
    constexpr int VN = Vec16<T>::n;
    const int c0 = (blockIdx.y * kConvThreads + threadIdx.x) * VN;
    if (c0 >= C) return;
    const int n = blockIdx.x;
    int64_t bos, eos;
    seq_bounds(cu, T_per, n, bos, eos);
    const int64_t L = eos - bos;
    T *st = cstate + (size_t)n * (W - 1) * C + c0;
    uint4 old[W - 1], nw[W - 1];
#pragma unroll
    for (int m = 0; m < W - 1; ++m) old[m] = ld16(st + (size_t)m * C);
#pragma unroll
    for (int m = 0; m < W - 1; ++m) {
        const int64_t s = eos - (W - 1) + m;
        if (s >= bos) {
            nw[m] = ld16(x + s * C + c0);
        } else {
            // old[m + L] (m + L < W - 1 when s < bos), selected without a dynamic index
            nw[m] = old[0];
#pragma unroll
            for (int r = 1; r < W - 1; ++r)
                if (r == m + L) nw[m] = old[r];
        }
    }
#pragma unroll
    for (int m = 0; m < W - 1; ++m) st16(st + (size_t)m * C, nw[m]);
}

template <typename T>
__global__ void __launch_bounds__(kGateThreads)
gate_kernel(T *o, const T *__restrict__ z, int64_t nvec) {
    constexpr int VN = Vec16<T>::n;
    constexpr int U = 4;
    const int64_t stride = (int64_t)gridDim.x * kGateThreads;
    for (int64_t i0 = (int64_t)blockIdx.x * kGateThreads + threadIdx.x; i0 < nvec; i0 += U * stride) {
        uint4 ov[U], zv[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = i0 + u * stride;
            if (i < nvec) {
                ov[u] = __ldcs(reinterpret_cast<const uint4 *>(o) + i);
                zv[u] = __ldcs(reinterpret_cast<const uint4 *>(z) + i);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = i0 + u * stride;
            if (i < nvec) {
                float of[VN], zf[VN];
                Vec16<T>::to_float(ov[u], of);
                Vec16<T>::to_float(zv[u], zf);
#pragma unroll
                for (int e = 0; e < VN; ++e) of[e] *= layer_sigmoid(zf[e]);
                __stcs(reinterpret_cast<uint4 *>(o) + i, Vec16<T>::from_float(of));
            }
        }
    }
}

template <typename T>
__global__ void __launch_bounds__(kGateThreads)
gate_factor_kernel(const T *__restrict__ z, void *__restrict__ f, int64_t nvec) {
    constexpr int VN = Vec16<T>::n;
    const int64_t stride = (int64_t)gridDim.x * kGateThreads;
    for (int64_t i = (int64_t)blockIdx.x * kGateThreads + threadIdx.x; i < nvec; i += stride) {
        float zf[VN];
        Vec16<T>::to_float(__ldcs(reinterpret_cast<const uint4 *>(z) + i), zf);
        if constexpr (VN == 8) {   // bf16 logits -> fp16 factors
            __half2 h[VN / 2];
#pragma unroll
            for (int e = 0; e < VN / 2; ++e)
                h[e] = __floats2half2_rn(layer_sigmoid(zf[2 * e]), layer_sigmoid(zf[2 * e + 1]));
            reinterpret_cast<uint4 *>(f)[i] = *reinterpret_cast<const uint4 *>(h);
        } else {                   // fp32 logits -> fp32 factors
            reinterpret_cast<float4 *>(f)[i] = make_float4(layer_sigmoid(zf[0]), layer_sigmoid(zf[1]),
                                                           layer_sigmoid(zf[2]), layer_sigmoid(zf[3]));
        }
    }
}

int sm_count() {
    int dev = 0, count = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || count < 1)
        count = 1;
    return count;
}

template <typename T, int W, bool GZ>
cudaError_t launch_conv_segments(const ConvArgs &a, int64_t Ttot, cudaStream_t stream) {
    // one segment of tokens per SM and channel block (a multiple of the tile)
    constexpr int VN = Vec16<T>::n;
    constexpr int NT = conv_threads<T, W>();
    constexpr size_t smem = conv_smem<T, W, GZ>();
    const int64_t cb = (a.C / VN + NT - 1) / NT;
    const int64_t tiles = (Ttot + kConvTile - 1) / kConvTile;
    int64_t nseg = ((int64_t)sm_count() + cb - 1) / cb;
    if (nseg > tiles) nseg = tiles;
    const int64_t seg_len = (tiles + nseg - 1) / nseg * kConvTile;
    nseg = (Ttot + seg_len - 1) / seg_len;
    auto kern = conv_kernel<T, W, GZ>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(nseg * cb), NT, smem, stream>>>(
        static_cast<const T *>(a.x), a.weight, a.bias, static_cast<const T *>(a.conv_state), a.cu_seqlens,
        a.N, a.T, Ttot, a.C, (int)cb, seg_len, a.silu, static_cast<T *>(a.y), static_cast<T *>(a.y_lo),
        static_cast<const T *>(a.z), a.f);
    return cudaGetLastError();
}

template <typename T, int W>
cudaError_t launch_conv_w(const ConvArgs &a, cudaStream_t stream) {
    constexpr int VN = Vec16<T>::n;
    const int vecs = a.C / VN;
    const unsigned cblocks = (unsigned)((vecs + kConvThreads - 1) / kConvThreads);
    const int64_t Ttot = a.cu_seqlens ? a.T : (int64_t)a.N * a.T;
    const T *x = static_cast<const T *>(a.x);
    T *cs = static_cast<T *>(a.conv_state);
    if (Ttot > 0) {
        const cudaError_t e = a.z ? launch_conv_segments<T, W, true>(a, Ttot, stream)
                                  : launch_conv_segments<T, W, false>(a, Ttot, stream);
        if (e != cudaSuccess) return e;
    }
    if (cs) {
        conv_state_kernel<T, W><<<dim3((unsigned)a.N, cblocks), kConvThreads, 0, stream>>>(
            x, cs, a.cu_seqlens, a.T, a.C);
        return cudaGetLastError();
    }
    return cudaSuccess;
}

template <typename T>
cudaError_t launch_conv_t(const ConvArgs &a, cudaStream_t stream) {
    switch (a.width) {
        case 2: return launch_conv_w<T, 2>(a, stream);
        case 3: return launch_conv_w<T, 3>(a, stream);
        case 4: return launch_conv_w<T, 4>(a, stream);
        case 5: return launch_conv_w<T, 5>(a, stream);
        case 6: return launch_conv_w<T, 6>(a, stream);
        case 7: return launch_conv_w<T, 7>(a, stream);
        case 8: return launch_conv_w<T, 8>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t launch_gate_t(void *o, const void *z, int64_t elems, cudaStream_t stream) {
    const int64_t nvec = elems / Vec16<T>::n;
    int64_t blocks = (nvec + kGateThreads * 4 - 1) / (kGateThreads * 4);
    const int64_t cap = (int64_t)sm_count() * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    gate_kernel<T><<<(unsigned)blocks, kGateThreads, 0, stream>>>(static_cast<T *>(o),
                                                                  static_cast<const T *>(z), nvec);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_gate_factor_t(const void *z, void *f, int64_t elems, cudaStream_t stream) {
    const int64_t nvec = elems / Vec16<T>::n;
    int64_t blocks = (nvec + kGateThreads - 1) / kGateThreads;
    const int64_t cap = (int64_t)sm_count() * 16;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    gate_factor_kernel<T><<<(unsigned)blocks, kGateThreads, 0, stream>>>(
        static_cast<const T *>(z), f, nvec);
    return cudaGetLastError();
}

}  // namespace

int conv_vector_channels(gdn_dtype dtype) { return dtype == GDN_BF16 ? 8 : 4; }

cudaError_t launch_gate_factor(const void *z, void *factors, int64_t elems, gdn_dtype dtype,
                               cudaStream_t stream) {
    if (elems == 0) return cudaSuccess;
    return dtype == GDN_BF16 ? launch_gate_factor_t<__nv_bfloat16>(z, factors, elems, stream)
                             : launch_gate_factor_t<float>(z, factors, elems, stream);
}

cudaError_t launch_short_conv(const ConvArgs &a, cudaStream_t stream) {
    if (a.N == 0) return cudaSuccess;
    return a.dtype == GDN_BF16 ? launch_conv_t<__nv_bfloat16>(a, stream) : launch_conv_t<float>(a, stream);
}

cudaError_t launch_output_gate(void *o, const void *z, int64_t elems, gdn_dtype dtype,
                               cudaStream_t stream) {
    if (elems == 0) return cudaSuccess;
    return dtype == GDN_BF16 ? launch_gate_t<__nv_bfloat16>(o, z, elems, stream)
                             : launch_gate_t<float>(o, z, elems, stream);
}

}  // namespace gdn
