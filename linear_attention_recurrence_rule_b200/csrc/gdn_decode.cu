// Fused single-token decode step of the gated delta rule.
//
// Rule ("Qwen3-Next", sghael.github.io, section "Correcting a memory instead of
// adding to it": decay first, then correct along the current key; read-out
// after the update as in "The Evolving Transformer / Qwen3-Next", section 01):
//
//   per row i of the dv x dk state S (row = value index):
//     sk_i = S_i . k          sq_i = S_i . q          (old state)
//     u_i  = beta * (v_i - alpha * sk_i)
//     S_i <- alpha * S_i + u_i * k
//     o_i  = scale * (alpha * sq_i + u_i * (k . q))   (= scale * S_i(new) . q)
//
// Every row is independent, so the kernel is a single streaming pass over the
// fp32 state: each state element is loaded once (128-bit, evict-first) and
// stored once (128-bit, streaming).  The two dot products of a row are reduced
// with warp shuffles inside the lanes that hold the row.
//
// Work split: CTAs of 8 warps, each owning a band of rows of one (sequence,
// value head) state (grid.y walks the bands).  A row of dk fp32 is held by dk/4
// lanes (one float4 each); a warp instruction covers 32/(dk/4) rows; each warp
// issues NB such loads before using any of them, so every lane has NB x 16 B of
// state in flight.  Bands of 8 x NB rows (64 at dk = 128) keep CTAs short and
// several of them resident per SM, so their load, update and store phases
// overlap.
//
// The layer instance (gdn_recurrent_step_layer) adds the steps around the rule
// for one token: the short convolution on v with its carried inputs, and the
// sigmoid gate on o (readings in gdn_layer.cu).  The band's threads compute the
// convolved values and gates of its rows into shared memory while the state
// loads are in flight; the carried inputs (W-1 values per channel) are the
// only extra HBM traffic besides v, z and the weights.
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kDecodeWarps = 8;
constexpr int kDecodeNB = 8;

template <int DK>
constexpr int band_rows() { return kDecodeWarps * (32 / (DK / 4)) * kDecodeNB; }

// The layer steps of gdn_recurrent_step_layer: the short convolution on v (its
// carried inputs updated in place) and the sigmoid gate on o.
template <typename Tin>
struct LayerStep {
    const float *cw, *cb;   // [HV*dv][W], [HV*dv] or null
    Tin *cs;                // [N][W-1][HV*dv]
    const Tin *z;           // [N][HV][dv] or null
    int W;                  // 0: no convolution
    bool silu;
};

// PRO: the input prologue flags are read; RD (implies PRO): one decay per value
// row; LY (implies PRO): the layer steps.  Separate instances, so none of them
// costs the paths that do not use it.
template <int DK, typename Tin, bool PRO, bool RD, bool LY>
__global__ void __launch_bounds__(kDecodeWarps * 32, 3)
decode_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
              const float *__restrict__ g, const float *__restrict__ beta, float *state,
              Tin *__restrict__ o, int HK, int HV, int dv, float scale, unsigned pro,
              LayerStep<Tin> ly) {
    constexpr int LPR = DK / 4;    // lanes per state row
    constexpr int RPI = 32 / LPR;  // rows per warp instruction
    const int nh = blockIdx.x;     // n * HV + h
    const int n = nh / HV, h = nh - n * HV;
    const int c = h / (HV / HK);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane / LPR;
    const int col = (lane % LPR) * 4;

    float4 kk = load4(k + ((size_t)n * HK + c) * DK + col);
    float4 qq = load4(q + ((size_t)n * HK + c) * DK + col);
    constexpr bool rowdec = RD;   // g: one entry per value row
    const float graw = rowdec ? 0.f : g[nh], braw = beta[nh];
    const Tin *vrow = v + (size_t)nh * dv;
    Tin *orow = o + (size_t)nh * dv;
    float *S = state + (size_t)nh * dv * DK;

    constexpr int rows_per_batch = kDecodeWarps * RPI * kDecodeNB;
    {
        const int base = blockIdx.y * rows_per_batch;
        // layer steps of this band's rows (one row per thread of the first
        // rows_per_batch / 32 warps, before their own state loads; the other warps'
        // state loads are in flight meanwhile): the convolved value and the output
        // gate of each row, shared by its lanes
        __shared__ float lyv[LY ? rows_per_batch : 1], lyg[LY ? rows_per_batch : 1];
        if (LY && threadIdx.x < rows_per_batch && base + (int)threadIdx.x < dv) {
            const size_t C = (size_t)HV * dv;
            const int r = threadIdx.x;
            const int row = base + r;
            const size_t ch = (size_t)h * dv + row;
            const float vin = to_f32(vrow[row]);
            float vc = vin;
            if (ly.W > 0) {
                // every tap's loads go out together (predicated, not a runtime loop)
                constexpr int MW = kConvMaxWidth;
                const int W = ly.W;
                Tin *cs = ly.cs + (size_t)n * (W - 1) * C + ch;
                const float *wr = ly.cw + ch * W;
                Tin hist[MW - 1];
                float wt[MW];
#pragma unroll
                for (int m = 0; m < MW - 1; ++m)
                    if (m < W - 1) hist[m] = cs[m * C];
#pragma unroll
                for (int m = 0; m < MW; ++m)
                    if (m < W) wt[m] = wr[m];
                float a = ly.cb ? ly.cb[ch] : 0.f;
#pragma unroll
                for (int m = 0; m < MW - 1; ++m)
                    if (m < W - 1) a = fmaf(wt[m], to_f32(hist[m]), a);
#pragma unroll
                for (int m = 0; m < MW; ++m)
                    if (m == W - 1) a = fmaf(wt[m], vin, a);
                vc = ly.silu ? a * layer_sigmoid(a) : a;
                // the carried inputs move one token on; this token's raw value last
#pragma unroll
                for (int m = 0; m < MW - 2; ++m)
                    if (m < W - 2) cs[m * C] = hist[m + 1];
                cs[(W - 2) * C] = vrow[row];
            }
            lyv[r] = vc;
            lyg[r] = ly.z ? layer_sigmoid(to_f32(ly.z[(size_t)nh * dv + row])) : 1.f;
        }
        // the state loads go out first (after the layer steps in the layer
        // instance's first warps): nothing below them waits on q, k
        float4 s[kDecodeNB];
        float grow[RD ? kDecodeNB : 1];   // per-row decays (GDN_ROW_DECAY), loaded with the state
#pragma unroll
        for (int j = 0; j < kDecodeNB; ++j) {
            const int row = base + (j * kDecodeWarps + warp) * RPI + sub;
            s[j] = row < dv ? __ldcs(reinterpret_cast<const float4 *>(S + (size_t)row * DK + col))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
            if (RD) grow[RD ? j : 0] = row < dv ? g[(size_t)nh * dv + row] : 0.f;
        }
        if (LY) __syncthreads();   // the band's convolved values and gates are in place
        if (PRO && (pro & (GDN_PROLOGUE_NORM_Q | GDN_PROLOGUE_NORM_K))) {
            // the lanes of a row hold the whole q and k: reduce the squared norms there
            float ssk = dot4(kk, kk), ssq = dot4(qq, qq);
#pragma unroll
            for (int off = LPR / 2; off > 0; off >>= 1) {
                ssk += __shfl_xor_sync(0xffffffffu, ssk, off);
                ssq += __shfl_xor_sync(0xffffffffu, ssq, off);
            }
            if (pro & GDN_PROLOGUE_NORM_K) kk = scale4(kk, inv_l2norm(ssk));
            if (pro & GDN_PROLOGUE_NORM_Q) qq = scale4(qq, inv_l2norm(ssq));
        }
        float kq = dot4(kk, qq);
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
        const bool logits = PRO && (pro & GDN_PROLOGUE_GATE_LOGITS) != 0;
        const float alpha_h = logits ? gate_sigmoid(graw) : expf(graw);
        const float b = logits ? gate_sigmoid(braw) : braw;
#pragma unroll
        for (int j = 0; j < kDecodeNB; ++j) {
            const int row = base + (j * kDecodeWarps + warp) * RPI + sub;
            float sk = dot4(s[j], kk), sq = dot4(s[j], qq);
#pragma unroll
            for (int off = LPR / 2; off > 0; off >>= 1) {
                sk += __shfl_xor_sync(0xffffffffu, sk, off);
                sq += __shfl_xor_sync(0xffffffffu, sq, off);
            }
            if (row < dv) {
                const float alpha =
                    rowdec ? (logits ? gate_sigmoid(grow[RD ? j : 0]) : expf(grow[RD ? j : 0]))
                           : alpha_h;
                const float vval = LY ? lyv[LY ? row - base : 0] : to_f32(vrow[row]);
                const float u = b * (vval - alpha * sk);
                float4 ns;
                ns.x = fmaf(alpha, s[j].x, u * kk.x);
                ns.y = fmaf(alpha, s[j].y, u * kk.y);
                ns.z = fmaf(alpha, s[j].z, u * kk.z);
                ns.w = fmaf(alpha, s[j].w, u * kk.w);
                __stcs(reinterpret_cast<float4 *>(S + (size_t)row * DK + col), ns);
                if ((lane % LPR) == 0) {
                    float out = scale * fmaf(alpha, sq, u * kq);
                    if (LY) out *= lyg[LY ? row - base : 0];
                    orow[row] = from_f32<Tin>(out);
                }
            }
        }
    }
}

template <int DK, typename Tin>
void launch_dk(const StepArgs &a, dim3 grid, dim3 block, cudaStream_t stream) {
    const bool layer = a.conv_width > 0 || a.z != nullptr;
    const bool rd = (a.prologue & GDN_ROW_DECAY) != 0;
    auto kern = layer ? (rd ? decode_kernel<DK, Tin, true, true, true>
                            : decode_kernel<DK, Tin, true, false, true>)
                : rd          ? decode_kernel<DK, Tin, true, true, false>
                : a.prologue  ? decode_kernel<DK, Tin, true, false, false>
                              : decode_kernel<DK, Tin, false, false, false>;
    const LayerStep<Tin> ly{a.conv_w, a.conv_b, static_cast<Tin *>(a.conv_state),
                            static_cast<const Tin *>(a.z), a.conv_width, a.conv_silu};
    kern<<<grid, block, 0, stream>>>(static_cast<const Tin *>(a.q), static_cast<const Tin *>(a.k),
                                     static_cast<const Tin *>(a.v), a.g, a.beta, a.state,
                                     static_cast<Tin *>(a.o), a.HK, a.HV, a.dv, a.scale,
                                     a.prologue, ly);
}

template <typename Tin>
cudaError_t launch_typed(const StepArgs &a, cudaStream_t stream) {
    const int band = a.dk == 128 ? band_rows<128>() : a.dk == 64 ? band_rows<64>() : band_rows<32>();
    const dim3 grid((unsigned)((size_t)a.N * a.HV), (unsigned)((a.dv + band - 1) / band)),
        block(kDecodeWarps * 32);
    switch (a.dk) {
        case 32: launch_dk<32, Tin>(a, grid, block, stream); break;
        case 64: launch_dk<64, Tin>(a, grid, block, stream); break;
        case 128: launch_dk<128, Tin>(a, grid, block, stream); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace

bool decode_supported(int dk, int dv) {
    return (dk == 32 || dk == 64 || dk == 128) && dv >= 1 && dv <= 256;
}

cudaError_t launch_decode(const StepArgs &a, cudaStream_t stream) {
    if (a.N == 0) return cudaSuccess;
    return a.dtype == GDN_BF16 ? launch_typed<__nv_bfloat16>(a, stream)
                               : launch_typed<float>(a, stream);
}

}  // namespace gdn
