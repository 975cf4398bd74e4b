// Multi-token verify of speculative drafts for the gated delta rule, and the two
// roll-back calls that keep the accepted prefix.
//
// Speculative decoding ("Qwen3-Next", sghael.github.io, section "Speed depends on
// the serving software"): the model checks several proposed tokens at once and
// keeps those it agrees with.  For the recurrence that means running K draft
// tokens through the decode rule from one state, then keeping the state after
// the last accepted draft.
//
// Rule per draft t and row i of the dv x dk state (decay first, then correct
// along the key; read-out after the update), alpha_t = exp(g_t):
//     u_i  = beta_t (v_i - alpha_t S_i . k_t)
//     S_i <- alpha_t S_i + u_i k_t             o_i = scale * S_i(new) . q_t
//
// All kernels are single streaming passes over fp32 state bands of one
// (sequence, value head): CTAs of 8 warps, rows of dk fp32 held by dk/16 lanes
// with four float4 each (lane l of a row owns float4 l, l + dk/16, ..., so a
// warp instruction reads whole 128-byte lines), two rows per lane.
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kVerifyWarps = 8;

// Multi-token verify: K draft tokens per sequence, the band of the state held in
// registers from token to token; the state input is only read.  For roll-back the
// kernel writes, when asked, the state after every token (states) and/or the
// update vector of every token, u_t = beta_t (v_t - alpha_t S_{t-1} k_t), with
// which S_t = alpha_t S_{t-1} + u_t k_t^T (u).
//
// Layout for K tokens per state load: a row is held by dk/16 lanes with 16
// columns each (four float4, lane l of the row owning float4 l, l + dk/16, ...
// so a warp instruction reads whole 128-byte lines), and the two dot products
// of a row reduce in log2(dk/16) shuffle steps.  With one warp per row (the
// decode layout) the shuffle pipe, not HBM, would bound a 4-token pass.  The K
// tokens' q, k, v, alpha, beta are staged in shared memory while the state
// loads are in flight.
constexpr int kVerifyF4 = 4;     // float4 per lane per row
constexpr int kVerifyRows = 2;   // rows per lane

template <int DK>
__host__ __device__ constexpr int verify_band() { return kVerifyWarps * (32 / (DK / (4 * kVerifyF4))) * kVerifyRows; }

// Input prologue on rows staged in shared memory: L2-normalise rows [0, nrows),
// one warp per row.
template <int DK>
__device__ __forceinline__ void normalize_rows(float4 (*rows)[DK / 4], int nrows, int warp,
                                               int lane) {
    for (int t = warp; t < nrows; t += kVerifyWarps) {
        float ss = 0.f;
        for (int j = lane; j < DK / 4; j += 32) ss += dot4(rows[t][j], rows[t][j]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float r = inv_l2norm(ss);
        for (int j = lane; j < DK / 4; j += 32) rows[t][j] = scale4(rows[t][j], r);
    }
}

template <int DK>
__device__ __forceinline__ void prologue_qk(float4 (*ks)[DK / 4], float4 (*qs)[DK / 4], int K,
                                            unsigned pro, int warp, int lane) {
    if (pro & GDN_PROLOGUE_NORM_K) normalize_rows<DK>(ks, K, warp, lane);
    if (pro & GDN_PROLOGUE_NORM_Q) normalize_rows<DK>(qs, K, warp, lane);
}

__device__ __forceinline__ float gate_alpha(float g, unsigned pro) {
    return (pro & GDN_PROLOGUE_GATE_LOGITS) ? gate_sigmoid(g) : expf(g);
}
__device__ __forceinline__ float gate_beta(float b, unsigned pro) {
    return (pro & GDN_PROLOGUE_GATE_LOGITS) ? gate_sigmoid(b) : b;
}

template <int DK, typename Tin, bool PRO>
__global__ void __launch_bounds__(kVerifyWarps * 32, 2)
verify_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
              const float *__restrict__ g, const float *__restrict__ beta,
              const float *__restrict__ state, float *__restrict__ states, float *__restrict__ u_out,
              Tin *__restrict__ o, int K, int HK, int HV, int dv, float scale, unsigned pro_arg) {
    const unsigned pro = PRO ? pro_arg : 0u;   // compiled out without the prologue
    constexpr int LPR = DK / (4 * kVerifyF4);   // lanes per row: 2, 4, 8
    constexpr int RPW = 32 / LPR;               // rows per warp instruction
    constexpr int BAND = verify_band<DK>();
    __shared__ float4 ks[kVerifyMaxDrafts][DK / 4], qs[kVerifyMaxDrafts][DK / 4];
    __shared__ float vs[kVerifyMaxDrafts][BAND];
    __shared__ float al[kVerifyMaxDrafts], be[kVerifyMaxDrafts];
    const int nh = blockIdx.x;
    const int n = nh / HV, h = nh - n * HV;
    const int c = h / (HV / HK);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane / LPR, li = lane % LPR;
    const size_t state_elems = (size_t)dv * DK;
    const int base = blockIdx.y * BAND;
    float4 s[kVerifyRows][kVerifyF4];
    const float *S = state + (size_t)nh * state_elems;
#pragma unroll
    for (int jr = 0; jr < kVerifyRows; ++jr) {
        const int row = base + (jr * kVerifyWarps + warp) * RPW + sub;
#pragma unroll
        for (int i = 0; i < kVerifyF4; ++i)
            s[jr][i] = row < dv ? __ldcs(reinterpret_cast<const float4 *>(S + (size_t)row * DK) +
                                         li + LPR * i)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int idx = threadIdx.x; idx < K * (DK / 4); idx += blockDim.x) {
        const int t = idx / (DK / 4), j = idx - t * (DK / 4);
        const size_t off = (((size_t)n * K + t) * HK + c) * DK + 4 * j;
        ks[t][j] = load4(k + off);
        qs[t][j] = load4(q + off);
    }
    for (int idx = threadIdx.x; idx < K * BAND; idx += blockDim.x) {
        const int t = idx / BAND, r = idx - t * BAND;
        const int row = base + r;
        vs[t][r] = row < dv ? to_f32(v[(((size_t)n * K + t) * HV + h) * dv + row]) : 0.f;
    }
    if (threadIdx.x < K) {
        const size_t gi = ((size_t)n * K + threadIdx.x) * HV + h;
        al[threadIdx.x] = gate_alpha(g[gi], pro);
        be[threadIdx.x] = gate_beta(beta[gi], pro);
    }
    __syncthreads();
    if (pro & (GDN_PROLOGUE_NORM_Q | GDN_PROLOGUE_NORM_K)) {
        prologue_qk<DK>(ks, qs, K, pro, warp, lane);
        __syncthreads();
    }
    for (int t = 0; t < K; ++t) {
        float4 kk[kVerifyF4];
        float kq = 0.f;
#pragma unroll
        for (int i = 0; i < kVerifyF4; ++i) {
            kk[i] = ks[t][li + LPR * i];
            kq += dot4(kk[i], qs[t][li + LPR * i]);
        }
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
        const float alpha = al[t], b = be[t];
        const size_t nt = (size_t)n * K + t;
        Tin *orow = o + (nt * HV + h) * dv;
        float *Sout = states ? states + (nt * HV + h) * state_elems : nullptr;
        float *urow = u_out ? u_out + (nt * HV + h) * dv : nullptr;
#pragma unroll
        for (int jr = 0; jr < kVerifyRows; ++jr) {
            const int r = (jr * kVerifyWarps + warp) * RPW + sub;
            const int row = base + r;
            float sk = 0.f, sq = 0.f;
#pragma unroll
            for (int i = 0; i < kVerifyF4; ++i) {
                sk += dot4(s[jr][i], kk[i]);
                sq += dot4(s[jr][i], qs[t][li + LPR * i]);
            }
#pragma unroll
            for (int off = LPR / 2; off > 0; off >>= 1) {
                sk += __shfl_xor_sync(0xffffffffu, sk, off);
                sq += __shfl_xor_sync(0xffffffffu, sq, off);
            }
            const float u = b * (vs[t][r] - alpha * sk);
#pragma unroll
            for (int i = 0; i < kVerifyF4; ++i) {
                s[jr][i].x = fmaf(alpha, s[jr][i].x, u * kk[i].x);
                s[jr][i].y = fmaf(alpha, s[jr][i].y, u * kk[i].y);
                s[jr][i].z = fmaf(alpha, s[jr][i].z, u * kk[i].z);
                s[jr][i].w = fmaf(alpha, s[jr][i].w, u * kk[i].w);
            }
            if (row < dv) {
                if (Sout) {
#pragma unroll
                    for (int i = 0; i < kVerifyF4; ++i)
                        __stcs(reinterpret_cast<float4 *>(Sout + (size_t)row * DK) + li + LPR * i,
                               s[jr][i]);
                }
                if (li == 0) {
                    orow[row] = from_f32<Tin>(scale * fmaf(alpha, sq, u * kq));
                    if (urow) urow[row] = u;
                }
            }
        }
    }
}

// Verify without the per-draft states (u_out form): the input state S_0 is never
// updated.  Unrolling S_t = alpha_t S_{t-1} + u_t k_t^T over the drafts (the chunk
// form of the rule restricted to K tokens), for one row r of the state,
//   S_{t-1}[r] . k_t = gamma_{t-1} a_t + sum_{j<t}  G(j,t-1) (k_j . k_t) u_j[r]
//   S_t[r]     . q_t = gamma_t     b_t + sum_{j<=t} G(j,t)   (k_j . q_t) u_j[r]
// with a_t = S_0[r] . k_t, b_t = S_0[r] . q_t, gamma_t = prod_{s<=t} alpha_s and
// G(j,t) = prod_{j<s<=t} alpha_s.  So a lane computes the 2K dot products of its
// rows against S_0 (independent of each other), then a K-step recurrence on
// per-row scalars whose coefficients (the K x K Gram products k_j . k_t and
// k_j . q_t times the decays, times beta and scale) are tabled once per CTA.
// KT is the compile-time bound on K (4, 8 or 16).
template <int DK, int KT, typename Tin, bool PRO>
__global__ void __launch_bounds__(kVerifyWarps * 32, KT <= 4 ? 3 : 2)
verify_wy_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                 const float *__restrict__ g, const float *__restrict__ beta,
                 const float *__restrict__ state, float *__restrict__ u_out, Tin *__restrict__ o,
                 int K, int HK, int HV, int dv, float scale, unsigned pro_arg) {
    const unsigned pro = PRO ? pro_arg : 0u;
    constexpr int LPR = DK / (4 * kVerifyF4);
    constexpr int RPW = 32 / LPR;
    constexpr int BAND = verify_band<DK>();
    __shared__ float4 ks[KT][DK / 4], qs[KT][DK / 4];
    __shared__ float vs[KT][BAND];
    __shared__ float al[KT], be[KT];
    __shared__ float gram[2][KT][KT];      // [0][j][t] = k_j . k_t, [1][j][t] = k_j . q_t
    __shared__ float ck[KT][KT], cq[KT][KT], a1[KT], b1[KT];
    const int nh = blockIdx.x;
    const int n = nh / HV, h = nh - n * HV;
    const int c = h / (HV / HK);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane / LPR, li = lane % LPR;
    const int base = blockIdx.y * BAND;
    float4 s[kVerifyRows][kVerifyF4];
    const float *S = state + (size_t)nh * dv * DK;
#pragma unroll
    for (int jr = 0; jr < kVerifyRows; ++jr) {
        const int row = base + (jr * kVerifyWarps + warp) * RPW + sub;
#pragma unroll
        for (int i = 0; i < kVerifyF4; ++i)
            s[jr][i] = row < dv ? __ldcs(reinterpret_cast<const float4 *>(S + (size_t)row * DK) +
                                         li + LPR * i)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int idx = threadIdx.x; idx < K * (DK / 4); idx += blockDim.x) {
        const int t = idx / (DK / 4), j = idx - t * (DK / 4);
        const size_t off = (((size_t)n * K + t) * HK + c) * DK + 4 * j;
        ks[t][j] = load4(k + off);
        qs[t][j] = load4(q + off);
    }
    for (int idx = threadIdx.x; idx < K * BAND; idx += blockDim.x) {
        const int t = idx / BAND, r = idx - t * BAND;
        const int row = base + r;
        vs[t][r] = row < dv ? to_f32(v[(((size_t)n * K + t) * HV + h) * dv + row]) : 0.f;
    }
    if (threadIdx.x < K) {
        const size_t gi = ((size_t)n * K + threadIdx.x) * HV + h;
        al[threadIdx.x] = gate_alpha(g[gi], pro);
        be[threadIdx.x] = gate_beta(beta[gi], pro);
    }
    __syncthreads();
    if (pro & (GDN_PROLOGUE_NORM_Q | GDN_PROLOGUE_NORM_K)) {
        prologue_qk<DK>(ks, qs, K, pro, warp, lane);
        __syncthreads();
    }
    // Gram products, one warp per pair
    for (int p = warp; p < 2 * K * K; p += kVerifyWarps) {
        const int which = p / (K * K), rem = p - which * K * K;
        const int j = rem / K, t = rem - j * K;
        float acc = 0.f;
        for (int f = lane; f < DK / 4; f += 32) acc += dot4(ks[j][f], which ? qs[t][f] : ks[t][f]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) gram[which][j][t] = acc;
    }
    __syncthreads();
    if (threadIdx.x < K) {
        const int t = threadIdx.x;
        // u_t = beta_t v_t - a1[t] a_t - sum_{j<t} ck[t][j] u_j
        float G = 1.f;   // G(j, t-1), walking j down from t-1
        for (int j = t - 1; j >= 0; --j) {
            ck[t][j] = be[t] * al[t] * G * gram[0][j][t];
            G *= al[j];
        }
        a1[t] = be[t] * al[t] * G;   // G is now gamma_{t-1}
        // o_t = b1[t] b_t + sum_{j<=t} cq[t][j] u_j
        float H = 1.f;   // G(j, t)
        for (int j = t; j >= 0; --j) {
            cq[t][j] = scale * H * gram[1][j][t];
            H *= al[j];
        }
        b1[t] = scale * H;           // scale * gamma_t
    }
    __syncthreads();
    float uh[kVerifyRows][KT];
#pragma unroll
    for (int t = 0; t < KT; ++t) {
        if (t >= K) break;
        float a[kVerifyRows], b[kVerifyRows];
#pragma unroll
        for (int jr = 0; jr < kVerifyRows; ++jr) {
            a[jr] = 0.f;
            b[jr] = 0.f;
        }
#pragma unroll
        for (int i = 0; i < kVerifyF4; ++i) {
            const float4 kk = ks[t][li + LPR * i], qq = qs[t][li + LPR * i];
#pragma unroll
            for (int jr = 0; jr < kVerifyRows; ++jr) {
                a[jr] += dot4(s[jr][i], kk);
                b[jr] += dot4(s[jr][i], qq);
            }
        }
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1) {
#pragma unroll
            for (int jr = 0; jr < kVerifyRows; ++jr) {
                a[jr] += __shfl_xor_sync(0xffffffffu, a[jr], off);
                b[jr] += __shfl_xor_sync(0xffffffffu, b[jr], off);
            }
        }
        const size_t nt = (size_t)n * K + t;
#pragma unroll
        for (int jr = 0; jr < kVerifyRows; ++jr) {
            const int r = (jr * kVerifyWarps + warp) * RPW + sub;
            float x = be[t] * vs[t][r] - a1[t] * a[jr];
#pragma unroll
            for (int j = 0; j < t; ++j) x = fmaf(-ck[t][j], uh[jr][j], x);
            uh[jr][t] = x;
            float y = b1[t] * b[jr];
#pragma unroll
            for (int j = 0; j <= t; ++j) y = fmaf(cq[t][j], uh[jr][j], y);
            const int row = base + r;
            if (row < dv && li == 0) {
                o[(nt * HV + h) * dv + row] = from_f32<Tin>(y);
                if (u_out) u_out[(nt * HV + h) * dv + row] = x;
            }
        }
    }
}

// Roll back after verification: state[n] <- states[n][accepted[n] - 1] when
// 1 <= accepted[n] <= K, unchanged otherwise.
__global__ void __launch_bounds__(256)
commit_kernel(const float *__restrict__ states, const int32_t *__restrict__ accepted,
              float *__restrict__ state, int K, int HV, size_t state_elems) {
    const int nh = blockIdx.x;
    const int n = nh / HV, h = nh - n * HV;
    const int a = accepted[n];
    if (a < 1 || a > K) return;
    const float4 *src = reinterpret_cast<const float4 *>(
        states + (((size_t)n * K + (a - 1)) * HV + h) * state_elems);
    float4 *dst = reinterpret_cast<float4 *>(state + (size_t)nh * state_elems);
    for (size_t i = blockIdx.y * (size_t)blockDim.x + threadIdx.x; i < state_elems / 4;
         i += (size_t)gridDim.y * blockDim.x)
        __stcs(dst + i, __ldcs(src + i));
}

// Roll back from the update vectors of a verify pass, in place: with a = accepted[n]
// drafts kept,  S_a = (prod_{t<a} alpha_t) S_0 + sum_{t<a} (prod_{t<s<a} alpha_s) u_t k_t^T,
// which is the recurrence S_t = alpha_t S_{t-1} + u_t k_t^T unrolled.  Each state
// element is read and written once; k_t and the scaled u_t of the band sit in
// shared memory.  Same row layout and bands as the verify kernel; all of a lane's
// state loads are issued before the staging and the arithmetic.
template <int DK, typename Tin, bool PRO>
__global__ void __launch_bounds__(kVerifyWarps * 32, 3)
commit_deltas_kernel(const Tin *__restrict__ k, const float *__restrict__ g,
                     const float *__restrict__ u, const int32_t *__restrict__ accepted,
                     float *__restrict__ state, int K, int HK, int HV, int dv,
                     unsigned pro_arg) {
    const unsigned pro = PRO ? pro_arg : 0u;
    constexpr int LPR = DK / (4 * kVerifyF4);
    constexpr int RPW = 32 / LPR;
    constexpr int BAND = verify_band<DK>();
    __shared__ float4 ks[kVerifyMaxDrafts][DK / 4];
    __shared__ float us[kVerifyMaxDrafts][BAND];
    __shared__ float coef[kVerifyMaxDrafts + 1];
    const int nh = blockIdx.x;
    const int n = nh / HV, h = nh - n * HV;
    const int c = h / (HV / HK);
    const int a = accepted[n];
    if (a < 1 || a > K) return;   // nothing kept: the state stays as it is
    const int base = blockIdx.y * BAND;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane / LPR, li = lane % LPR;
    float *S = state + (size_t)nh * dv * DK;
    float4 x[kVerifyRows][kVerifyF4];
#pragma unroll
    for (int jr = 0; jr < kVerifyRows; ++jr) {
        const int row = base + (jr * kVerifyWarps + warp) * RPW + sub;
#pragma unroll
        for (int i = 0; i < kVerifyF4; ++i)
            x[jr][i] = row < dv ? __ldcs(reinterpret_cast<const float4 *>(S + (size_t)row * DK) +
                                         li + LPR * i)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (threadIdx.x == 0) {
        // coef[t] = prod_{t<s<a} alpha_s, coef[K_max] = prod_{s<a} alpha_s
        float c_run = 1.f;
        for (int t = a - 1; t >= 0; --t) {
            coef[t] = c_run;
            c_run *= gate_alpha(g[((size_t)n * K + t) * HV + h], pro);
        }
        coef[kVerifyMaxDrafts] = c_run;
    }
    for (int i = threadIdx.x; i < a * (DK / 4); i += blockDim.x) {
        const int t = i / (DK / 4), j = i - t * (DK / 4);
        ks[t][j] = load4(k + (((size_t)n * K + t) * HK + c) * DK + 4 * j);
    }
    __syncthreads();
    if (pro & GDN_PROLOGUE_NORM_K) normalize_rows<DK>(ks, a, warp, lane);   // read after the next barrier
    for (int i = threadIdx.x; i < a * BAND; i += blockDim.x) {
        const int t = i / BAND, r = i - t * BAND;
        const int row = base + r;
        us[t][r] = row < dv ? coef[t] * u[(((size_t)n * K + t) * HV + h) * dv + row] : 0.f;
    }
    __syncthreads();
    const float gam = coef[kVerifyMaxDrafts];
#pragma unroll
    for (int jr = 0; jr < kVerifyRows; ++jr) {
#pragma unroll
        for (int i = 0; i < kVerifyF4; ++i) {
            x[jr][i].x *= gam; x[jr][i].y *= gam; x[jr][i].z *= gam; x[jr][i].w *= gam;
        }
    }
    for (int t = 0; t < a; ++t) {
        float4 kk[kVerifyF4];
#pragma unroll
        for (int i = 0; i < kVerifyF4; ++i) kk[i] = ks[t][li + LPR * i];
#pragma unroll
        for (int jr = 0; jr < kVerifyRows; ++jr) {
            const float f = us[t][(jr * kVerifyWarps + warp) * RPW + sub];
#pragma unroll
            for (int i = 0; i < kVerifyF4; ++i) {
                x[jr][i].x = fmaf(f, kk[i].x, x[jr][i].x);
                x[jr][i].y = fmaf(f, kk[i].y, x[jr][i].y);
                x[jr][i].z = fmaf(f, kk[i].z, x[jr][i].z);
                x[jr][i].w = fmaf(f, kk[i].w, x[jr][i].w);
            }
        }
    }
#pragma unroll
    for (int jr = 0; jr < kVerifyRows; ++jr) {
        const int row = base + (jr * kVerifyWarps + warp) * RPW + sub;
        if (row >= dv) continue;
#pragma unroll
        for (int i = 0; i < kVerifyF4; ++i)
            __stcs(reinterpret_cast<float4 *>(S + (size_t)row * DK) + li + LPR * i, x[jr][i]);
    }
}

template <int DK, int KT, typename Tin>
void launch_verify_wy(const VerifyArgs &a, dim3 grid, dim3 block, cudaStream_t stream) {
    auto kern = a.prologue ? verify_wy_kernel<DK, KT, Tin, true> : verify_wy_kernel<DK, KT, Tin, false>;
    kern<<<grid, block, 0, stream>>>(
        static_cast<const Tin *>(a.q), static_cast<const Tin *>(a.k),
        static_cast<const Tin *>(a.v), a.g, a.beta, a.state, a.u, static_cast<Tin *>(a.o), a.K,
        a.HK, a.HV, a.dv, a.scale, a.prologue);
}

template <int DK, typename Tin>
void launch_verify_wy_k(const VerifyArgs &a, dim3 grid, dim3 block, cudaStream_t stream) {
    if (a.K <= 4)
        launch_verify_wy<DK, 4, Tin>(a, grid, block, stream);
    else if (a.K <= 8)
        launch_verify_wy<DK, 8, Tin>(a, grid, block, stream);
    else
        launch_verify_wy<DK, 16, Tin>(a, grid, block, stream);
}

template <int DK, typename Tin>
void launch_verify_seq(const VerifyArgs &a, dim3 grid, dim3 block, cudaStream_t stream) {
    auto kern = a.prologue ? verify_kernel<DK, Tin, true> : verify_kernel<DK, Tin, false>;
    kern<<<grid, block, 0, stream>>>(static_cast<const Tin *>(a.q), static_cast<const Tin *>(a.k),
                                     static_cast<const Tin *>(a.v), a.g, a.beta, a.state,
                                     a.states, a.u, static_cast<Tin *>(a.o), a.K, a.HK, a.HV,
                                     a.dv, a.scale, a.prologue);
}

template <typename Tin>
cudaError_t launch_verify_typed(const VerifyArgs &a, cudaStream_t stream) {
    const int band = a.dk == 128 ? verify_band<128>() : a.dk == 64 ? verify_band<64>()
                                                                   : verify_band<32>();
    const dim3 grid((unsigned)((size_t)a.N * a.HV), (unsigned)((a.dv + band - 1) / band)),
        block(kVerifyWarps * 32);
    if (a.states == nullptr) {
        // no per-draft states asked for: the state is never updated in registers
        switch (a.dk) {
            case 32: launch_verify_wy_k<32, Tin>(a, grid, block, stream); break;
            case 64: launch_verify_wy_k<64, Tin>(a, grid, block, stream); break;
            case 128: launch_verify_wy_k<128, Tin>(a, grid, block, stream); break;
            default: return cudaErrorInvalidValue;
        }
        return cudaGetLastError();
    }
    switch (a.dk) {
        case 32: launch_verify_seq<32, Tin>(a, grid, block, stream); break;
        case 64: launch_verify_seq<64, Tin>(a, grid, block, stream); break;
        case 128: launch_verify_seq<128, Tin>(a, grid, block, stream); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_verify(const VerifyArgs &a, cudaStream_t stream) {
    if (a.N == 0) return cudaSuccess;
    return a.dtype == GDN_BF16 ? launch_verify_typed<__nv_bfloat16>(a, stream)
                               : launch_verify_typed<float>(a, stream);
}

template <int DK, typename Tin>
void launch_commit_dk(const CommitDeltasArgs &a, dim3 grid, dim3 block, cudaStream_t stream) {
    auto kern = a.prologue ? commit_deltas_kernel<DK, Tin, true> : commit_deltas_kernel<DK, Tin, false>;
    kern<<<grid, block, 0, stream>>>(static_cast<const Tin *>(a.k), a.g, a.u, a.accepted, a.state,
                                     a.K, a.HK, a.HV, a.dv, a.prologue);
}

template <typename Tin>
cudaError_t launch_commit_deltas_typed(const CommitDeltasArgs &a, cudaStream_t stream) {
    const int band = a.dk == 128 ? verify_band<128>() : a.dk == 64 ? verify_band<64>()
                                                                   : verify_band<32>();
    const dim3 grid((unsigned)((size_t)a.N * a.HV), (unsigned)((a.dv + band - 1) / band)),
        block(kVerifyWarps * 32);
    switch (a.dk) {
        case 32: launch_commit_dk<32, Tin>(a, grid, block, stream); break;
        case 64: launch_commit_dk<64, Tin>(a, grid, block, stream); break;
        case 128: launch_commit_dk<128, Tin>(a, grid, block, stream); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_commit_deltas(const CommitDeltasArgs &a, cudaStream_t stream) {
    if (a.N == 0) return cudaSuccess;
    return a.dtype == GDN_BF16 ? launch_commit_deltas_typed<__nv_bfloat16>(a, stream)
                               : launch_commit_deltas_typed<float>(a, stream);
}

cudaError_t launch_commit(const float *states, const int32_t *accepted, float *state, int N, int K,
                          int HV, int dv, int dk, cudaStream_t stream) {
    if (N == 0) return cudaSuccess;
    const size_t elems = (size_t)dv * dk;
    const unsigned ys = (unsigned)((elems / 4 + 2047) / 2048);
    commit_kernel<<<dim3((unsigned)((size_t)N * HV), ys), 256, 0, stream>>>(states, accepted, state,
                                                                          K, HV, elems);
    return cudaGetLastError();
}

}  // namespace gdn
