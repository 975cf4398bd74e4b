// Multi-token verify of speculative drafts for the gated delta rule, and the two
// roll-back calls that keep the accepted prefix.
//
// Speculative decoding ("Qwen3-Next", sghael.github.io, section "Speed depends on
// the serving software"): drafted tokens are verified together and only an
// accepted prefix is kept.  For the recurrence that means running K draft
// tokens through the decode rule from one state, then keeping the state after
// the last accepted draft.
//
// Rule per draft t and row i of the dv x dk state (decay first, then correct
// along the key; read-out after the update), alpha_t = exp(g_t):
//     u_i  = beta_t (v_i - alpha_t S_i . k_t)
//     S_i <- alpha_t S_i + u_i k_t             o_i = scale * S_i(new) . q_t
//
// Kernels: single streaming passes over fp32 state bands (64 rows at dk = 128,
// 32 KB) of one (sequence, value head), CTAs of 8 warps, rows of dk fp32 held by
// dk/16 lanes with four float4 each (lane l of a row owns float4 l, l + dk/16,
// ..., so a warp instruction reads whole 128-byte lines), two rows per lane:
//   verify_kernel          per-draft states asked for: the band stays in
//                          registers from draft to draft
//   verify_setup_kernel +  update vectors only: per-head tables, then a
//   verify_wy_kernel       persistent pass fed by bulk copies through a ring of
//                          shared-memory stages (the state is only read)
//   verify_tc_kernel       the same products on tensor cores (bf16 inputs,
//                          dk = dv = 128, up to 8 drafts)
//   commit_kernel          copy of the state after the last kept draft
//   commit_deltas_kernel   in-place rebuild from S_0 and the kept u_t
#include "gdn_common.cuh"
#include "gdn_internal.h"
#include <type_traits>

#include "tc_primitives.cuh"
#include "tma_host.h"

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
__device__ __forceinline__ void normalize_row(float4 *row, int lane) {
    float ss = 0.f;
    for (int j = lane; j < DK / 4; j += 32) ss += dot4(row[j], row[j]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float r = inv_l2norm(ss);
    for (int j = lane; j < DK / 4; j += 32) row[j] = scale4(row[j], r);
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

template <int DK, typename Tin, bool PRO, bool RD>
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
    // per-row decays (GDN_ROW_DECAY), only in the row-decay instance
    __shared__ float ar[RD ? kVerifyMaxDrafts : 1][RD ? BAND : 1];
    constexpr bool rowdec = RD;
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
        if (RD)
            ar[RD ? t : 0][RD ? r : 0] =
                row < dv ? gate_alpha(g[(((size_t)n * K + t) * HV + h) * dv + row], pro) : 1.f;
    }
    if (threadIdx.x < K) {
        const size_t gi = ((size_t)n * K + threadIdx.x) * HV + h;
        al[threadIdx.x] = rowdec ? 1.f : gate_alpha(g[gi], pro);
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
        const float alpha_h = al[t], b = be[t];
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
            const float alpha = rowdec ? ar[RD ? t : 0][RD ? r : 0] : alpha_h;
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
//   u_t = beta_t v_t - a1_t a_t - sum_{j<t} ck_tj u_j,     a_t = S_0[r] . k_t
//   o_t = b1_t b_t + sum_{j<=t} cq_tj u_j,                 b_t = S_0[r] . q_t
// with a1_t = beta_t alpha_t gamma_{t-1}, ck_tj = beta_t alpha_t G(j,t-1) (k_j . k_t),
// b1_t = scale gamma_t, cq_tj = scale G(j,t) (k_j . q_t), gamma_t = prod_{s<=t} alpha_s
// and G(j,t) = prod_{j<s<=t} alpha_s.  The recurrence is linear: with
// M = (I + Ck)^-1 (unit lower triangular, K x K),
//   u = M diag(beta) v - M diag(a1) a,      o = diag(b1) b + Cq u,
// and a, b are themselves linear in the row S_0[r].  So every output of a row is
// one dot product of S_0[r] with a vector mixed once per (sequence, value head):
//   u_t = S_0[r] . k'_t + sum_j Vu_tj v_j[r],   k'_t = -sum_j M_tj a1_j k_j,    Vu = M diag(beta)
//   o_t = S_0[r] . q'_t + sum_j Vy_tj v_j[r],   q'_t = b1_t q_t + sum_j E_tj k_j,
//                                               E = -Cq M diag(a1),            Vy = Cq Vu.
// verify_setup_kernel builds k', q', Vu, Vy per (sequence, value head) into a
// workspace (one small CTA each, many resident per SM, so their serial K-step
// loops overlap); verify_wy_kernel streams the state bands and does 2K plain dot
// products per row.

// workspace: a 16-byte header (word 0: status of the streaming kernel's bounded
// waits, 0 = ok), then per (sequence, value head) k', q' [K][dk], Vu, Vy [K][K],
// rounded up to 16 bytes
constexpr int kWsHeaderFloats = 4;
__host__ __device__ inline size_t wy_item_floats(int K, int dk) {
    return ((size_t)2 * K * dk + 2 * (size_t)K * K + 3) & ~(size_t)3;
}
// fused commit-then-verify: after all the items' tables, per (sequence, value head)
// the previous round's kept drafts as kt~_t = c_t k_t [Kp][dk] (c_t = prod_{t<s<a}
// alpha_s), then gamma = prod_{s<a} alpha_s and the kept count a (as int bits)
__host__ __device__ inline size_t pend_item_floats(int Kp, int dk) {
    return ((size_t)Kp * dk + 4 + 3) & ~(size_t)3;
}

// one warp per (sequence, value head); a CTA holds a few such warps, each with
// its own shared-memory slice, and only warp-level syncs
template <int KT>
__host__ __device__ constexpr int setup_warps() { return KT <= 8 ? 4 : 2; }

template <int DK, int KT>
struct SetupSlice {
    float4 ks[KT][DK / 4], qs[KT][DK / 4];
    float al[KT], be[KT], a1[KT], b1[KT];
    float gkk[KT][KT], gkq[KT][KT], ck[KT][KT], cq[KT][KT], Mi[KT][KT], Dm[KT][KT], Em[KT][KT];
};

template <int DK, int KT, typename Tin, bool PRO>
__global__ void __launch_bounds__(setup_warps<KT>() * 32)
verify_setup_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k,
                    const float *__restrict__ g, const float *__restrict__ beta,
                    float *__restrict__ ws, int items, int K, int HK, int HV, float scale,
                    unsigned pro_arg, const Tin *__restrict__ pk, const float *__restrict__ pg,
                    const int32_t *__restrict__ accepted, float *__restrict__ pend, int Kp) {
    const unsigned pro = PRO ? pro_arg : 0u;
    constexpr int D4 = DK / 4;
    __shared__ SetupSlice<DK, KT> slices[setup_warps<KT>()];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nh = blockIdx.x * setup_warps<KT>() + warp;
    if (nh >= items) return;   // whole warps only; nothing below syncs the block
    SetupSlice<DK, KT> &S = slices[warp];
    const int n = nh / HV, h = nh - n * HV;
    const int c = h / (HV / HK);
    for (int idx = lane; idx < K * D4; idx += 32) {
        const int t = idx / D4, j = idx - t * D4;
        const size_t off = (((size_t)n * K + t) * HK + c) * DK + 4 * j;
        S.ks[t][j] = load4(k + off);
        S.qs[t][j] = load4(q + off);
    }
    if (lane < K) {
        const size_t gi = ((size_t)n * K + lane) * HV + h;
        S.al[lane] = gate_alpha(g[gi], pro);
        S.be[lane] = gate_beta(beta[gi], pro);
    }
    __syncwarp();
    if (pro & GDN_PROLOGUE_NORM_K)
        for (int t = 0; t < K; ++t) normalize_row<DK>(S.ks[t], lane);
    if (pro & GDN_PROLOGUE_NORM_Q)
        for (int t = 0; t < K; ++t) normalize_row<DK>(S.qs[t], lane);
    __syncwarp();
    // Gram products: one lane per entry, each walking the columns from its own
    // offset (rows of the same column would share a bank)
    for (int p = lane; p < 2 * K * K; p += 32) {
        const int which = p / (K * K), rem = p - which * K * K;
        const int j = rem / K, t = rem - j * K;
        const float4 *a = S.ks[j];
        const float4 *b = which ? S.qs[t] : S.ks[t];
        float acc = 0.f;
#pragma unroll 8
        for (int f = 0; f < D4; ++f) {
            const int fs = (f + lane) & (D4 - 1);
            acc += dot4(a[fs], b[fs]);
        }
        (which ? S.gkq : S.gkk)[j][t] = acc;
    }
    __syncwarp();
    if (lane < K) {   // recurrence coefficients, one lane per draft
        const int t = lane;
        float G = 1.f;   // G(j, t-1), walking j down from t-1
        for (int j = t - 1; j >= 0; --j) {
            S.ck[t][j] = S.be[t] * S.al[t] * G * S.gkk[j][t];
            G *= S.al[j];
        }
        S.a1[t] = S.be[t] * S.al[t] * G;   // G is now gamma_{t-1}
        float H = 1.f;   // G(j, t)
        for (int j = t; j >= 0; --j) {
            S.cq[t][j] = scale * H * S.gkq[j][t];
            H *= S.al[j];
        }
        S.b1[t] = scale * H;               // scale * gamma_t
    }
    __syncwarp();
    if (lane < K) {   // M = (I + Ck)^-1 by forward substitution, one lane per column
        const int col = lane;
        for (int t = 0; t < K; ++t) {
            float m = (t == col) ? 1.f : 0.f;
            for (int j = col; j < t; ++j) m = fmaf(-S.ck[t][j], S.Mi[j][col], m);
            S.Mi[t][col] = t >= col ? m : 0.f;
        }
    }
    __syncwarp();
    float *out = ws + kWsHeaderFloats + (size_t)nh * wy_item_floats(K, DK);
    float *vu_out = out + 2 * (size_t)K * DK, *vy_out = vu_out + (size_t)K * K;
    for (int e = lane; e < K * K; e += 32) {   // D = -M diag(a1), Vu = M diag(beta)
        const int t = e / K, j = e - t * K;
        S.Dm[t][j] = -S.Mi[t][j] * S.a1[j];
        vu_out[e] = S.Mi[t][j] * S.be[j];
    }
    __syncwarp();
    for (int e = lane; e < K * K; e += 32) {   // E = Cq D, Vy = Cq Vu
        const int t = e / K, i = e - t * K;
        float ev = 0.f, vv = 0.f;
        for (int j = i; j <= t; ++j) {
            ev = fmaf(S.cq[t][j], S.Dm[j][i], ev);
            vv = fmaf(S.cq[t][j], S.Mi[j][i] * S.be[i], vv);
        }
        S.Em[t][i] = ev;
        vy_out[e] = vv;
    }
    __syncwarp();
    float4 *kp = reinterpret_cast<float4 *>(out), *qp = kp + (size_t)K * D4;
    for (int idx = lane; idx < K * D4; idx += 32) {   // mixed key and query vectors
        const int t = idx / D4, f = idx - t * D4;
        float4 kk = make_float4(0.f, 0.f, 0.f, 0.f);
        float4 qq = scale4(S.qs[t][f], S.b1[t]);
        for (int j = 0; j <= t; ++j) {
            const float4 kj = S.ks[j][f];
            const float d = S.Dm[t][j], e = S.Em[t][j];
            kk.x = fmaf(d, kj.x, kk.x); kk.y = fmaf(d, kj.y, kk.y);
            kk.z = fmaf(d, kj.z, kk.z); kk.w = fmaf(d, kj.w, kk.w);
            qq.x = fmaf(e, kj.x, qq.x); qq.y = fmaf(e, kj.y, qq.y);
            qq.z = fmaf(e, kj.z, qq.z); qq.w = fmaf(e, kj.w, qq.w);
        }
        kp[idx] = kk;
        qp[idx] = qq;
    }
    if (pend == nullptr) return;
    // ---- the previous round's kept drafts (fused commit-then-verify) ----
    __syncwarp();   // the slice's rows are read by the loop above
    float *po = pend + (size_t)nh * pend_item_floats(Kp, DK);
    int a = accepted[n];
    if (a < 0 || a > Kp) a = 0;
    for (int idx = lane; idx < a * D4; idx += 32) {
        const int t = idx / D4, j = idx - t * D4;
        S.ks[t][j] = load4(pk + (((size_t)n * Kp + t) * HK + c) * DK + 4 * j);
    }
    if (lane < a) S.al[lane] = gate_alpha(pg[((size_t)n * Kp + lane) * HV + h], pro);
    __syncwarp();
    if (pro & GDN_PROLOGUE_NORM_K)
        for (int t = 0; t < a; ++t) normalize_row<DK>(S.ks[t], lane);
    if (lane == 0) {   // c_t = prod_{t<s<a} alpha_s, gamma = prod_{s<a} alpha_s
        float c_run = 1.f;
        for (int t = a - 1; t >= 0; --t) {
            S.a1[t] = c_run;
            c_run *= S.al[t];
        }
        po[(size_t)Kp * DK] = c_run;
        po[(size_t)Kp * DK + 1] = __int_as_float(a);
    }
    __syncwarp();
    float4 *ko = reinterpret_cast<float4 *>(po);
    for (int idx = lane; idx < a * D4; idx += 32) {
        const int t = idx / D4, f = idx - t * D4;
        ko[idx] = scale4(S.ks[t][f], S.a1[t]);
    }
}

// Streaming kernel, persistent: each CTA walks bands b = blockIdx.x + i * gridDim.x
// of the (sequence, value head, band) list.  Thread 0 keeps NST bands in flight:
// every band's 32 KB of state rows (contiguous) and its head's tables arrive by
// 1-D bulk copies into a ring of shared-memory stages, completing on the stage's
// mbarrier, so the state stream does not stop while the CTA computes.  Per band:
// 2K dot products per row against S_0, a reduce-scatter over the row's lanes (a
// lane keeps the upper half of its values where its lane bit is set, the lower
// half otherwise) and the outputs the lane ends up holding.  One block barrier per
// band, which also frees the previous band's stage for the next copy.  Waits are
// bounded: a timeout sets the workspace status word, and the CTA drains its copies
// in flight (bounded) before it returns.
constexpr uint32_t kWyWaitLimit = 2000;   // ~2 s of 1 ms sleeping polls

template <int KT, bool FUSED>
__host__ __device__ constexpr int wy_stages() { return (KT <= 4 && !FUSED) ? 3 : 2; }
template <int DK, int KT, bool FUSED>
__host__ __device__ constexpr size_t wy_stage_bytes() {
    return (size_t)verify_band<DK>() * DK * sizeof(float) +
           ((2 * (size_t)KT * DK + 2 * (size_t)KT * KT + 3) & ~(size_t)3) * sizeof(float) +
           (FUSED ? (((size_t)KT * DK + 4 + 3) & ~(size_t)3) * sizeof(float) : 0);
}
template <int DK, int KT, bool FUSED>
__host__ __device__ constexpr size_t wy_smem_bytes() {
    // stages, the v (and, fused, previous u) buffers [2][KT][BAND] fp32, the mbarriers
    return wy_stages<KT, FUSED>() * wy_stage_bytes<DK, KT, FUSED>() +
           (FUSED ? 4 : 2) * (size_t)KT * verify_band<DK>() * sizeof(float) +
           wy_stages<KT, FUSED>() * sizeof(uint64_t) + 16;
}

// TMO: a test-only instance whose first wait -- before thread 0 issues any copy --
// has a limit of zero polls on a stage barrier nothing has armed: the timeout path
// (status word, early return with nothing in flight) runs without a real hang.
template <int DK, int KT, typename Tin, bool FUSED, bool TMO = false>
__global__ void __launch_bounds__(kVerifyWarps * 32, KT <= 8 ? 2 : 1)
verify_wy_kernel(const Tin *__restrict__ v, float *state, float *__restrict__ ws,
                 float *__restrict__ u_out, Tin *__restrict__ o, int N, int K, int HV, int dv,
                 const float *__restrict__ prev_u, int Kp) {
    constexpr int LPR = DK / (4 * kVerifyF4);   // lanes per row: 2, 4, 8
    constexpr int RPW = 32 / LPR;
    constexpr int BAND = verify_band<DK>();
    constexpr int D4 = DK / 4;
    constexpr int NV = 2 * KT;                  // partial sums per row: u then o
    static_assert(NV % LPR == 0, "reduce-scatter needs 2 KT >= lanes per row");
    constexpr int NL = NV / LPR;                // finished values per lane
    constexpr int NST = wy_stages<KT, FUSED>();
    constexpr size_t SB = wy_stage_bytes<DK, KT, FUSED>();
    extern __shared__ __align__(128) uint8_t wy_smem[];
    // v (and, fused, the previous round's u) of a band, loaded one band ahead (plain
    // loads into registers during the previous band's arithmetic, stored here after it)
    float *vsm = reinterpret_cast<float *>(wy_smem + NST * SB);   // [2][KT][BAND]
    float *usm = vsm + 2 * KT * BAND;                            // [2][KT][BAND], fused only
    uint64_t *bars = reinterpret_cast<uint64_t *>(vsm + (FUSED ? 4 : 2) * KT * BAND);
    constexpr int VPT = (KT * BAND + kVerifyWarps * 32 - 1) / (kVerifyWarps * 32);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int sub = lane / LPR, li = lane % LPR;
    const int nbands = (dv + BAND - 1) / BAND;
    const long long total = (long long)N * HV * nbands;
    const long long mine = total > blockIdx.x ? (total - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const size_t item_floats = wy_item_floats(K, DK);
    const float *tables = ws + kWsHeaderFloats;
    const size_t pend_floats = FUSED ? pend_item_floats(Kp, DK) : 0;
    const float *pend = tables + (size_t)N * HV * item_floats;

    // (value-head index, band) of this CTA's i-th band, b = blockIdx.x + i * gridDim.x,
    // advanced by the grid stride without a division per band
    struct BandIt {
        int nh, y;
        __device__ void init(long long b, int nb) {
            nh = (int)(b / nb);
            y = (int)(b - (long long)nh * nb);
        }
        __device__ void next(int step_nh, int step_y, int nb) {
            nh += step_nh;
            y += step_y;
            if (y >= nb) {
                y -= nb;
                ++nh;
            }
        }
    };
    const int step_nh = (int)(gridDim.x / nbands), step_y = (int)(gridDim.x % nbands);
    auto band_rows = [&](int y) { return dv - y * BAND < BAND ? dv - y * BAND : BAND; };
    BandIt it_issue;   // thread 0: the next band to copy in
    it_issue.init(blockIdx.x, nbands);
    auto issue = [&](long long i) {   // thread 0: band i of this CTA into stage i % NST
        const int nh = it_issue.nh, base = it_issue.y * BAND, rows = band_rows(it_issue.y);
        it_issue.next(step_nh, step_y, nbands);
        uint8_t *stg = wy_smem + (i % NST) * SB;
        uint64_t *bar = &bars[i % NST];
        const uint32_t sbytes = (uint32_t)rows * DK * sizeof(float);
        const uint32_t tbytes = (uint32_t)(item_floats * sizeof(float));
        const uint32_t pbytes = (uint32_t)(pend_floats * sizeof(float));
        tc::mbar_arrive_expect_tx(bar, sbytes + tbytes + pbytes);
        tc::bulk_load_g2s(stg, state + ((size_t)nh * dv + base) * DK, sbytes, bar);
        tc::bulk_load_g2s(stg + (size_t)BAND * DK * sizeof(float), tables + (size_t)nh * item_floats,
                          tbytes, bar);
        if (FUSED)
            tc::bulk_load_g2s(stg + (size_t)BAND * DK * sizeof(float) + tbytes,
                              pend + (size_t)nh * pend_floats, pbytes, bar);
    };
    BandIt it_v;   // the band whose v is loaded next
    it_v.init(blockIdx.x, nbands);
    auto load_v = [&](float (&vr)[VPT], float (&ur)[VPT]) {   // band it_v, then advance it
        const int nh = it_v.nh, base = it_v.y * BAND, rows = band_rows(it_v.y);
        it_v.next(step_nh, step_y, nbands);
        const int n = nh / HV, h = nh - n * HV;
#pragma unroll
        for (int e0 = 0; e0 < VPT; ++e0) {
            const int e = tid + e0 * kVerifyWarps * 32;
            const int j = e / BAND, r = e - j * BAND;
            vr[e0] = (j < K && r < rows) ? to_f32(v[(((size_t)n * K + j) * HV + h) * dv + base + r])
                                         : 0.f;
            if (FUSED)
                ur[e0] = (j < Kp && r < rows) ? prev_u[(((size_t)n * Kp + j) * HV + h) * dv + base + r]
                                              : 0.f;
        }
    };
    auto store_v = [&](long long i, const float (&vr)[VPT], const float (&ur)[VPT]) {
        float *dst = vsm + (i & 1) * KT * BAND;
        float *udst = usm + (i & 1) * KT * BAND;
#pragma unroll
        for (int e0 = 0; e0 < VPT; ++e0) {
            const int e = tid + e0 * kVerifyWarps * 32;
            if (e < KT * BAND) {
                dst[e] = vr[e0];
                if (FUSED) udst[e] = ur[e0];
            }
        }
    };
    if (TMO) {
        int gave_up = 0;
        if (tid == 0) {
            for (int st = 0; st < NST; ++st) tc::mbar_init(&bars[st], 1);
            tc::fence_barrier_init();
            if (!tc::mbar_test_wait(&bars[0], 0u)) {
                atomicExch(reinterpret_cast<unsigned int *>(ws), 1u);
                gave_up = 1;
            }
        }
        if (__syncthreads_or(gave_up)) return;
    }
    if (tid == 0) {
        if (!TMO) {
            for (int st = 0; st < NST; ++st) tc::mbar_init(&bars[st], 1);
            tc::fence_barrier_init();
        }
        for (long long i = 0; i < NST && i < mine; ++i) issue(i);
    }
    if (mine > 0) {
        float vr[VPT], ur[VPT];
        load_v(vr, ur);
        store_v(0, vr, ur);
    }
    __syncthreads();
    BandIt it;   // the band being computed
    it.init(blockIdx.x, nbands);
    long long issued = mine < NST ? mine : NST, done = 0;
    bool ok = true;
    for (long long i = 0; i < mine; ++i) {
        const int st = (int)(i % NST);
        bool landed = tc::mbar_wait(&bars[st], (uint32_t)((i / NST) & 1), kWyWaitLimit);
        ok = __syncthreads_and(landed);   // also: every thread is done with band i - 1
        if (!ok) break;
        done = i + 1;
        if (tid == 0 && i >= 1 && i - 1 + NST < mine) {   // band i - 1's stage is free again
            issue(i - 1 + NST);
            ++issued;
        }
        float vnext[VPT], unext[VPT];
        if (i + 1 < mine) load_v(vnext, unext);   // band i + 1: lands during this band's arithmetic
        const int nh = it.nh, base = it.y * BAND, rows = band_rows(it.y);
        it.next(step_nh, step_y, nbands);
        const int n = nh / HV, h = nh - n * HV;
        const float *vb = vsm + (i & 1) * KT * BAND;   // [j][r] of this band
        const uint8_t *stg = wy_smem + st * SB;
        const float4 *srow = reinterpret_cast<const float4 *>(stg);
        const float *item = reinterpret_cast<const float *>(stg + (size_t)BAND * DK * sizeof(float));
        const float4 *kp = reinterpret_cast<const float4 *>(item);
        const float4 *qp = kp + (size_t)K * D4;
        const float *vu = item + 2 * (size_t)K * DK, *vy = vu + (size_t)K * K;
        float4 s[kVerifyRows][kVerifyF4];
#pragma unroll
        for (int jr = 0; jr < kVerifyRows; ++jr) {
            const int r = (jr * kVerifyWarps + warp) * RPW + sub;
#pragma unroll
            for (int q4 = 0; q4 < kVerifyF4; ++q4) s[jr][q4] = srow[r * D4 + li + LPR * q4];
        }
        if (FUSED) {
            // commit the previous round's kept drafts into the band first:
            // S <- gamma S + sum_{t<a} u_t[r] kt~_t, written back to the state
            const float *pitem = item + item_floats;
            const int a = __float_as_int(pitem[(size_t)Kp * DK + 1]);
            if (a > 0) {
                const float gam = pitem[(size_t)Kp * DK];
                const float4 *pkt = reinterpret_cast<const float4 *>(pitem);
                const float *ub = usm + (i & 1) * KT * BAND;
#pragma unroll
                for (int jr = 0; jr < kVerifyRows; ++jr) {
                    const int r = (jr * kVerifyWarps + warp) * RPW + sub;
#pragma unroll
                    for (int q4 = 0; q4 < kVerifyF4; ++q4) s[jr][q4] = scale4(s[jr][q4], gam);
                    for (int t = 0; t < a; ++t) {
                        const float f = ub[t * BAND + r];
                        const float2 ff = make_float2(f, f);
#pragma unroll
                        for (int q4 = 0; q4 < kVerifyF4; ++q4) {
                            const float4 kk = pkt[t * D4 + li + LPR * q4];
                            const float2 lo = fma2(ff, make_float2(kk.x, kk.y),
                                                   make_float2(s[jr][q4].x, s[jr][q4].y));
                            const float2 hi = fma2(ff, make_float2(kk.z, kk.w),
                                                   make_float2(s[jr][q4].z, s[jr][q4].w));
                            s[jr][q4] = make_float4(lo.x, lo.y, hi.x, hi.y);
                        }
                    }
                    if (r < rows) {
                        float4 *dst = reinterpret_cast<float4 *>(state + ((size_t)nh * dv + base + r) * DK);
#pragma unroll
                        for (int q4 = 0; q4 < kVerifyF4; ++q4) __stcs(dst + li + LPR * q4, s[jr][q4]);
                    }
                }
            }
        }
        // dot products on packed pairs (even / odd columns), summed once at the end
        float2 acc2[kVerifyRows][NV];
#pragma unroll
        for (int jr = 0; jr < kVerifyRows; ++jr)
#pragma unroll
            for (int m = 0; m < NV; ++m) acc2[jr][m] = make_float2(0.f, 0.f);
#pragma unroll
        for (int t = 0; t < KT; ++t) {
            if (t < K) {
#pragma unroll
                for (int q4 = 0; q4 < kVerifyF4; ++q4) {
                    const float4 kv = kp[t * D4 + li + LPR * q4], qv = qp[t * D4 + li + LPR * q4];
                    const float2 klo = make_float2(kv.x, kv.y), khi = make_float2(kv.z, kv.w);
                    const float2 qlo = make_float2(qv.x, qv.y), qhi = make_float2(qv.z, qv.w);
#pragma unroll
                    for (int jr = 0; jr < kVerifyRows; ++jr) {
                        const float4 x = s[jr][q4];
                        const float2 xlo = make_float2(x.x, x.y), xhi = make_float2(x.z, x.w);
                        acc2[jr][t] = fma2(xhi, khi, fma2(xlo, klo, acc2[jr][t]));
                        acc2[jr][KT + t] = fma2(xhi, qhi, fma2(xlo, qlo, acc2[jr][KT + t]));
                    }
                }
            }
        }
        float acc[kVerifyRows][NV];
#pragma unroll
        for (int jr = 0; jr < kVerifyRows; ++jr)
#pragma unroll
            for (int m = 0; m < NV; ++m) acc[jr][m] = acc2[jr][m].x + acc2[jr][m].y;
#pragma unroll
        for (int jr = 0; jr < kVerifyRows; ++jr) {
            int n_cur = NV;
#pragma unroll
            for (int off = LPR / 2; off > 0; off >>= 1) {
                const bool upper = (li & off) != 0;
                const int half = n_cur / 2;
#pragma unroll
                for (int m = 0; m < NV / 2; ++m) {
                    if (m < half) {
                        const float keep = upper ? acc[jr][m + half] : acc[jr][m];
                        const float send = upper ? acc[jr][m] : acc[jr][m + half];
                        acc[jr][m] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                    }
                }
                n_cur = half;
            }
        }
        int first = 0;   // index of this lane's first finished value
        {
            int half = NV / 2;
#pragma unroll
            for (int off = LPR / 2; off > 0; off >>= 1) {
                if (li & off) first += half;
                half /= 2;
            }
        }
#pragma unroll
        for (int jr = 0; jr < kVerifyRows; ++jr) {
            const int r = (jr * kVerifyWarps + warp) * RPW + sub;
            if (r >= rows) continue;
            const int row = base + r;
#pragma unroll
            for (int m = 0; m < NL; ++m) {
                const int idx = first + m;
                const bool is_u = idx < KT;
                const int t = is_u ? idx : idx - KT;
                if (t >= K || (is_u && !u_out)) continue;
                const float *coef = (is_u ? vu : vy) + t * K;
                float val = acc[jr][m];
                for (int j = 0; j <= t; ++j) val = fmaf(coef[j], vb[j * BAND + r], val);
                const size_t ot = (((size_t)n * K + t) * HV + h) * dv + row;
                if (is_u)
                    u_out[ot] = val;
                else
                    o[ot] = from_f32<Tin>(val);
            }
        }
        if (i + 1 < mine) store_v(i + 1, vnext, unext);   // published by the next band's barrier
    }
    if (!ok && tid == 0) {
        atomicExch(reinterpret_cast<unsigned int *>(ws), 1u);
        // copies still in flight land before this CTA's shared memory is released
        for (long long i = done; i < issued; ++i)
            tc::mbar_wait(&bars[i % NST], (uint32_t)((i / NST) & 1), kWyWaitLimit);
    }
}

// Update vectors on tensor cores (bf16 inputs, dk = dv = 128, K <= 8).  The 2K
// dot products per state row of the streaming kernel above are, per (sequence,
// value head), one product of the [128 x 128] state with the 16 mixed vectors
// (k'_t in row t, q'_t in row 8 + t).  Both factors are split into bf16 hi + lo:
// the B operand stacks [k'; q'] hi (rows 0..15) over its lo parts (rows
// 16..31), and D = S_hi B^T + S_lo B^T (N = 32) gives in column n + 16 c the
// product with part c of mixed vector n, so D[:, n] + D[:, n + 16] is the whole
// fp32 dot product up to the rounding of the two lo parts (~2^-17 of each
// term, the order of fp32 accumulation over 128 terms).
//   * states stream through three 64 KB shared-memory stages by TMA (four
//     [128 rows x 32 fp32] boxes, 128-byte swizzle); a stage is refilled with
//     the item three ahead as soon as the CTA has read it;
//   * thread = tensor-memory lane = state row: warps w and w + 4 take the two
//     64-column halves of rows 32 (w % 4) .. + 31, split them into bf16 hi / lo
//     (two per 32-bit column) and store them to tensor memory as the A operand
//     (two buffers);
//   * k', q' (fp32 tables of the setup kernel, read one item ahead into
//     registers) become the swizzled B tile (two buffers);
//   * one elected thread issues 2 x 8 MMAs (M = 128, N = 32, K = 16) into one
//     of two accumulators and commits them to an mbarrier;
//   * the read-out of item i - 1 (accumulator -> registers, plus the K x K
//     value terms, stores of u and o) runs while the MMAs of item i execute.
// Waits are bounded: a timeout sets the workspace status word, and the CTA
// waits (bounded) for its copies and MMAs in flight before it frees its tensor
// memory and returns.  TMO: a test-only instance whose first wait -- before any
// copy or MMA is issued -- has a limit of zero polls on a barrier nothing has
// armed, so the timeout path runs without a real hang.
constexpr int kTcThreads = 256;
constexpr int kTcStages = 3;
constexpr int kTcDrafts = 8;
constexpr uint32_t kTcStateBytes = 128u * 128u * 4u;   // one fp32 state
constexpr uint32_t kTcBTile = 8192;                    // [32 x 128] bf16: hi rows, lo rows
constexpr int kTcCoef = 2 * kTcDrafts * kTcDrafts;    // Vu, Vy, each [8][8]
// tensor-memory columns: A (hi 64 + lo 64) x 2 buffers, then D (32) x 2
constexpr uint32_t kTcColA = 0, kTcColD = 256, kTcCols = 512;
constexpr size_t tc_smem_bytes() {
    return 1024 + kTcStages * (size_t)kTcStateBytes + 2 * (size_t)kTcBTile +
           kTcStages * (size_t)kTcCoef * sizeof(float) + (kTcStages + 2) * sizeof(uint64_t) + 16;
}

__device__ __forceinline__ void split_bf16x2(float a, float b, uint32_t &hi, uint32_t &lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    const float2 hf = __bfloat1622float2(h);
    hi = *reinterpret_cast<const uint32_t *>(&h);
    lo = tc::pack_bf16x2(a - hf.x, b - hf.y);
}

template <bool TMO = false>
__global__ void __launch_bounds__(kTcThreads, 1)
verify_tc_kernel(const __grid_constant__ CUtensorMap tm_s, const __nv_bfloat16 *__restrict__ v,
                 float *__restrict__ ws, float *__restrict__ u_out, __nv_bfloat16 *__restrict__ o,
                 int N, int K, int HV) {
    extern __shared__ uint8_t tc_smem_raw[];
    const uint32_t raw_s = tc::smem_u32(tc_smem_raw);
    uint8_t *sm = tc_smem_raw + (((raw_s + 1023u) & ~1023u) - raw_s);
    uint8_t *stages = sm;                                         // [3][64 KB]
    uint8_t *btile = sm + kTcStages * (size_t)kTcStateBytes;      // [2][8 KB]
    float *coef = reinterpret_cast<float *>(btile + 2 * kTcBTile);   // [3][Vu | Vy]
    uint64_t *bars = reinterpret_cast<uint64_t *>(coef + kTcStages * kTcCoef);   // stages
    uint64_t *mbar = bars + kTcStages;                                           // MMAs [2]
    uint32_t *slot = reinterpret_cast<uint32_t *>(mbar + 2);
    constexpr uint32_t kIdesc = tc::idesc_bf16(128, 32, false, false);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r = 32 * (warp & 3) + lane;   // this thread's state row (tensor-memory lane)
    const int kh = warp >> 2;               // its column half; also: 0 reads out u, 1 o
    const long long total = (long long)N * HV;
    const int mine = total > blockIdx.x ? (int)((total - 1 - blockIdx.x) / gridDim.x) + 1 : 0;
    const size_t item_floats = wy_item_floats(K, 128);
    const float *tables = ws + kWsHeaderFloats;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;

    // what item nh needs besides its state, read one item ahead: the thread's
    // 8 values of [k'; q'] (row tid / 16, columns 8 (tid % 16) ..), one table
    // coefficient (entry tid of [Vu | Vy] padded to [2][8][8]), and the K values
    // of v at row r (raw bf16).  Heads < 2^31 (the launcher checks).
    struct Pre {
        float4 kq0, kq1;
        float c;
        int n, h;
        unsigned short vr[kTcDrafts];
    };
    auto prefetch = [&](int nh, Pre &p) {
        p.n = nh / HV;
        p.h = nh - p.n * HV;
        const float *tab = tables + (size_t)nh * item_floats;
        const int rr = tid >> 4, t = rr & 7;
        if (t < K) {
            const float4 *src = reinterpret_cast<const float4 *>(
                tab + (size_t)((rr < 8 ? 0 : K) + t) * 128 + (tid & 15) * 8);
            p.kq0 = __ldg(src);
            p.kq1 = __ldg(src + 1);
        } else {
            p.kq0 = p.kq1 = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        const int ct = (tid >> 3) & 7, cj = tid & 7;
        p.c = (tid < kTcCoef && ct < K && cj < K)
                  ? __ldg(tab + 2 * (size_t)K * 128 + (tid >> 6) * K * K + ct * K + cj)
                  : 0.f;
        const unsigned short *vs = reinterpret_cast<const unsigned short *>(v) +
                                   ((size_t)p.n * K * HV + p.h) * 128 + r;
        const size_t vstride = (size_t)HV * 128;
#pragma unroll
        for (int j = 0; j < kTcDrafts; ++j)
            p.vr[j] = j < K ? __ldg(vs + j * vstride) : (unsigned short)0;
    };
    auto issue = [&](int i) {   // thread 0: item i's state into stage i % 3
        const int nh = (int)blockIdx.x + i * (int)gridDim.x;
        uint8_t *dst = stages + (size_t)(i % kTcStages) * kTcStateBytes;
        uint64_t *bar = &bars[i % kTcStages];
        tc::mbar_arrive_expect_tx(bar, kTcStateBytes);
#pragma unroll
        for (int b = 0; b < 4; ++b) tc::tma_load_3d(dst + b * 16384, &tm_s, bar, 32 * b, 0, nh);
    };

    if (tid == 0) {
        for (int b = 0; b < kTcStages + 2; ++b) tc::mbar_init(&bars[b], 1);
        tc::fence_barrier_init();
    }
    if (warp == 0) tc::tmem_alloc(slot, kTcCols);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *slot;
    if (TMO) {
        int gave_up = 0;
        if (tid == 0 && !tc::mbar_test_wait(&bars[0], 0u)) {
            atomicExch(reinterpret_cast<unsigned int *>(ws), 1u);
            gave_up = 1;
        }
        if (__syncthreads_or(gave_up)) {
            if (warp == 0) tc::tmem_dealloc(tmem, kTcCols);
            return;
        }
    }
    int issued = 0;   // thread 0
    if (tid == 0)
        for (; issued < kTcStages && issued < mine; ++issued) issue(issued);

    bool mfail = false;
    // read-out of item p (sequence n, value head h):
    //   u_t = S_0[r] . k'_t + sum_{j<=t} Vu[t][j] v_j[r]   (warps 0-3)
    //   o_t = S_0[r] . q'_t + sum_{j<=t} Vy[t][j] v_j[r]   (warps 4-7)
    auto readout = [&](int p, int n, int h, const unsigned short (&vv)[kTcDrafts]) {
        if (!tc::mbar_wait(&mbar[p & 1], (uint32_t)((p >> 1) & 1), kWyWaitLimit)) mfail = true;
        tc::tc_fence_after();
        float d0[16], d1[16];
        const uint32_t dcol = tmem + kTcColD + (uint32_t)(p & 1) * 32u + lane_off;
        tc::tmem_ld16(dcol, d0);
        tc::tmem_ld16(dcol + 16u, d1);
        tc::tmem_wait_ld();
        const float *cf = coef + (p % kTcStages) * kTcCoef + kh * 64;
        float vf[kTcDrafts];
#pragma unroll
        for (int j = 0; j < kTcDrafts; ++j) vf[j] = __uint_as_float((uint32_t)vv[j] << 16);
        const size_t obase = ((size_t)n * K * HV + h) * 128 + r, ostride = (size_t)HV * 128;
#pragma unroll
        for (int t = 0; t < kTcDrafts; ++t) {
            if (t < K) {
                float val = kh ? d0[8 + t] + d1[8 + t] : d0[t] + d1[t];
#pragma unroll
                for (int j = 0; j <= t; ++j) val = fmaf(cf[t * kTcDrafts + j], vf[j], val);
                if (kh == 0) {
                    if (u_out) u_out[obase + t * ostride] = val;
                } else {
                    o[obase + t * ostride] = __float2bfloat16_rn(val);
                }
            }
        }
    };

    Pre cur, nxt;
    unsigned short vprev[kTcDrafts];
    int nprev = 0, hprev = 0;
    if (mine > 0) prefetch((int)blockIdx.x, cur);
    bool ok = true;
    int consumed = 0;   // items whose state landed and whose MMAs were issued
    for (int i = 0; i < mine; ++i) {
        if (i + 1 < mine) prefetch((int)blockIdx.x + (i + 1) * (int)gridDim.x, nxt);
        const int st = i % kTcStages;
        const bool landed = tc::mbar_wait(&bars[st], (uint32_t)((i / kTcStages) & 1), kWyWaitLimit);
        // row r, columns [64 kh, 64 kh + 64): boxes 2 kh and 2 kh + 1, 16-byte
        // chunk c of a row at chunk position c ^ (r % 8)
        const uint8_t *stg = stages + (size_t)st * kTcStateBytes;
        float4 x[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int box = 2 * kh + (j >> 3), c = j & 7;
            x[j] = *reinterpret_cast<const float4 *>(stg + box * 16384 + r * 128 +
                                                     (((c ^ r) & 7) << 4));
        }
        // A operand: hi at columns [0, 64), lo at [64, 128) of this item's buffer,
        // bf16 pair (2w, 2w + 1) of the row in column w
        const uint32_t abuf = tmem + kTcColA + (uint32_t)(i & 1) * 128u + lane_off + 32u * kh;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float hw[16], lw[16];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 e = x[8 * half + q];
                uint32_t h0, l0, h1, l1;
                split_bf16x2(e.x, e.y, h0, l0);
                split_bf16x2(e.z, e.w, h1, l1);
                hw[2 * q] = __uint_as_float(h0);
                hw[2 * q + 1] = __uint_as_float(h1);
                lw[2 * q] = __uint_as_float(l0);
                lw[2 * q + 1] = __uint_as_float(l1);
            }
            tc::tmem_st16(abuf + 16u * half, hw);
            tc::tmem_st16(abuf + 64u + 16u * half, lw);
        }
        // B operand: row tid / 16 of [k'; q'], columns 8 (tid % 16) .. + 7, as one
        // 16-byte chunk of hi row rr and of lo row 16 + rr (64-column atoms of
        // 32 rows, 4 KB each)
        {
            const int rr = tid >> 4, cc = tid & 15;
            const uint32_t atom = (uint32_t)(cc >> 3) * 4096u;
            uint8_t *bt = btile + (i & 1) * kTcBTile;
            uint32_t hb[4], lb[4];
            split_bf16x2(cur.kq0.x, cur.kq0.y, hb[0], lb[0]);
            split_bf16x2(cur.kq0.z, cur.kq0.w, hb[1], lb[1]);
            split_bf16x2(cur.kq1.x, cur.kq1.y, hb[2], lb[2]);
            split_bf16x2(cur.kq1.z, cur.kq1.w, hb[3], lb[3]);
            *reinterpret_cast<uint4 *>(bt + atom + tc::sw128_chunk((uint32_t)rr, (uint32_t)cc)) =
                make_uint4(hb[0], hb[1], hb[2], hb[3]);
            *reinterpret_cast<uint4 *>(bt + atom + tc::sw128_chunk((uint32_t)(16 + rr), (uint32_t)cc)) =
                make_uint4(lb[0], lb[1], lb[2], lb[3]);
        }
        if (tid < kTcCoef) coef[st * kTcCoef + tid] = cur.c;
        tc::tmem_wait_st();
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        ok = __syncthreads_and(landed && !mfail);   // also: item i - 1's read-out is done
        if (!ok) break;
        consumed = i + 1;
        if (tid == 0 && issued < mine) {   // stage st has been read: the item 3 ahead
            issue(issued);
            ++issued;
        }
        if (warp == 0) {
            tc::tc_fence_after();
            if (tc::elect_one()) {
                const uint32_t dacc = tmem + kTcColD + (uint32_t)(i & 1) * 32u;
                const uint32_t abase = tmem + kTcColA + (uint32_t)(i & 1) * 128u;
                const uint32_t bbase = tc::smem_u32(btile + (i & 1) * kTcBTile);
#pragma unroll
                for (int kk = 0; kk < 16; ++kk) {   // S_hi k-steps, then S_lo k-steps
                    const int k8 = kk & 7;
                    const uint64_t bd = tc::sdesc_sw128(
                        bbase + (uint32_t)(k8 >> 2) * 4096u + (uint32_t)(k8 & 3) * 32u, 16, 1024);
                    tc::mma_bf16_ts(dacc, abase + (kk >= 8 ? 64u : 0u) + 8u * k8, bd, kIdesc, kk > 0);
                }
                tc::mma_commit(&mbar[i & 1]);
            }
            __syncwarp();
        }
        if (i >= 1) readout(i - 1, nprev, hprev, vprev);
#pragma unroll
        for (int j = 0; j < kTcDrafts; ++j) vprev[j] = cur.vr[j];
        nprev = cur.n;
        hprev = cur.h;
        cur = nxt;
    }
    if (ok && mine > 0) readout(mine - 1, nprev, hprev, vprev);
    tc::tc_fence_before();
    const bool all_ok = __syncthreads_and(ok && !mfail);
    if (!all_ok && tid == 0) {
        atomicExch(reinterpret_cast<unsigned int *>(ws), 1u);
        // copies still in flight land, and the last MMAs complete, before this
        // CTA's shared and tensor memory are released
        for (int j = consumed; j < issued; ++j)
            tc::mbar_wait(&bars[j % kTcStages], (uint32_t)((j / kTcStages) & 1), kWyWaitLimit);
        if (consumed > 0)
            tc::mbar_wait(&mbar[(consumed - 1) & 1], (uint32_t)(((consumed - 1) >> 1) & 1), kWyWaitLimit);
    }
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, kTcCols);
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
template <int DK, typename Tin, bool PRO, bool RD>
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
    __shared__ float gr[RD ? BAND : 1];   // per-row decay products (GDN_ROW_DECAY)
    constexpr bool rowdec = RD;
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
    if (threadIdx.x == 0 && !rowdec) {
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
    if (rowdec) {
        // the same products per value row, one thread per row
        for (int r = threadIdx.x; r < BAND; r += blockDim.x) {
            const int row = base + r;
            float c_run = 1.f;
            for (int t = a - 1; t >= 0; --t) {
                const size_t e = (((size_t)n * K + t) * HV + h) * dv + row;
                us[t][r] = row < dv ? c_run * u[e] : 0.f;
                if (row < dv) c_run *= gate_alpha(g[e], pro);
            }
            gr[RD ? r : 0] = c_run;
        }
    } else {
        for (int i = threadIdx.x; i < a * BAND; i += blockDim.x) {
            const int t = i / BAND, r = i - t * BAND;
            const int row = base + r;
            us[t][r] = row < dv ? coef[t] * u[(((size_t)n * K + t) * HV + h) * dv + row] : 0.f;
        }
    }
    __syncthreads();
#pragma unroll
    for (int jr = 0; jr < kVerifyRows; ++jr) {
        const float gam =
            rowdec ? gr[RD ? (jr * kVerifyWarps + warp) * RPW + sub : 0] : coef[kVerifyMaxDrafts];
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

int device_sm_count() {
    int dev = 0, count = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        count < 1)
        count = 1;
    return count;
}

// The states of `items` heads as a [items][128][128] fp32 tensor, read in
// [128 rows x 32 columns] boxes with the 128-byte swizzle.
bool tc_state_map(CUtensorMap *tm, const float *state, int items) {
    if ((reinterpret_cast<uintptr_t>(state) & 15) != 0) return false;
    const uint64_t dims[3] = {128, 128, (uint64_t)items};
    const uint64_t strides[2] = {128 * sizeof(float), 128 * 128 * sizeof(float)};
    const uint32_t box[3] = {32, 128, 1};
    return encode_f32_map(tm, state, 3, dims, strides, box);
}

cudaError_t launch_verify_tc(const CUtensorMap &tm, const VerifyArgs &a, float *ws, int items,
                             cudaStream_t stream) {
    constexpr size_t smem = tc_smem_bytes();
    cudaError_t e = cudaFuncSetAttribute(verify_tc_kernel<false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int sms = device_sm_count();
    const unsigned grid = (unsigned)(items < sms ? items : sms);
    verify_tc_kernel<false><<<grid, kTcThreads, smem, stream>>>(
        tm, static_cast<const __nv_bfloat16 *>(a.v), ws, a.u, static_cast<__nv_bfloat16 *>(a.o),
        a.N, a.K, a.HV);
    return cudaGetLastError();
}

template <int DK, int KT, typename Tin, bool FUSED>
cudaError_t launch_verify_wy(const VerifyArgs &a, dim3 block, cudaStream_t stream) {
    auto setup = a.prologue ? verify_setup_kernel<DK, KT, Tin, true>
                            : verify_setup_kernel<DK, KT, Tin, false>;
    const int items = a.N * a.HV;
    constexpr int W = setup_warps<KT>();
    float *ws = static_cast<float *>(a.workspace);
    float *pend = FUSED ? ws + kWsHeaderFloats + (size_t)items * wy_item_floats(a.K, DK) : nullptr;
    cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(unsigned int), stream);
    if (e != cudaSuccess) return e;
    setup<<<(unsigned)((items + W - 1) / W), W * 32, 0, stream>>>(
        static_cast<const Tin *>(a.q), static_cast<const Tin *>(a.k), a.g, a.beta, ws, items, a.K,
        a.HK, a.HV, a.scale, a.prologue, static_cast<const Tin *>(a.prev_k), a.prev_g, a.accepted,
        pend, a.prev_K);
    auto kern = verify_wy_kernel<DK, KT, Tin, FUSED>;
    constexpr size_t smem = wy_smem_bytes<DK, KT, FUSED>();
    e = cudaGetLastError();   // the setup launch
    if (e != cudaSuccess) return e;
    if constexpr (DK == 128 && KT <= kTcDrafts && !FUSED &&
                  std::is_same<Tin, __nv_bfloat16>::value) {
        CUtensorMap tm;
        if (a.dv == 128 && (long long)a.N * a.HV < (1LL << 31) && tc_state_map(&tm, a.state, items))
            return launch_verify_tc(tm, a, ws, items, stream);
    }
    // per device and cheap: set on every launch (a process may drive several GPUs)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kVerifyWarps * 32, smem) !=
            cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    const long long bands = (long long)items * ((a.dv + verify_band<DK>() - 1) / verify_band<DK>());
    const long long slots = (long long)per_sm * device_sm_count();
    const unsigned grid = (unsigned)(bands < slots ? bands : slots);
    kern<<<grid, block, smem, stream>>>(static_cast<const Tin *>(a.v), const_cast<float *>(a.state),
                                        ws, a.u, static_cast<Tin *>(a.o), a.N, a.K, a.HV, a.dv,
                                        a.prev_u, a.prev_K);
    return cudaGetLastError();
}

template <int DK, typename Tin>
cudaError_t launch_verify_wy_k(const VerifyArgs &a, dim3 block, cudaStream_t stream) {
    const int kb = a.K > a.prev_K ? a.K : a.prev_K;   // bound for both rounds' drafts
    const bool fused = a.prev_K > 0;
    if (kb <= 4)
        return fused ? launch_verify_wy<DK, 4, Tin, true>(a, block, stream)
                     : launch_verify_wy<DK, 4, Tin, false>(a, block, stream);
    if (kb <= 8)
        return fused ? launch_verify_wy<DK, 8, Tin, true>(a, block, stream)
                     : launch_verify_wy<DK, 8, Tin, false>(a, block, stream);
    return fused ? launch_verify_wy<DK, 16, Tin, true>(a, block, stream)
                 : launch_verify_wy<DK, 16, Tin, false>(a, block, stream);
}

template <int DK, typename Tin>
void launch_verify_seq(const VerifyArgs &a, dim3 grid, dim3 block, cudaStream_t stream) {
    auto kern = (a.prologue & GDN_ROW_DECAY) ? verify_kernel<DK, Tin, true, true>
                : a.prologue                 ? verify_kernel<DK, Tin, true, false>
                                             : verify_kernel<DK, Tin, false, false>;
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
    if (a.states == nullptr && !(a.prologue & GDN_ROW_DECAY)) {
        // no per-draft states asked for: the state is never updated in registers
        // (with one decay per value row the mixed vectors would be per row: that
        // form runs on the per-draft kernel below, writing no states)
        switch (a.dk) {
            case 32: return launch_verify_wy_k<32, Tin>(a, block, stream);
            case 64: return launch_verify_wy_k<64, Tin>(a, block, stream);
            case 128: return launch_verify_wy_k<128, Tin>(a, block, stream);
            default: return cudaErrorInvalidValue;
        }
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

size_t verify_workspace_floats(int N, int K, int HV, int dk, int prev_K) {
    return kWsHeaderFloats + (size_t)N * HV * wy_item_floats(K, dk) +
           (prev_K > 0 ? (size_t)N * HV * pend_item_floats(prev_K, dk) : 0);
}

cudaError_t launch_verify(const VerifyArgs &a, cudaStream_t stream) {
    if (a.N == 0) return cudaSuccess;
    return a.dtype == GDN_BF16 ? launch_verify_typed<__nv_bfloat16>(a, stream)
                               : launch_verify_typed<float>(a, stream);
}

template <int DK, typename Tin>
void launch_commit_dk(const CommitDeltasArgs &a, dim3 grid, dim3 block, cudaStream_t stream) {
    auto kern = (a.prologue & GDN_ROW_DECAY) ? commit_deltas_kernel<DK, Tin, true, true>
                : a.prologue                 ? commit_deltas_kernel<DK, Tin, true, false>
                                             : commit_deltas_kernel<DK, Tin, false, false>;
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

// Test-only: the update-vector streaming kernel (d = 128, up to 4 drafts, bf16) whose
// first wait gives up at once; the workspace status word reads nonzero afterwards.
cudaError_t launch_verify_wy_timeout_test(const VerifyArgs &a, cudaStream_t stream) {
    auto kern = verify_wy_kernel<128, 4, __nv_bfloat16, false, true>;
    constexpr size_t smem = wy_smem_bytes<128, 4, false>();
    cudaError_t e = cudaMemsetAsync(a.workspace, 0, sizeof(unsigned int), stream);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long bands = (long long)a.N * a.HV * ((a.dv + verify_band<128>() - 1) / verify_band<128>());
    const unsigned grid = (unsigned)(bands < device_sm_count() ? bands : device_sm_count());
    kern<<<grid, kVerifyWarps * 32, smem, stream>>>(
        static_cast<const __nv_bfloat16 *>(a.v), const_cast<float *>(a.state),
        static_cast<float *>(a.workspace), a.u, static_cast<__nv_bfloat16 *>(a.o), a.N, a.K, a.HV,
        a.dv, nullptr, 0);
    return cudaGetLastError();
}

// Test-only: the tensor-core update-vector kernel (d = 128, up to 8 drafts, bf16)
// whose first wait gives up at once; the workspace status word reads nonzero
// afterwards.
cudaError_t launch_verify_tc_timeout_test(const VerifyArgs &a, cudaStream_t stream) {
    const long long heads = (long long)a.N * a.HV;
    if (heads >= (1LL << 31)) return cudaErrorInvalidValue;
    CUtensorMap tm;
    if (!tc_state_map(&tm, a.state, (int)heads)) return cudaErrorInvalidValue;
    constexpr size_t smem = tc_smem_bytes();
    cudaError_t e = cudaMemsetAsync(a.workspace, 0, sizeof(unsigned int), stream);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(verify_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    const int sms = device_sm_count();
    const unsigned grid = (unsigned)(heads < sms ? heads : sms);
    verify_tc_kernel<true><<<grid, kTcThreads, smem, stream>>>(
        tm, static_cast<const __nv_bfloat16 *>(a.v), static_cast<float *>(a.workspace), a.u,
        static_cast<__nv_bfloat16 *>(a.o), a.N, a.K, a.HV);
    return cudaGetLastError();
}

}  // namespace gdn
