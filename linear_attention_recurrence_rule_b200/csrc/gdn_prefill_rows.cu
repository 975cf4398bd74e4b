// Prefill with one decay per value row (GDN_ROW_DECAY: g is [..][HV][dv]) on CUDA
// cores, token by token.
//
// Under this rule row i of the state meets only what every row shares (k_t, q_t,
// b_t) and what is its own (v_t[i] and the decay a_t[i] = exp(g_t[i])):
//   s_i <- a_t[i] s_i,   u = b_t (v_t[i] - s_i.k_t),   s_i <- s_i + u k_t,
//   o_t[i] = scale * s_i.q_t
// (the decay-then-correct recurrence of "Qwen3-Next", sghael.github.io, section
// "Correcting a memory instead of adding to it", with row i's decay in place of
// the head's single one).  The rows never mix, so each state row is carried
// through the whole sequence by its own group of lanes: no chunk algebra, no
// exponentials of decay differences, and the result is the recurrence itself in
// fp32 for any decays (a chunkwise form would have to scale values by the inverse
// of a row's decay inside a chunk, which overflows fp32 once that decay passes
// e^-88).
//
// Work split: a CTA carries 32 state rows of one (sequence, value head) in 8
// warps; a warp carries 4 rows, 8 lanes per row, lane j of a row holding the
// state columns VE j + 8 VE m .. + VE - 1 (VE = the elements of one 16-byte
// piece of k: 8 bf16 or 4 fp32), so that the 8 lanes of a row read one 128-byte
// line of a shared-memory k or q row with one 16-byte load each: conflict-free,
// and the warp's 4 rows read the same line (a broadcast).  k and q stay in their
// input type in shared memory (half the load instructions for bf16); the L2
// norms of the prologue enter as per-token scalars on the reduced dots and the
// update's coefficients.  The tokens stream through shared memory in blocks of
// 32, double buffered: the next block's raw inputs are copied in by cp.async
// while the warps run the current one, then one pass over that block forms, once
// for the whole CTA, the prologue's scalars (1/|q|, 1/|k|, sigmoid gates), the
// decays exp(g), the betas and the products k_r.k_t, k_r.q_t of the tokens of
// each group of four.
//
// Four tokens per step: from s (the state before tokens 1..4 of a group), with
// A_t = a_1 ... a_t and R(t, r) = A_t / A_r = a_{r+1} ... a_t,
//   u_t = b_t (v_t - A_t s.k_t - sum_{r<t} R(t, r) u_r k_r.k_t)
//   o_t = A_t s.q_t + sum_{r<=t} R(t, r) u_r k_r.q_t
//   s  <- A_4 s + sum_r R(4, r) u_r k_r
// which is the recurrence unrolled four times (exact algebra, no divisions): the
// eight dot products s.k_t, s.q_t share one 8-lane reduction, so a group of four
// tokens costs one round of three shuffle levels instead of four.
#include <cuda_fp16.h>

#include <type_traits>

#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kRowsWarps = 8;
constexpr int kRowsThreads = kRowsWarps * 32;
constexpr int kRowsPerCta = 32;   // 8 warps x 4 rows
constexpr int kTB = 32;           // tokens per block: 8 groups of 4, one per warp in the pass
constexpr int kRowP = 36;         // pitch of the per-row tables (16-byte rows, 4 rows on 16 banks)

template <typename Tin, int DK>
struct RowsSmem {
    // raw block: k, q [kTB][DK], v [kTB][32] (Tin); g [kTB][32], beta [kTB] (fp32)
    static constexpr size_t raw_k = 0;
    static constexpr size_t raw_q = raw_k + (size_t)kTB * DK * sizeof(Tin);
    static constexpr size_t raw_v = raw_q + (size_t)kTB * DK * sizeof(Tin);
    static constexpr size_t raw_g = raw_v + (size_t)kTB * kRowsPerCta * sizeof(Tin);
    static constexpr size_t raw_b = raw_g + (size_t)kTB * kRowsPerCta * 4;
    static constexpr size_t raw_bytes = (raw_b + kTB * 4 + 127) & ~(size_t)127;
    // prepared block: decay and v per row [32][kRowP] (a row's tokens contiguous); per
    // group of four tokens the 16 products; per token beta, 1/|k|, 1/|q|
    static constexpr size_t rd_a = 2 * raw_bytes;
    static constexpr size_t rd_v = rd_a + (size_t)kRowsPerCta * kRowP * 4;
    static constexpr size_t rd_g = rd_v + (size_t)kRowsPerCta * kRowP * 4;
    static constexpr size_t rd_b = rd_g + (size_t)(kTB / 4) * 16 * 4;
    static constexpr size_t rd_rk = rd_b + (size_t)kTB * 4;
    static constexpr size_t rd_rq = rd_rk + (size_t)kTB * 4;
    static constexpr size_t out = rd_rq + (size_t)kTB * 4;   // outputs [kTB][32] fp32
    static constexpr size_t bytes = out + (size_t)kTB * kRowsPerCta * 4;
};

// elementwise product of two fp32 pairs (sm_100 packed multiply, each lane rounded
// as a scalar multiply)
__device__ __forceinline__ float2 mulf2(float2 a, float2 b) {
    unsigned long long ua, ub, ud;
    memcpy(&ua, &a, 8);
    memcpy(&ub, &b, 8);
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(ud) : "l"(ua), "l"(ub));
    float2 d;
    memcpy(&d, &ud, 8);
    return d;
}

// VE consecutive elements (one 8- or 16-byte shared-memory load) as fp32 pairs
template <typename Tin, int VE>
__device__ __forceinline__ void lds_pairs(const Tin *p, float2 (&f)[VE / 2]) {
    if constexpr (std::is_same<Tin, float>::value) {
        static_assert(VE == 4, "fp32 pieces are 4 elements");
        const float4 x = *reinterpret_cast<const float4 *>(p);
        f[0] = make_float2(x.x, x.y);
        f[1] = make_float2(x.z, x.w);
    } else if constexpr (VE == 8) {
        const uint4 u = *reinterpret_cast<const uint4 *>(p);
        f[0] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
        f[1] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
        f[2] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.z));
        f[3] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.w));
    } else {
        static_assert(VE == 4, "bf16 pieces are 4 or 8 elements");
        const uint2 u = *reinterpret_cast<const uint2 *>(p);
        f[0] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
        f[1] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
    }
}

__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

template <typename Tin, int DK>
__global__ void __launch_bounds__(kRowsThreads, 1)
prefill_rows_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                    const float *__restrict__ g, const float *__restrict__ beta,
                    const float *__restrict__ h0, const int32_t *__restrict__ cu, int64_t T, int HK,
                    int HV, int dv, float scale, Tin *__restrict__ o, float *__restrict__ hT,
                    unsigned pro, const void *__restrict__ gate) {
    using L_ = RowsSmem<Tin, DK>;
    // a lane's columns: NCH pieces of VE elements, VE j + 8 VE m (m < NCH)
    constexpr int VE = (16 / (int)sizeof(Tin)) < DK / 8 ? 16 / (int)sizeof(Tin) : DK / 8;
    constexpr int NCH = DK / (8 * VE);
    constexpr int NP = DK / 16;   // fp32 pairs of state per lane
    extern __shared__ __align__(128) uint8_t sm[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rg = lane >> 3, j = lane & 7;
    const int row = warp * 4 + rg;            // 0..31 within the CTA
    const int e0 = blockIdx.x * kRowsPerCta;  // first state row of the CTA
    const int h = blockIdx.y, n = blockIdx.z;
    const int cqk = h / (HV / HK);
    int64_t bos, eos;
    if (cu) {
        bos = cu[n];
        eos = cu[n + 1];
    } else {
        bos = (int64_t)n * T;
        eos = bos + T;
    }
    const bool logits = (pro & GDN_PROLOGUE_GATE_LOGITS) != 0;
    const bool nq = (pro & GDN_PROLOGUE_NORM_Q) != 0, nk = (pro & GDN_PROLOGUE_NORM_K) != 0;

    // ---- state row (this lane's columns) ----
    const size_t srow = (((size_t)n * HV + h) * dv + e0 + row) * DK;
    float2 s[NP];
#pragma unroll
    for (int m = 0; m < NCH; ++m)
#pragma unroll
        for (int e = 0; e < VE / 4; ++e) {
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (h0) x = *reinterpret_cast<const float4 *>(h0 + srow + 8 * VE * m + VE * j + 4 * e);
            s[m * VE / 2 + 2 * e] = make_float2(x.x, x.y);
            s[m * VE / 2 + 2 * e + 1] = make_float2(x.z, x.w);
        }

    // ---- raw block starting at token t0 into buffer buf by cp.async (tokens past
    //      the end are not read; prepare() zeroes their k and q rows) ----
    auto issue = [&](int64_t t0, int buf) {
        uint8_t *rb = sm + buf * L_::raw_bytes;
        const int L = (int)((eos - t0) < kTB ? (eos - t0) : kTB);
        constexpr int KCH = DK * (int)sizeof(Tin) / 16;   // 16-byte pieces of a k or q row
        for (int idx = tid; idx < 2 * kTB * KCH; idx += kRowsThreads) {
            const int which = idx / (kTB * KCH), r = idx - which * kTB * KCH;
            const int t = r / KCH, pc = r - t * KCH;
            if (t < L) {
                const Tin *src = (which ? q : k) + ((t0 + t) * HK + cqk) * DK;
                cp_async16(rb + (which ? L_::raw_q : L_::raw_k) + ((size_t)t * KCH + pc) * 16,
                           reinterpret_cast<const uint8_t *>(src) + pc * 16);
            }
        }
        constexpr int VCH = kRowsPerCta * (int)sizeof(Tin) / 16;   // 16-byte pieces of v
        constexpr int GCH = kRowsPerCta * 4 / 16;
        for (int idx = tid; idx < kTB * (VCH + GCH); idx += kRowsThreads) {
            const int t = idx / (VCH + GCH), pc = idx - t * (VCH + GCH);
            if (t < L) {
                const size_t base = ((size_t)(t0 + t) * HV + h) * dv + e0;
                if (pc < VCH)
                    cp_async16(rb + L_::raw_v + ((size_t)t * VCH + pc) * 16,
                               reinterpret_cast<const uint8_t *>(v + base) + pc * 16);
                else
                    cp_async16(rb + L_::raw_g + ((size_t)t * GCH + pc - VCH) * 16,
                               reinterpret_cast<const uint8_t *>(g + base) + (pc - VCH) * 16);
            }
        }
        if (tid < L) cp_async4(rb + L_::raw_b + tid * 4, beta + (t0 + tid) * HV + h);
        cp_async_commit();
    };

    // ---- the prepared block: the scalars of the prologue, decays, values, products ----
    float *RK = reinterpret_cast<float *>(sm + L_::rd_rk);  // [token] 1/|k| (1 without the norm)
    float *RQ = reinterpret_cast<float *>(sm + L_::rd_rq);  // [token] 1/|q|
    float *Af = reinterpret_cast<float *>(sm + L_::rd_a);   // [row][kRowP] decays
    float *Vf = reinterpret_cast<float *>(sm + L_::rd_v);   // [row][kRowP] values
    float *Gp = reinterpret_cast<float *>(sm + L_::rd_g);   // [group][16] products
    float *Bt = reinterpret_cast<float *>(sm + L_::rd_b);   // [token] betas
    float *Os = reinterpret_cast<float *>(sm + L_::out);
    // Products of group w (tokens 4w + 1..4 numbered 1..4), in the order the step reads:
    //   kk12 kk13 kk23 kk14 kk24 kk34 | kq11 kq12 kq22 kq13 kq23 kq33 kq14 kq24 kq34 kq44
    // Tokens past the end of the sequence come out as k = q = 0, b = 0, a = 1, v = 0:
    // the step leaves the state unchanged through them.
    auto prepare = [&](int L, int buf) {
        uint8_t *rb = sm + buf * L_::raw_bytes;
        Tin *Kr = reinterpret_cast<Tin *>(rb + L_::raw_k);
        Tin *Qr = reinterpret_cast<Tin *>(rb + L_::raw_q);
        {
            constexpr int E = DK / 32;
            const int tb = 4 * warp;
            float kx[4][E], qx[4][E];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const bool ok = tb + r < L;
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    kx[r][e] = ok ? to_f32(Kr[(tb + r) * DK + 32 * e + lane]) : 0.f;
                    qx[r][e] = ok ? to_f32(Qr[(tb + r) * DK + 32 * e + lane]) : 0.f;
                }
            }
            // partial sums: |k_r|^2, |q_r|^2, then the 16 products in the order above
            float p[24];
#pragma unroll
            for (int i = 0; i < 24; ++i) p[i] = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) {
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    p[r] = fmaf(kx[r][e], kx[r][e], p[r]);
                    p[4 + r] = fmaf(qx[r][e], qx[r][e], p[4 + r]);
                }
                p[8] = fmaf(kx[0][e], kx[1][e], p[8]);
                p[9] = fmaf(kx[0][e], kx[2][e], p[9]);
                p[10] = fmaf(kx[1][e], kx[2][e], p[10]);
                p[11] = fmaf(kx[0][e], kx[3][e], p[11]);
                p[12] = fmaf(kx[1][e], kx[3][e], p[12]);
                p[13] = fmaf(kx[2][e], kx[3][e], p[13]);
                p[14] = fmaf(kx[0][e], qx[0][e], p[14]);
                p[15] = fmaf(kx[0][e], qx[1][e], p[15]);
                p[16] = fmaf(kx[1][e], qx[1][e], p[16]);
                p[17] = fmaf(kx[0][e], qx[2][e], p[17]);
                p[18] = fmaf(kx[1][e], qx[2][e], p[18]);
                p[19] = fmaf(kx[2][e], qx[2][e], p[19]);
                p[20] = fmaf(kx[0][e], qx[3][e], p[20]);
                p[21] = fmaf(kx[1][e], qx[3][e], p[21]);
                p[22] = fmaf(kx[2][e], qx[3][e], p[22]);
                p[23] = fmaf(kx[3][e], qx[3][e], p[23]);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
#pragma unroll
                for (int i = 0; i < 24; ++i) p[i] += __shfl_xor_sync(0xffffffffu, p[i], off);
            float rk[4], rq[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                rk[r] = nk ? inv_l2norm(p[r]) : 1.f;
                rq[r] = nq ? inv_l2norm(p[4 + r]) : 1.f;
                if (tb + r >= L) {
                    // past the end: zero rows, so that the step reads finite values
#pragma unroll
                    for (int e = 0; e < E; ++e) {
                        Kr[(tb + r) * DK + 32 * e + lane] = from_f32<Tin>(0.f);
                        Qr[(tb + r) * DK + 32 * e + lane] = from_f32<Tin>(0.f);
                    }
                }
            }
            if (lane < 16) {
                // product i of the list (lane i), normalised: its k-side token kr and
                // its other token kt (a k for i < 6, a q after)
                constexpr int kr_[16] = {0, 0, 1, 0, 1, 2, 0, 0, 1, 0, 1, 2, 0, 1, 2, 3};
                constexpr int kt_[16] = {1, 2, 2, 3, 3, 3, 0, 1, 1, 2, 2, 2, 3, 3, 3, 3};
                float pv = 0.f;
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    if (i == lane) pv = p[8 + i] * rk[kr_[i]] * (i < 6 ? rk[kt_[i]] : rq[kt_[i]]);
                Gp[warp * 16 + lane] = pv;
            } else if (lane < 20) {
                const int r = lane - 16, t = tb + r;
                const float b = t < L ? reinterpret_cast<const float *>(rb + L_::raw_b)[t] : 0.f;
                Bt[t] = (logits && t < L) ? gate_sigmoid(b) : b;
                float rkt = rk[0], rqt = rq[0];
#pragma unroll
                for (int i = 1; i < 4; ++i)
                    if (i == r) {
                        rkt = rk[i];
                        rqt = rq[i];
                    }
                RK[t] = rkt;
                RQ[t] = rqt;
            }
        }
        const Tin *Vr = reinterpret_cast<const Tin *>(rb + L_::raw_v);
        const float *Gr = reinterpret_cast<const float *>(rb + L_::raw_g);
        for (int idx = tid; idx < kTB * kRowsPerCta; idx += kRowsThreads) {
            const int t = idx / kRowsPerCta, r = idx - t * kRowsPerCta;
            float a = 1.f, vv = 0.f;
            if (t < L) {
                const float gv = Gr[idx];
                a = expf(logits ? gate_log_sigmoid(gv) : gv);
                vv = to_f32(Vr[idx]);
            }
            Af[r * kRowP + t] = a;
            Vf[r * kRowP + t] = vv;
        }
    };

    auto write_out = [&](int64_t t0, int L) {
        for (int idx = tid; idx < L * kRowsPerCta; idx += kRowsThreads) {
            const int t = idx / kRowsPerCta, r = idx - t * kRowsPerCta;
            const size_t oi = ((size_t)(t0 + t) * HV + h) * dv + e0 + r;
            float out = Os[idx];
            if (gate)   // output gate before the one rounding: fp32 factors for fp32, else fp16
                out *= std::is_same<Tin, float>::value ? static_cast<const float *>(gate)[oi]
                                                       : __half2float(static_cast<const __half *>(gate)[oi]);
            o[oi] = from_f32<Tin>(out);
        }
    };

    int buf = 0;
    if (bos < eos) {
        issue(bos, 0);
        cp_async_wait_all();
        __syncthreads();
        prepare((int)((eos - bos) < kTB ? (eos - bos) : kTB), 0);
        __syncthreads();
    }
    for (int64_t t0 = bos; t0 < eos; t0 += kTB) {
        const int L = (int)((eos - t0) < kTB ? (eos - t0) : kTB);
        const int64_t t1 = t0 + kTB;
        if (t1 < eos) issue(t1, buf ^ 1);
        // ---- the recurrence over this block's tokens, four at a time ----
        const Tin *kb = reinterpret_cast<const Tin *>(sm + buf * L_::raw_bytes + L_::raw_k) + VE * j;
        const Tin *qb = reinterpret_cast<const Tin *>(sm + buf * L_::raw_bytes + L_::raw_q) + VE * j;
        for (int tg = 0; tg < L; tg += 4) {
            // s.k_t and s.q_t for the group's four tokens (this lane's columns)
            float2 pk[4], pq[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) pk[r] = pq[r] = make_float2(0.f, 0.f);
#pragma unroll
            for (int m = 0; m < NCH; ++m) {
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    float2 kf[VE / 2], qf[VE / 2];
                    lds_pairs<Tin, VE>(kb + (tg + r) * DK + 8 * VE * m, kf);
                    lds_pairs<Tin, VE>(qb + (tg + r) * DK + 8 * VE * m, qf);
#pragma unroll
                    for (int e = 0; e < VE / 2; ++e) {
                        pk[r] = fma2(s[m * VE / 2 + e], kf[e], pk[r]);
                        pq[r] = fma2(s[m * VE / 2 + e], qf[e], pq[r]);
                    }
                }
            }
            float sk[4], sq[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                sk[r] = pk[r].x + pk[r].y;
                sq[r] = pq[r].x + pq[r].y;
            }
#pragma unroll
            for (int off = 1; off < 8; off <<= 1)
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    sk[r] += __shfl_xor_sync(0xffffffffu, sk[r], off);
                    sq[r] += __shfl_xor_sync(0xffffffffu, sq[r], off);
                }
            // the norms of the prologue: s.k^ = (s.k) / |k|, s.q^ = (s.q) / |q|
            const float4 rkv = *reinterpret_cast<const float4 *>(RK + tg);
            const float4 rqv = *reinterpret_cast<const float4 *>(RQ + tg);
            sk[0] *= rkv.x;
            sk[1] *= rkv.y;
            sk[2] *= rkv.z;
            sk[3] *= rkv.w;
            sq[0] *= rqv.x;
            sq[1] *= rqv.y;
            sq[2] *= rqv.z;
            sq[3] *= rqv.w;
            const float4 av = *reinterpret_cast<const float4 *>(Af + row * kRowP + tg);
            const float4 vv = *reinterpret_cast<const float4 *>(Vf + row * kRowP + tg);
            const float4 bt = *reinterpret_cast<const float4 *>(Bt + tg);
            const float4 g0 = *reinterpret_cast<const float4 *>(Gp + tg * 4);
            const float4 g1 = *reinterpret_cast<const float4 *>(Gp + tg * 4 + 4);
            const float4 g2 = *reinterpret_cast<const float4 *>(Gp + tg * 4 + 8);
            const float4 g3 = *reinterpret_cast<const float4 *>(Gp + tg * 4 + 12);
            // g0 = kk12 kk13 kk23 kk14, g1 = kk24 kk34 kq11 kq12, g2 = kq22 kq13 kq23 kq33,
            // g3 = kq14 kq24 kq34 kq44
            const float A1 = av.x, A2 = A1 * av.y, A3 = A2 * av.z, A4 = A3 * av.w;
            const float R32 = av.z, R43 = av.w, R31 = av.y * av.z, R42 = av.z * av.w,
                        R41 = av.y * R42;
            const float u1 = bt.x * fmaf(-A1, sk[0], vv.x);
            const float u2 = bt.y * (fmaf(-A2, sk[1], vv.y) - av.y * u1 * g0.x);
            const float u3 = bt.z * (fmaf(-A3, sk[2], vv.z) - R31 * u1 * g0.y - R32 * u2 * g0.z);
            const float u4 = bt.w * (fmaf(-A4, sk[3], vv.w) - R41 * u1 * g0.w - R42 * u2 * g1.x -
                                     R43 * u3 * g1.y);
            if (j == 0) {
                float *os = Os + tg * kRowsPerCta + row;
                os[0] = scale * fmaf(A1, sq[0], u1 * g1.z);
                os[kRowsPerCta] = scale * (fmaf(A2, sq[1], av.y * u1 * g1.w) + u2 * g2.x);
                os[2 * kRowsPerCta] =
                    scale * (fmaf(A3, sq[2], R31 * u1 * g2.y) + R32 * u2 * g2.z + u3 * g2.w);
                os[3 * kRowsPerCta] = scale * (fmaf(A4, sq[3], R41 * u1 * g3.x) + R42 * u2 * g3.y +
                                               R43 * u3 * g3.z + u4 * g3.w);
            }
            // s <- A4 s + R41 u1 k^1 + R42 u2 k^2 + R43 u3 k^3 + u4 k^4 (k^ = k / |k|)
            float2 cc[4];
            cc[0] = make_float2(R41 * u1 * rkv.x, R41 * u1 * rkv.x);
            cc[1] = make_float2(R42 * u2 * rkv.y, R42 * u2 * rkv.y);
            cc[2] = make_float2(R43 * u3 * rkv.z, R43 * u3 * rkv.z);
            cc[3] = make_float2(u4 * rkv.w, u4 * rkv.w);
            const float2 a4 = make_float2(A4, A4);
#pragma unroll
            for (int m = 0; m < NCH; ++m) {
                float2 acc[VE / 2];
#pragma unroll
                for (int e = 0; e < VE / 2; ++e) acc[e] = mulf2(a4, s[m * VE / 2 + e]);
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    float2 kf[VE / 2];
                    lds_pairs<Tin, VE>(kb + (tg + r) * DK + 8 * VE * m, kf);
#pragma unroll
                    for (int e = 0; e < VE / 2; ++e) acc[e] = fma2(cc[r], kf[e], acc[e]);
                }
#pragma unroll
                for (int e = 0; e < VE / 2; ++e) s[m * VE / 2 + e] = acc[e];
            }
        }
        cp_async_wait_all();
        __syncthreads();
        write_out(t0, L);
        if (t1 < eos) prepare((int)((eos - t1) < kTB ? (eos - t1) : kTB), buf ^ 1);
        __syncthreads();
        buf ^= 1;
    }
    if (hT) {
#pragma unroll
        for (int m = 0; m < NCH; ++m)
#pragma unroll
            for (int e = 0; e < VE / 4; ++e) {
                const float2 a = s[m * VE / 2 + 2 * e], b = s[m * VE / 2 + 2 * e + 1];
                *reinterpret_cast<float4 *>(hT + srow + 8 * VE * m + VE * j + 4 * e) =
                    make_float4(a.x, a.y, b.x, b.y);
            }
    }
}

template <typename Tin, int DK>
cudaError_t launch_rows_typed(const PrefillArgs &a, cudaStream_t stream) {
    constexpr size_t smem = RowsSmem<Tin, DK>::bytes;
    auto kern = prefill_rows_kernel<Tin, DK>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    const dim3 grid(a.dv / kRowsPerCta, a.HV, a.N), block(kRowsThreads);
    kern<<<grid, block, smem, stream>>>(
        static_cast<const Tin *>(a.q), static_cast<const Tin *>(a.k), static_cast<const Tin *>(a.v), a.g,
        a.beta, a.h0, a.cu_seqlens, a.T, a.HK, a.HV, a.dv, a.scale, static_cast<Tin *>(a.o), a.hT,
        a.prologue, a.gate);
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_rows_dk(const PrefillArgs &a, cudaStream_t stream) {
    switch (a.dk) {
        case 32: return launch_rows_typed<Tin, 32>(a, stream);
        case 64: return launch_rows_typed<Tin, 64>(a, stream);
        case 128: return launch_rows_typed<Tin, 128>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool prefill_rows_supported(int dk, int dv) {
    return (dk == 32 || dk == 64 || dk == 128) && (dv == 32 || dv == 64 || dv == 128);
}

cudaError_t launch_prefill_rows(const PrefillArgs &a, cudaStream_t stream) {
    if (a.N == 0) return cudaSuccess;
    return a.dtype == GDN_BF16 ? launch_rows_dk<__nv_bfloat16>(a, stream) : launch_rows_dk<float>(a, stream);
}

}  // namespace gdn
