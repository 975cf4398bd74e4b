// Chunkwise prefill of the gated delta rule on the tcgen05 tensor cores
// (bf16 q/k/v, head dim 128, chunk 64, fp32 state and accumulation).
//
// Rule: S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T, o_t = S_t q_t
// ("Qwen3-Next", sghael.github.io, section "Correcting a memory instead of
// adding to it": decay first, then correct along the current key; value head h
// reads query/key head h / (HV/HK); model card "Qwen3-Next-80B-A3B-Instruct",
// section "Model Overview": 32 V heads, 16 QK heads, head dim 128).
//
// Chunk form (C = 64 tokens, start state S0, G = chunk-local running sum of g,
// gamma = exp(G), L = valid rows of the chunk):
//   A_ij = b_i exp(G_i - G_j) k_i.k_j (j < i)      T = (I + A)^-1
//   P_ij = exp(G_i - G_j) q_i.k_j     (j <= i)
//   W = T diag(b gamma) K,  U~ = T diag(b) V        (state independent)
//   U = U~ - W S0^T                                  (sequential)
//   O = diag(gamma) Q S0^T + P U
//   S = gamma_L S0 + U^T diag(gamma_L / gamma) K
//
// Mapping onto tcgen05 (every product has M = 128 by working with transposes;
// i = value index, a = key index, t, s = token in chunk):
//   X  : D1[128x64]  = [Q;K] K^T            -> rows 0..63: Q K^T, 64..127: K K^T
//   Wt : DW[a][t]    = sum_s K[s][a] T'[t][s],  T' = T diag(b gamma)
//   Ut : DU[i][t]    = sum_s V[s][i] T''[t][s], T'' = T diag(b)
//   O1 : DQ[i][t]    = sum_a S0[i][a] q_t[a]
//   M1 : DU[i][t]   -= sum_a S0[i][a] W[t][a]   (negated A, accumulate)
//   M3 : DO[i][t]    = sum_s U[i][s] P[t][s]
//   M4 : DS[i][a]    = sum_s (U[i][s] gamma_L/gamma_s) K[s][a]
// with o_t = scale (gamma_t DQ[:, t] + DO[:, t]).
// and S(fp32, TMEM) = gamma_L S + DS.  q/k/v tiles arrive by TMA (128B
// swizzle); operands produced on chip are written by threads in the same
// swizzled layout.  One CTA per (sequence, value head) walks its chunks in
// order, prefetching the next chunk's tiles while it computes the current one.
// The UT inverse runs on CUDA cores (column-wise forward substitution).
//
// Precision: q, k, v are exact bf16 operands.  Operands produced on chip from
// fp32 values (T', T'', P, U and U diag(gamma_L/gamma)) are passed as a bf16
// pair hi + lo (hi = bf16(x), lo = bf16(x - hi)) and multiplied as hi*y + lo*y
// (plus the hi*lo cross term where both sides are split), which keeps ~16
// significant bits; the decay gamma_t of the inter-chunk read-out is applied in
// fp32 to a separate accumulator instead of being folded into a bf16 copy of q.
// Only S0 and W enter as single bf16 operands.
#include <cuda.h>

#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "tc_primitives.cuh"
#include "tma_host.h"

namespace gdn {
namespace {

using namespace tc;

constexpr int C = 64;      // chunk
constexpr int DH = 128;    // head dim (dk = dv)
constexpr int kThreads = 128;
constexpr uint32_t kWait = 1u << 22;   // polls before an on-device wait gives up

// shared memory layout (bytes from a 1024-aligned base)
constexpr uint32_t OFF_QK = 0;         // 2 stages x 32 KB: [atom0: Q | K][atom1: Q | K]
constexpr uint32_t QK_STAGE = 32768;
constexpr uint32_t OFF_V = 65536;      // 16 KB: [atom0][atom1], 64 rows each
constexpr uint32_t OFF_S = 81920;      // S0 bf16, 2 atom cols x 128 rows
constexpr uint32_t OFF_W = 114688;     // W as MN-major B: 128 rows (a) x 64 (t)
constexpr uint32_t OFF_P = 131072;     // P hi, P lo: 64 rows (t) x 64 (s) each
// One 64 KB region used twice per chunk: first by the UT inverse (A fp32,
// then T' and T'' as hi/lo tiles), later by U and U diag(gamma_L/gamma) (hi/lo).
constexpr uint32_t OFF_UNION = 147456;
constexpr uint32_t OFF_U = OFF_UNION;            // U hi, U lo     (2 x 16 KB)
constexpr uint32_t OFF_UB = OFF_UNION + 32768;   // Ub hi, Ub lo   (2 x 16 KB)
constexpr uint32_t OFF_A = OFF_UNION;            // A fp32 [64][65]
constexpr uint32_t A_LD = 65;
constexpr uint32_t OFF_TP = OFF_UNION + 17408;   // T' hi, T' lo   (2 x 8 KB)
constexpr uint32_t OFF_TPP = OFF_TP + 16384;     // T'' hi, T'' lo (2 x 8 KB)
constexpr uint32_t OFF_SMALL = OFF_UNION + 65536;  // G, gamma, beta, misc
constexpr uint32_t OFF_BAR = OFF_SMALL + 4 * 64 * 4;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 64 + 1024;   // + alignment slack
static_assert(OFF_A + 64 * A_LD * 4 <= OFF_TP, "A overlaps T tiles");
static_assert(OFF_TPP + 16384 <= OFF_SMALL, "T tiles overflow the union region");

// TMEM columns
constexpr uint32_t TM_D1 = 0;      // X, then W^T
constexpr uint32_t TM_U = 64;
constexpr uint32_t TM_O = 128;     // U P^T
constexpr uint32_t TM_Q = 192;     // S0 Q^T
constexpr uint32_t TM_DS = 256;
constexpr uint32_t TM_S = 384;

struct TcParams {
    const float *g, *beta, *h0;
    const int32_t *cu;
    int64_t T;
    int HK, HV;
    float scale;
    __nv_bfloat16 *o;
    float *hT;
    unsigned int *status;
};

__device__ __forceinline__ void ld_row64(uint32_t tmem, int warp, uint32_t col, float *v) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        float t[16];
        tmem_ld16(tmem_addr(tmem, warp, col + 16 * p), t);
#pragma unroll
        for (int j = 0; j < 16; ++j) v[16 * p + j] = t[j];
    }
    tmem_wait_ld();
}

// Row of 64 floats -> hi tile (bf16(x)) and lo tile (bf16(x - hi)), same row.
__device__ __forceinline__ void st_row64_hilo(uint32_t hi_base, uint32_t lo_base, uint32_t r,
                                              const float *f) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        float hi[8], lo[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            hi[e] = __bfloat162float(__float2bfloat16_rn(f[8 * c + e]));
            lo[e] = f[8 * c + e] - hi[e];
        }
        st_shared_bf16x8(hi_base + sw128_chunk(r, c), hi);
        st_shared_bf16x8(lo_base + sw128_chunk(r, c), lo);
    }
}

__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const TcParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    float *A_s = reinterpret_cast<float *>(sm + OFF_A);
    float *G_s = reinterpret_cast<float *>(sm + OFF_SMALL);
    float *gam_s = G_s + 64;
    float *beta_s = gam_s + 64;
    float *misc_s = beta_s + 64;
    uint64_t *bar_tma = reinterpret_cast<uint64_t *>(sm + OFF_BAR);  // [2]: q/k stages
    uint64_t *bar_v = bar_tma + 2;
    uint64_t *bar_mma = bar_tma + 3;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar_tma + 4);
    volatile int *abort_s = reinterpret_cast<volatile int *>(bar_tma + 5);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x, n = blockIdx.y;
    const int HV = p.HV;
    const int cqk = h / (HV / p.HK);
    int64_t bos, eos;
    if (p.cu) {
        bos = p.cu[n];
        eos = p.cu[n + 1];
    } else {
        bos = (int64_t)n * p.T;
        eos = bos + p.T;
    }
    const int nchunks = (int)((eos - bos + C - 1) / C);

    if (tid == 0) {
        mbar_init(&bar_tma[0], 1);
        mbar_init(&bar_tma[1], 1);
        mbar_init(bar_v, 1);
        mbar_init(bar_mma, 1);
        *abort_s = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (warp == 0) tmem_alloc(tslot, 512);
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;

    auto issue_tma_qk = [&](int c, int st) {
        const int s0 = (int)(bos + (int64_t)c * C);
        uint8_t *qk = sm + OFF_QK + st * QK_STAGE;
        mbar_arrive_expect_tx(&bar_tma[st], 4 * 8192);
        tma_load_3d(qk, &tm_q, &bar_tma[st], 0, cqk, s0);
        tma_load_3d(qk + 16384, &tm_q, &bar_tma[st], 64, cqk, s0);
        tma_load_3d(qk + 8192, &tm_k, &bar_tma[st], 0, cqk, s0);
        tma_load_3d(qk + 24576, &tm_k, &bar_tma[st], 64, cqk, s0);
    };
    auto issue_tma_v = [&](int c) {
        const int s0 = (int)(bos + (int64_t)c * C);
        mbar_arrive_expect_tx(bar_v, 2 * 8192);
        tma_load_3d(sm + OFF_V, &tm_v, bar_v, 0, h, s0);
        tma_load_3d(sm + OFF_V + 8192, &tm_v, bar_v, 64, h, s0);
    };

    // ---- start state: fp32 into TMEM, bf16 into the S0 operand tile ----
    const size_t sbase = ((size_t)n * HV + h) * (size_t)DH * DH;
    {
        const int i = tid;
#pragma unroll 1
        for (int q4 = 0; q4 < 8; ++q4) {
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
                v[j] = p.h0 ? p.h0[sbase + (size_t)i * DH + 16 * q4 + j] : 0.f;
            tmem_st16(tmem_addr(tmem, warp, TM_S + 16 * q4), v);
            const uint32_t atom = sb + OFF_S + (q4 >> 2) * 16384;
            const uint32_t c0 = (q4 & 3) * 2;
            st_shared_bf16x8(atom + sw128_chunk(i, c0), v);
            st_shared_bf16x8(atom + sw128_chunk(i, c0 + 1), v + 8);
        }
        tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && nchunks > 0) {
        issue_tma_qk(0, 0);
        issue_tma_v(0);
    }

    uint32_t mma_phase = 0;
    bool ok = true;
    auto wait_mma = [&]() {
        if (!mbar_wait(bar_mma, mma_phase, kWait)) ok = false;
        mma_phase ^= 1;
        tc_fence_after();
    };

    for (int c = 0; c < nchunks; ++c) {
        const int64_t s0 = bos + (int64_t)c * C;
        const int L = (int)((eos - s0) < C ? (eos - s0) : C);
        const int st = c & 1;
        const uint32_t qk = sb + OFF_QK + st * QK_STAGE;
        const uint32_t vt = sb + OFF_V;

        // ---- decay running sum and write strengths (rows >= L: g = 0, b = 0) ----
        float gv = 0.f, bv = 0.f;
        if (tid < C && tid < L) {
            gv = p.g[(s0 + tid) * HV + h];
            bv = p.beta[(s0 + tid) * HV + h];
        }
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, gv, off);
            if (lane >= off) gv += y;
        }
        if (tid == 31) misc_s[0] = gv;
        __syncthreads();
        if (tid >= 32 && tid < 64) gv += misc_s[0];
        if (tid < C) {
            G_s[tid] = gv;
            gam_s[tid] = expf(gv);
            beta_s[tid] = bv;
        }
        if (!mbar_wait(&bar_tma[st], (uint32_t)((c >> 1) & 1), kWait)) ok = false;
        if (!mbar_wait(bar_v, (uint32_t)(c & 1), kWait)) ok = false;
        if (!ok) *abort_s = 1;
        __syncthreads();
        if (*abort_s) break;
        if (tid == 0 && c + 1 < nchunks) issue_tma_qk(c + 1, st ^ 1);

        // ---- X: [Q;K] K^T ----
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
                mma_bf16(tmem + TM_D1, sdesc_sw128(qk + off, 16, 1024),
                         sdesc_sw128(qk + 8192 + off, 16, 1024), id, k > 0);
            }
            mma_commit(bar_mma);
        }
        __syncwarp();
        wait_mma();
        {
            float v[64];
            ld_row64(tmem, warp, TM_D1, v);
            if (tid < C) {  // P row i = tid
                const int i = tid;
                const float Gi = G_s[i];
#pragma unroll
                for (int j = 0; j < 64; ++j) v[j] = (j <= i) ? expf(Gi - G_s[j]) * v[j] : 0.f;
                st_row64_hilo(sb + OFF_P, sb + OFF_P + 8192, i, v);
            } else {  // A row i = tid - 64
                const int i = tid - C;
                const float Gi = G_s[i], bi = beta_s[i];
#pragma unroll
                for (int j = 0; j < 64; ++j)
                    A_s[i * A_LD + j] = (j < i) ? bi * expf(Gi - G_s[j]) * v[j] : 0.f;
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- UT inverse (threads 0..63, one column each) ----
        if (tid < C) {
            const int j = tid;
            float Tc[64];
#pragma unroll
            for (int i = 0; i < 64; ++i) {
                float acc = (i == j) ? 1.f : 0.f;
#pragma unroll
                for (int m = 0; m < i; ++m) acc = fmaf(-A_s[i * A_LD + m], Tc[m], acc);
                Tc[i] = acc;
            }
            const float bj = beta_s[j], bgj = bj * gam_s[j];
#pragma unroll
            for (int i = 0; i < 64; ++i) {
                const uint32_t off = sw128_offset(i, j);
                const float x1 = Tc[i] * bgj, x2 = Tc[i] * bj;
                const __nv_bfloat16 h1 = __float2bfloat16_rn(x1), h2 = __float2bfloat16_rn(x2);
                const __nv_bfloat16 l1 = __float2bfloat16_rn(x1 - __bfloat162float(h1));
                const __nv_bfloat16 l2 = __float2bfloat16_rn(x2 - __bfloat162float(h2));
                asm volatile("st.shared.b16 [%0], %1;" ::"r"(sb + OFF_TP + off),
                             "h"(*reinterpret_cast<const unsigned short *>(&h1)));
                asm volatile("st.shared.b16 [%0], %1;" ::"r"(sb + OFF_TP + 8192 + off),
                             "h"(*reinterpret_cast<const unsigned short *>(&l1)));
                asm volatile("st.shared.b16 [%0], %1;" ::"r"(sb + OFF_TPP + off),
                             "h"(*reinterpret_cast<const unsigned short *>(&h2)));
                asm volatile("st.shared.b16 [%0], %1;" ::"r"(sb + OFF_TPP + 8192 + off),
                             "h"(*reinterpret_cast<const unsigned short *>(&l2)));
            }
        }
        fence_proxy_async_smem();
        __syncthreads();

        // ---- W^T, U~^T (T', T'' as hi + lo), S0 Q^T ----
        if (tid == 0) {
            tc_fence_after();
            const uint32_t idw = idesc_bf16(128, 64, true, false);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint64_t ka = sdesc_sw128(qk + 8192 + k * 2048, 16384, 1024);
                const uint64_t va = sdesc_sw128(vt + k * 2048, 8192, 1024);
                mma_bf16(tmem + TM_D1, ka, sdesc_sw128(sb + OFF_TP + k * 32, 16, 1024), idw, k > 0);
                mma_bf16(tmem + TM_D1, ka, sdesc_sw128(sb + OFF_TP + 8192 + k * 32, 16, 1024), idw, 1);
                mma_bf16(tmem + TM_U, va, sdesc_sw128(sb + OFF_TPP + k * 32, 16, 1024), idw, k > 0);
                mma_bf16(tmem + TM_U, va, sdesc_sw128(sb + OFF_TPP + 8192 + k * 32, 16, 1024), idw, 1);
            }
            const uint32_t ido = idesc_bf16(128, 64, false, false);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
                mma_bf16(tmem + TM_Q, sdesc_sw128(sb + OFF_S + off, 16, 1024),
                         sdesc_sw128(qk + off, 16, 1024), ido, k > 0);
            }
            mma_commit(bar_mma);
        }
        __syncwarp();
        wait_mma();
        {
            float v[64];
            ld_row64(tmem, warp, TM_D1, v);  // W^T row a = tid
            st_row64_sw128(sb + OFF_W, tid, v);
        }
        if (tid == 0 && c + 1 < nchunks) issue_tma_v(c + 1);  // V tile consumed by U~
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- U = U~ - S0 W^T (accumulated onto U~ with A negated) ----
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, 64, false, true, true);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
                mma_bf16(tmem + TM_U, sdesc_sw128(sb + OFF_S + off, 16, 1024),
                         sdesc_sw128(sb + OFF_W + k * 2048, 8192, 1024), id, 1);
            }
            mma_commit(bar_mma);
        }
        __syncwarp();
        wait_mma();
        {
            float v[64];
            ld_row64(tmem, warp, TM_U, v);  // U^T row i = tid
#pragma unroll
            for (int t = 0; t < 64; ++t)
                if (t >= L) v[t] = 0.f;
            st_row64_hilo(sb + OFF_U, sb + OFF_U + 16384, tid, v);
            const float GL = G_s[63];
#pragma unroll
            for (int t = 0; t < 64; ++t) v[t] *= expf(GL - G_s[t]);
            st_row64_hilo(sb + OFF_UB, sb + OFF_UB + 16384, tid, v);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- DO = U P^T (hi/lo cross terms) ; DS = (U diag(gamma_L/gamma)) K ----
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id3 = idesc_bf16(128, 64, false, false);
            const uint32_t id4 = idesc_bf16(128, 128, false, true);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint64_t uh = sdesc_sw128(sb + OFF_U + k * 32, 16, 1024);
                const uint64_t ul = sdesc_sw128(sb + OFF_U + 16384 + k * 32, 16, 1024);
                const uint64_t ph = sdesc_sw128(sb + OFF_P + k * 32, 16, 1024);
                const uint64_t pl = sdesc_sw128(sb + OFF_P + 8192 + k * 32, 16, 1024);
                mma_bf16(tmem + TM_O, uh, ph, id3, k > 0);
                mma_bf16(tmem + TM_O, uh, pl, id3, 1);
                mma_bf16(tmem + TM_O, ul, ph, id3, 1);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint64_t kb = sdesc_sw128(qk + 8192 + k * 2048, 16384, 1024);
                mma_bf16(tmem + TM_DS, sdesc_sw128(sb + OFF_UB + k * 32, 16, 1024), kb, id4, k > 0);
                mma_bf16(tmem + TM_DS, sdesc_sw128(sb + OFF_UB + 16384 + k * 32, 16, 1024), kb, id4, 1);
            }
            mma_commit(bar_mma);
        }
        __syncwarp();
        wait_mma();
        {
            const int i = tid;
            float v[64];
            ld_row64(tmem, warp, TM_O, v);
            __nv_bfloat16 *orow = p.o + ((size_t)s0 * HV + h) * DH + i;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                float dq[16];
                tmem_ld16(tmem_addr(tmem, warp, TM_Q + 16 * q4), dq);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int t = 16 * q4 + j;
                    if (t < L)
                        orow[(size_t)t * HV * DH] =
                            __float2bfloat16_rn(p.scale * fmaf(gam_s[t], dq[j], v[t]));
                }
            }
            const float gL = gam_s[63];
#pragma unroll 1
            for (int q4 = 0; q4 < 8; ++q4) {
                float ds[16], s[16];
                tmem_ld16(tmem_addr(tmem, warp, TM_DS + 16 * q4), ds);
                tmem_ld16(tmem_addr(tmem, warp, TM_S + 16 * q4), s);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) s[j] = fmaf(gL, s[j], ds[j]);
                tmem_st16(tmem_addr(tmem, warp, TM_S + 16 * q4), s);
                const uint32_t atom = sb + OFF_S + (q4 >> 2) * 16384;
                const uint32_t c0 = (q4 & 3) * 2;
                st_shared_bf16x8(atom + sw128_chunk(i, c0), s);
                st_shared_bf16x8(atom + sw128_chunk(i, c0 + 1), s + 8);
            }
            tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
    }

    if (*abort_s || !ok) {
        if (tid == 0) atomicExch(p.status, (unsigned int)GDN_ERR_TIMEOUT);
        // let any copy or MMA still in flight land before TMEM is released
        if (tid == 0) {
            mbar_wait(bar_mma, mma_phase, kWait);
        }
    } else if (p.hT) {
        const int i = tid;
        float *dst = p.hT + sbase + (size_t)i * DH;
#pragma unroll 1
        for (int q4 = 0; q4 < 8; ++q4) {
            float s[16];
            tmem_ld16(tmem_addr(tmem, warp, TM_S + 16 * q4), s);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; j += 4)
                *reinterpret_cast<float4 *>(dst + 16 * q4 + j) =
                    make_float4(s[j], s[j + 1], s[j + 2], s[j + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace

bool prefill_tc_supported(int dk, int dv, int chunk, gdn_dtype dtype) {
    return dtype == GDN_BF16 && dk == DH && dv == DH && chunk == C;
}

size_t prefill_tc_workspace(int, int64_t, int, int, bool) { return 256; }

cudaError_t launch_prefill_tc(const PrefillArgs &a, cudaStream_t stream) {
    const int64_t Ttot = a.cu_seqlens ? a.T : (int64_t)a.N * a.T;
    if (Ttot >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    unsigned int *status = static_cast<unsigned int *>(a.workspace);
    cudaError_t err = cudaMemsetAsync(status, 0, sizeof(unsigned int), stream);
    if (err != cudaSuccess) return err;
    if (Ttot == 0 && a.hT == nullptr) return cudaSuccess;
    CUtensorMap tq, tk, tv;
    const uint64_t tok = (uint64_t)(Ttot > 0 ? Ttot : 1);
    uint64_t dq[3] = {(uint64_t)DH, (uint64_t)a.HK, tok};
    uint64_t sq[2] = {(uint64_t)DH * 2, (uint64_t)a.HK * DH * 2};
    uint64_t dv[3] = {(uint64_t)DH, (uint64_t)a.HV, tok};
    uint64_t sv[2] = {(uint64_t)DH * 2, (uint64_t)a.HV * DH * 2};
    uint32_t box[3] = {64, 1, 64};
    if (!encode_bf16_map(&tq, a.q, 3, dq, sq, box) || !encode_bf16_map(&tk, a.k, 3, dq, sq, box) ||
        !encode_bf16_map(&tv, a.v, 3, dv, sv, box))
        return cudaErrorInvalidValue;
    err = cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)SMEM_BYTES);
    if (err != cudaSuccess) return err;
    TcParams prm{a.g, a.beta, a.h0, a.cu_seqlens, a.T, a.HK, a.HV, a.scale,
                 static_cast<__nv_bfloat16 *>(a.o), a.hT, status};
    prefill_tc_kernel<<<dim3(a.HV, a.N), kThreads, SMEM_BYTES, stream>>>(tq, tk, tv, prm);
    return cudaGetLastError();
}

}  // namespace gdn
