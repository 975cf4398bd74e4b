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
//   M1 : DU[i][t]   -= sum_a S0[i][a] W[t][a]   (negated A, accumulate)
//   O1 : DQ[i][t]    = sum_a S0[i][a] q_t[a]
//   M4 : S[i][a]    += sum_s (U[i][s] gamma_L/gamma_s) K[s][a]   (U from TMEM)
//   M3 : DO[i][t]    = sum_s U[i][s] P[t][s]                     (U from TMEM)
// with o_t = scale (gamma_t DQ[:, t] + DO[:, t]).  The fp32 state S lives in
// tensor memory; before M4 of a chunk it is scaled in place by gamma_L, so M4
// accumulates the chunk's update straight into it.
//
// Work split: one CTA per (sequence, value head); its warps specialise and
// run the state-independent preparation of chunk c+1 while the sequential
// chain processes chunk c:
//   warp 0        TMA producer: q/k tiles (2-stage ring) and the v tile
//   warp 1        MMA issuer: the warp computes descriptors, one elected lane
//                 issues every MMA and commit, in dependency order
//   warps 2..9    chain: U (hi/lo into TMEM), the bf16 copy of S for the
//                 next chunk, the gamma_L scaling of S, outputs
//   warps 10..17  prep: A and P from [Q;K]K^T, the UT inverse T (blocked
//                 16 -> 32 -> 64 on CUDA cores), T', T'' tiles, W
// Two warps share each TMEM lane quadrant, each taking half of a row's columns.
// Stages hand over through mbarriers; every wait is bounded and a timeout
// winds the CTA down and reports GDN_ERR_TIMEOUT in the workspace status word.
//
// Precision: q, k, v are exact bf16 operands.  Operands produced on chip from
// fp32 values (T', T'', P, U and U diag(gamma_L/gamma)) are passed as a bf16
// pair hi + lo (hi = bf16(x), lo = bf16(x - hi)) and multiplied as hi*y + lo*y
// (plus the hi*lo cross term where both sides are split), which keeps ~16
// significant bits; the decay gamma_t of the inter-chunk read-out is applied in
// fp32 to a separate accumulator.  Only S0 and W enter as single bf16 operands.
#include <cuda.h>

#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "gdn_tc_common.cuh"
#include "tc_primitives.cuh"
#include "tma_host.h"

namespace gdn {
namespace {

using namespace tc;
using namespace tcc;

constexpr int C = 64;      // chunk
constexpr int DH = 128;    // head dim (dk = dv)
constexpr int kTmaWarp = 0, kMmaWarp = 1, kChainWarp0 = 2, kNumChainWarps = 8;
constexpr int kPrepWarp0 = kChainWarp0 + kNumChainWarps, kNumPrepWarps = 8;
constexpr int kThreads = 32 * (kPrepWarp0 + kNumPrepWarps);
constexpr int kPrepThreads = 32 * kNumPrepWarps;
constexpr uint32_t kWait = 2000;      // sleeping polls (<= ~1 ms each) before a wait gives up

// ---- shared memory layout (bytes from a 1024-aligned base) ----
constexpr uint32_t OFF_QK = 0;         // 2 stages x 32 KB: [atom0: Q | K][atom1: Q | K]
constexpr uint32_t QK_STAGE = 32768;
constexpr uint32_t OFF_V = 65536;      // 16 KB: [atom0][atom1], 64 rows each
constexpr uint32_t OFF_S = 81920;      // S0 bf16, 2 atom cols x 128 rows
constexpr uint32_t OFF_W = 114688;     // W as MN-major B: 128 rows (a) x 64 (t)
constexpr uint32_t OFF_P = 131072;     // 2 buffers x (P hi, P lo): 64 rows (t) x 64 (s)
constexpr uint32_t P_BUF = 16384;
constexpr uint32_t OFF_T = 163840;     // T' hi, T' lo, T'' hi, T'' lo (4 x 8 KB);
constexpr uint32_t OFF_A = OFF_T;      //   A fp32 [64][A_LD] shares it (dead before T' is written)
constexpr uint32_t A_LD = 68;
constexpr uint32_t OFF_TF = 196608;    // T fp32 [64][T_LD]
constexpr uint32_t T_LD = 68;
constexpr uint32_t OFF_X = OFF_TF + 64 * T_LD * 4;   // inverse scratch: 32 x X_LD fp32
constexpr uint32_t X_LD = 36;
constexpr uint32_t OFF_PB = OFF_X + 32 * X_LD * 4;   // prep: beta, gamma, G (3 x 64)
constexpr uint32_t OFF_CG = OFF_PB + 3 * 64 * 4;     // per chain warp: G, gamma (2 x 64)
constexpr uint32_t OFF_BAR = OFF_CG + kNumChainWarps * 128 * 4 + 64;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;  // + alignment slack
static_assert(OFF_A + 64 * A_LD * 4 <= OFF_T + 32768, "A overflows the T tiles");
static_assert(OFF_T + 32768 <= OFF_TF, "T tiles overlap T fp32");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// ---- TMEM columns ----
constexpr uint32_t TM_D1 = 0;      // X, then W^T
constexpr uint32_t TM_U = 64;      // U~, then U
constexpr uint32_t TM_Q = 128;     // S0 Q^T
constexpr uint32_t TM_O = 192;     // U P^T
constexpr uint32_t TM_S = 256;     // fp32 state (128 columns)
constexpr uint32_t TM_UH = 384, TM_UL = 416, TM_BH = 448, TM_BL = 480;  // bf16 A operands

// ---- mbarriers ----
enum Bar {
    B_QK_FULL0, B_QK_FULL1, B_QK_FREE0, B_QK_FREE1, B_V_FULL, B_V_FREE,
    B_X_FULL, B_T_FULL, B_WU_FULL, B_W_FULL, B_S0_FULL, B_U_MMA, B_U_FULL,
    B_DS_FULL, B_O_FULL, B_Q_FREE, B_P_FREE0, B_P_FREE1, B_COUNT
};

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

struct Ctx {
    uint64_t *bars;
    volatile int *abort_flag;
    unsigned int *status;
};

// Bounded wait; on timeout (or if another role already gave up) raises the
// CTA-wide abort flag and returns false.
__device__ __forceinline__ bool wait_bar(const Ctx &x, int b, uint32_t parity) {
    for (uint32_t i = 0; i < kWait; ++i) {
        if (mbar_try_wait_sleep(&x.bars[b], parity, 1000000u)) return true;
        if (*x.abort_flag) return false;
    }
    *x.abort_flag = 1;
    atomicExch(x.status, (unsigned int)GDN_ERR_TIMEOUT);
    return false;
}
__device__ __forceinline__ void arrive(const Ctx &x, int b) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&x.bars[b])) : "memory");
}
__device__ __forceinline__ void prep_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kPrepThreads) : "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const TcParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + B_COUNT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + B_COUNT + 1);
    const Ctx x{bars, abort_flag, p.status};

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
    const size_t sbase = ((size_t)n * HV + h) * (size_t)DH * DH;
    auto chunk_len = [&](int c) {
        const int64_t r = eos - (bos + (int64_t)c * C);
        return (int)(r < C ? r : C);
    };

    if (tid == 0) {
        for (int b = 0; b < B_COUNT; ++b) {
            uint32_t cnt = 1;
            if (b == B_T_FULL || b == B_W_FULL) cnt = kNumPrepWarps;
            if (b == B_S0_FULL || b == B_U_FULL || b == B_Q_FREE) cnt = kNumChainWarps;
            mbar_init(&bars[b], cnt);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(tslot, 512);
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;

    if (warp == kTmaWarp) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && nchunks > 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            for (int c = 0; c < nchunks; ++c) {
                const int st = c & 1;
                const int s0 = (int)(bos + (int64_t)c * C);
                if (c >= 2 && !wait_bar(x, B_QK_FREE0 + st, (uint32_t)(((c >> 1) - 1) & 1))) break;
                uint8_t *qk = sm + OFF_QK + st * QK_STAGE;
                mbar_arrive_expect_tx(&bars[B_QK_FULL0 + st], 4 * 8192);
                tma_load_3d(qk, &tm_q, &bars[B_QK_FULL0 + st], 0, cqk, s0);
                tma_load_3d(qk + 16384, &tm_q, &bars[B_QK_FULL0 + st], 64, cqk, s0);
                tma_load_3d(qk + 8192, &tm_k, &bars[B_QK_FULL0 + st], 0, cqk, s0);
                tma_load_3d(qk + 24576, &tm_k, &bars[B_QK_FULL0 + st], 64, cqk, s0);
                if (c >= 1 && !wait_bar(x, B_V_FREE, (uint32_t)((c - 1) & 1))) break;
                mbar_arrive_expect_tx(&bars[B_V_FULL], 2 * 8192);
                tma_load_3d(sm + OFF_V, &tm_v, &bars[B_V_FULL], 0, h, s0);
                tma_load_3d(sm + OFF_V + 8192, &tm_v, &bars[B_V_FULL], 64, h, s0);
            }
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (nchunks > 0) {
            const uint32_t id_x = idesc_bf16(128, 64, false, false);
            const uint32_t id_w = idesc_bf16(128, 64, true, false);
            const uint32_t id_m1 = idesc_bf16(128, 64, false, true, true);
            const uint32_t id_m4 = idesc_bf16(128, 128, false, true);
            auto commit = [&](int b) {
                if (elect_one()) mma_commit(&bars[b]);
                __syncwarp();
            };
            auto issue_x = [&](int c) {
                const uint32_t qk = sb + OFF_QK + (c & 1) * QK_STAGE;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
                    const uint64_t a = sdesc_sw128(qk + off, 16, 1024);
                    const uint64_t b = sdesc_sw128(qk + 8192 + off, 16, 1024);
                    if (elect_one()) mma_bf16(tmem + TM_D1, a, b, id_x, k > 0);
                    __syncwarp();
                }
                commit(B_X_FULL);
            };
            auto issue_wu = [&](int c) {
                const uint32_t qk = sb + OFF_QK + (c & 1) * QK_STAGE;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint64_t ka = sdesc_sw128(qk + 8192 + k * 2048, 16384, 1024);
                    const uint64_t va = sdesc_sw128(sb + OFF_V + k * 2048, 8192, 1024);
                    const uint64_t t1h = sdesc_sw128(sb + OFF_T + k * 32, 16, 1024);
                    const uint64_t t1l = sdesc_sw128(sb + OFF_T + 8192 + k * 32, 16, 1024);
                    const uint64_t t2h = sdesc_sw128(sb + OFF_T + 16384 + k * 32, 16, 1024);
                    const uint64_t t2l = sdesc_sw128(sb + OFF_T + 24576 + k * 32, 16, 1024);
                    if (elect_one()) {
                        mma_bf16(tmem + TM_D1, ka, t1h, id_w, k > 0);
                        mma_bf16(tmem + TM_D1, ka, t1l, id_w, 1);
                        mma_bf16(tmem + TM_U, va, t2h, id_w, k > 0);
                        mma_bf16(tmem + TM_U, va, t2l, id_w, 1);
                    }
                    __syncwarp();
                }
                commit(B_WU_FULL);
                commit(B_V_FREE);
            };
            bool ok = wait_bar(x, B_QK_FULL0, 0);
            if (ok) {
                tc_fence_after();
                issue_x(0);
                ok = wait_bar(x, B_T_FULL, 0) && wait_bar(x, B_V_FULL, 0);
            }
            if (ok) {
                tc_fence_after();
                issue_wu(0);
            }
            for (int c = 0; ok && c < nchunks; ++c) {
                const uint32_t ph = (uint32_t)(c & 1);
                const uint32_t qk = sb + OFF_QK + (c & 1) * QK_STAGE;
                if (!wait_bar(x, B_W_FULL, ph) || !wait_bar(x, B_S0_FULL, ph)) break;
                if (c >= 1 && !wait_bar(x, B_Q_FREE, (uint32_t)((c - 1) & 1))) break;
                tc_fence_after();
                // M1: U = U~ - S0 W^T (committed alone: it gates the chain)
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
                    const uint64_t a = sdesc_sw128(sb + OFF_S + off, 16, 1024);
                    const uint64_t b = sdesc_sw128(sb + OFF_W + k * 2048, 8192, 1024);
                    if (elect_one()) mma_bf16(tmem + TM_U, a, b, id_m1, 1);
                    __syncwarp();
                }
                commit(B_U_MMA);
                // O1: S0 Q^T
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
                    const uint64_t a = sdesc_sw128(sb + OFF_S + off, 16, 1024);
                    const uint64_t b = sdesc_sw128(qk + off, 16, 1024);
                    if (elect_one()) mma_bf16(tmem + TM_Q, a, b, id_x, k > 0);
                    __syncwarp();
                }
                if (c + 1 < nchunks) {
                    if (!wait_bar(x, B_QK_FULL0 + ((c + 1) & 1), (uint32_t)(((c + 1) >> 1) & 1)))
                        break;
                    tc_fence_after();
                    issue_x(c + 1);
                }
                if (!wait_bar(x, B_U_FULL, ph)) break;
                tc_fence_after();
                // M4: S += Ub K (Ub hi/lo from TMEM; S already scaled by gamma_L)
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint64_t kb = sdesc_sw128(qk + 8192 + k * 2048, 16384, 1024);
                    if (elect_one()) {
                        mma_bf16_ts(tmem + TM_S, tmem + TM_BH + k * 8, kb, id_m4, 1);
                        mma_bf16_ts(tmem + TM_S, tmem + TM_BL + k * 8, kb, id_m4, 1);
                    }
                    __syncwarp();
                }
                commit(B_DS_FULL);
                // M3: DO = U P^T (hi/lo cross terms)
                const uint32_t pb = sb + OFF_P + (c & 1) * P_BUF;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint64_t ph_d = sdesc_sw128(pb + k * 32, 16, 1024);
                    const uint64_t pl_d = sdesc_sw128(pb + 8192 + k * 32, 16, 1024);
                    if (elect_one()) {
                        mma_bf16_ts(tmem + TM_O, tmem + TM_UH + k * 8, ph_d, id_x, k > 0);
                        mma_bf16_ts(tmem + TM_O, tmem + TM_UH + k * 8, pl_d, id_x, 1);
                        mma_bf16_ts(tmem + TM_O, tmem + TM_UL + k * 8, ph_d, id_x, 1);
                    }
                    __syncwarp();
                }
                commit(B_O_FULL);
                commit(B_P_FREE0 + (c & 1));
                commit(B_QK_FREE0 + (c & 1));
                if (c + 1 < nchunks) {
                    const uint32_t ph1 = (uint32_t)((c + 1) & 1);
                    if (!wait_bar(x, B_T_FULL, ph1) || !wait_bar(x, B_V_FULL, ph1)) break;
                    tc_fence_after();
                    issue_wu(c + 1);
                }
            }
        }
    } else if (warp < kPrepWarp0) {
        // ------------------------------------------------------------ chain warps
        const int hh = (warp - kChainWarp0) >> 2;
        const int i = 32 * (warp & 3) + lane;  // state row (value index)
        float *cg = reinterpret_cast<float *>(sm + OFF_CG) + (warp - kChainWarp0) * 128;  // G, gamma
        {
            // start state: fp32 into TMEM (this thread's 64 columns), bf16 copy for S0
            float v[64];
            const float *src = p.h0 ? p.h0 + sbase + (size_t)i * DH + hh * 64 : nullptr;
#pragma unroll
            for (int j = 0; j < 64; j += 4) {
                const float4 v4 = src ? *reinterpret_cast<const float4 *>(src + j)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
                v[j] = v4.x;
                v[j + 1] = v4.y;
                v[j + 2] = v4.z;
                v[j + 3] = v4.w;
            }
            st_row64_sw128(sb + OFF_S + hh * 16384, i, v);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) arrive(x, B_S0_FULL);
            if (nchunks > 0) {
                // pre-scale by gamma_L of chunk 0
                const float2 gp = load_g_pair(p.g, bos, chunk_len(0), HV, h);
                const float gL = expf(__shfl_sync(0xffffffffu, warp_decay_scan(gp.x, gp.y).y, 31));
#pragma unroll
                for (int j = 0; j < 64; ++j) v[j] *= gL;
            }
            tmem_st32f(tmem_addr(tmem, warp, TM_S + 64 * hh), v);
            tmem_st32f(tmem_addr(tmem, warp, TM_S + 64 * hh + 32), v + 32);
            tmem_wait_st();
        }
        float2 gnext = nchunks > 0 ? load_g_pair(p.g, bos, chunk_len(0), HV, h) : make_float2(0.f, 0.f);
        for (int c = 0; c < nchunks; ++c) {
            const uint32_t ph = (uint32_t)(c & 1);
            const int64_t s0 = bos + (int64_t)c * C;
            const int L = chunk_len(c);
            {
                const float2 G = warp_decay_scan(gnext.x, gnext.y);
                cg[2 * lane] = G.x;
                cg[2 * lane + 1] = G.y;
                cg[64 + 2 * lane] = expf(G.x);
                cg[64 + 2 * lane + 1] = expf(G.y);
                __syncwarp();
            }
            const float GL = cg[63];
            if (c + 1 < nchunks) gnext = load_g_pair(p.g, s0 + C, chunk_len(c + 1), HV, h);
            if (!wait_bar(x, B_U_MMA, ph)) break;
            tc_fence_after();
            {  // U epilogue: this thread's 32 tokens t = 32 hh + j of row i
                float u[32];
                tmem_ld32(tmem_addr(tmem, warp, TM_U + 32 * hh), u);
                uint32_t whi[16], wlo[16];
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (32 * hh + j >= L) u[j] = 0.f;
                split_pack32(u, whi, wlo);
                tmem_st16w(tmem_addr(tmem, warp, TM_UH + 16 * hh), whi);
                tmem_st16w(tmem_addr(tmem, warp, TM_UL + 16 * hh), wlo);
#pragma unroll
                for (int j = 0; j < 32; ++j) u[j] *= __expf(GL - cg[32 * hh + j]);
                split_pack32(u, whi, wlo);
                tmem_st16w(tmem_addr(tmem, warp, TM_BH + 16 * hh), whi);
                tmem_st16w(tmem_addr(tmem, warp, TM_BL + 16 * hh), wlo);
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) arrive(x, B_U_FULL);
            // decay of the next chunk (for the in-place state scaling)
            float gLn = 1.f;
            if (c + 1 < nchunks) {
                const float2 Gn = warp_decay_scan(gnext.x, gnext.y);
                gLn = expf(__shfl_sync(0xffffffffu, Gn.y, 31));
            }
            if (!wait_bar(x, B_DS_FULL, ph)) break;
            tc_fence_after();
            {  // new state: bf16 copy for the next chunk's S0, then scale by its gamma_L
                float v[64];
                tmem_ld32(tmem_addr(tmem, warp, TM_S + 64 * hh), v);
                tmem_ld32(tmem_addr(tmem, warp, TM_S + 64 * hh + 32), v + 32);
                st_row64_sw128(sb + OFF_S + hh * 16384, i, v);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) arrive(x, B_S0_FULL);
                if (c + 1 < nchunks) {
#pragma unroll
                    for (int j = 0; j < 64; ++j) v[j] *= gLn;
                    tmem_st32f(tmem_addr(tmem, warp, TM_S + 64 * hh), v);
                    tmem_st32f(tmem_addr(tmem, warp, TM_S + 64 * hh + 32), v + 32);
                    tmem_wait_st();
                }
            }
            if (!wait_bar(x, B_O_FULL, ph)) break;
            tc_fence_after();
            {  // output: o_t = scale (gamma_t DQ[i][t] + DO[i][t]) for this thread's 32 tokens
                float dq[32], dout[32];
                tmem_ld32(tmem_addr(tmem, warp, TM_Q + 32 * hh), dq);
                tmem_ld32(tmem_addr(tmem, warp, TM_O + 32 * hh), dout);
                __nv_bfloat16 *orow = p.o + ((size_t)s0 * HV + h) * DH + i;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int t = 32 * hh + j;
                    const float gt = cg[64 + t];
                    if (t < L)
                        orow[(size_t)t * HV * DH] =
                            __float2bfloat16_rn(p.scale * fmaf(gt, dq[j], dout[j]));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) arrive(x, B_Q_FREE);
        }
        if (!*abort_flag && p.hT) {
            float v[64];
            tmem_ld32(tmem_addr(tmem, warp, TM_S + 64 * hh), v);
            tmem_ld32(tmem_addr(tmem, warp, TM_S + 64 * hh + 32), v + 32);
            float *dst = p.hT + sbase + (size_t)i * DH + hh * 64;
#pragma unroll
            for (int j = 0; j < 64; j += 4)
                *reinterpret_cast<float4 *>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
        }
    } else {
        // ------------------------------------------------------------ prep warps
        const int pt = tid - 32 * kPrepWarp0;          // 0..255
        const int r = 32 * (warp & 3) + lane;          // TMEM lane of this thread
        const int ph2 = (warp - kPrepWarp0) >> 2;      // which half of the row's columns
        float *beta_s = reinterpret_cast<float *>(sm + OFF_PB);
        float *gam_p = beta_s + 64;
        float *G_p = gam_p + 64;
        float *A_s = reinterpret_cast<float *>(sm + OFF_A);    // [64][A_LD]
        float *T_s = reinterpret_cast<float *>(sm + OFF_TF);   // [64][T_LD]
        float *X_s = reinterpret_cast<float *>(sm + OFF_X);    // [32][X_LD]
        float2 gnext = make_float2(0.f, 0.f), bnext = make_float2(0.f, 0.f);
        if (warp == kPrepWarp0 && nchunks > 0) {
            gnext = load_g_pair(p.g, bos, chunk_len(0), HV, h);
            bnext = load_g_pair(p.beta, bos, chunk_len(0), HV, h);
        }
        for (int c = 0; c < nchunks; ++c) {
            const uint32_t ph = (uint32_t)(c & 1);
            const int64_t s0 = bos + (int64_t)c * C;
            if (warp == kPrepWarp0) {
                const float2 Gv = warp_decay_scan(gnext.x, gnext.y);
                G_p[2 * lane] = Gv.x;
                G_p[2 * lane + 1] = Gv.y;
                gam_p[2 * lane] = expf(Gv.x);
                gam_p[2 * lane + 1] = expf(Gv.y);
                beta_s[2 * lane] = bnext.x;
                beta_s[2 * lane + 1] = bnext.y;
                if (c + 1 < nchunks) {
                    gnext = load_g_pair(p.g, s0 + C, chunk_len(c + 1), HV, h);
                    bnext = load_g_pair(p.beta, s0 + C, chunk_len(c + 1), HV, h);
                }
            }
            bool ok = wait_bar(x, B_X_FULL, ph);
            if (ok && r < 64 && c >= 2)
                ok = wait_bar(x, B_P_FREE0 + (c & 1), (uint32_t)(((c >> 1) - 1) & 1));
            prep_sync();
            if (*abort_flag) break;
            tc_fence_after();
            {  // P rows (r < 64) and A rows (r >= 64) from [Q;K] K^T, 32 columns per thread
                float v[32];
                tmem_ld32(tmem_addr(tmem, warp, TM_D1 + 32 * ph2), v);
                const int row = r & 63;
                const float Gi = G_p[row];
                if (r < 64) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int col = 32 * ph2 + j;
                        v[j] = (col <= row) ? __expf(Gi - G_p[col]) * v[j] : 0.f;
                    }
                    const uint32_t pb = sb + OFF_P + (c & 1) * P_BUF;
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        const uint32_t off = sw128_chunk(row, 4 * ph2 + cc);
                        st_chunk_hilo(pb + off, pb + 8192 + off, v + 8 * cc);
                    }
                } else {
                    const float bi = beta_s[row];
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int col = 32 * ph2 + j;
                        v[j] = (col < row) ? bi * __expf(Gi - G_p[col]) * v[j] : 0.f;
                    }
                    float4 *dst = reinterpret_cast<float4 *>(A_s + row * A_LD + 32 * ph2);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            prep_sync();
            // ---- UT inverse, step 1: 16x16 diagonal blocks (threads 0..63) ----
            if (pt < 64) {
                const int b = pt >> 4, j = pt & 15, o0 = 16 * b;
                float xc[16];
#pragma unroll
                for (int ii = 0; ii < 16; ++ii) {
                    const float *arow = A_s + (o0 + ii) * A_LD + o0;
                    float acc0 = (ii == j) ? 1.f : 0.f, acc1 = 0.f;
#pragma unroll
                    for (int m = 0; m < ii; m += 2) {
                        acc0 = fmaf(-arow[m], xc[m], acc0);
                        if (m + 1 < ii) acc1 = fmaf(-arow[m + 1], xc[m + 1], acc1);
                    }
                    xc[ii] = acc0 + acc1;
                    T_s[(o0 + ii) * T_LD + o0 + j] = xc[ii];
                }
            }
            prep_sync();
            // ---- step 2: within each 32x32 half, T10 = -T11 A10 T00 (16x16 blocks) ----
            {
                const int e = pt * 2;                  // 2 consecutive outputs (same row)
                const int hf = e >> 8, ii = (e >> 4) & 15, j = e & 15;
                const int r1 = 32 * hf + 16, c0 = 32 * hf;
                float a0 = 0.f, a1 = 0.f;
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    const float am = A_s[(r1 + ii) * A_LD + c0 + m];
                    const float t0 = (m >= j) ? T_s[(c0 + m) * T_LD + c0 + j] : 0.f;
                    const float t1 = (m >= j + 1) ? T_s[(c0 + m) * T_LD + c0 + j + 1] : 0.f;
                    a0 = fmaf(am, t0, a0);
                    a1 = fmaf(am, t1, a1);
                }
                X_s[(16 * hf + ii) * X_LD + j] = a0;
                X_s[(16 * hf + ii) * X_LD + j + 1] = a1;
            }
            prep_sync();
            {
                const int e = pt * 2;
                const int hf = e >> 8, ii = (e >> 4) & 15, j = e & 15;
                const int r1 = 32 * hf + 16, c0 = 32 * hf;
                float a0 = 0.f, a1 = 0.f;
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    const float tm = (m <= ii) ? T_s[(r1 + ii) * T_LD + r1 + m] : 0.f;
                    a0 = fmaf(tm, X_s[(16 * hf + m) * X_LD + j], a0);
                    a1 = fmaf(tm, X_s[(16 * hf + m) * X_LD + j + 1], a1);
                }
                T_s[(r1 + ii) * T_LD + c0 + j] = -a0;
                T_s[(r1 + ii) * T_LD + c0 + j + 1] = -a1;
            }
            prep_sync();
            // ---- step 3: T[32:64][0:32] = -T22 A21 T11 (32x32 blocks), 4 outputs per thread ----
            {
                const int ii = pt >> 3, j = (pt & 7) * 4;
                float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
                for (int m = 0; m < 32; ++m) {
                    const float am = A_s[(32 + ii) * A_LD + m];
                    const float4 tv = *reinterpret_cast<const float4 *>(T_s + m * T_LD + j);
                    a[0] = fmaf(am, (m >= j) ? tv.x : 0.f, a[0]);
                    a[1] = fmaf(am, (m >= j + 1) ? tv.y : 0.f, a[1]);
                    a[2] = fmaf(am, (m >= j + 2) ? tv.z : 0.f, a[2]);
                    a[3] = fmaf(am, (m >= j + 3) ? tv.w : 0.f, a[3]);
                }
                *reinterpret_cast<float4 *>(X_s + ii * X_LD + j) = make_float4(a[0], a[1], a[2], a[3]);
            }
            prep_sync();
            {
                const int ii = pt >> 3, j = (pt & 7) * 4;
                float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
                for (int m = 0; m < 32; ++m) {
                    const float tm = (m <= ii) ? T_s[(32 + ii) * T_LD + 32 + m] : 0.f;
                    const float4 xv = *reinterpret_cast<const float4 *>(X_s + m * X_LD + j);
                    a[0] = fmaf(tm, xv.x, a[0]);
                    a[1] = fmaf(tm, xv.y, a[1]);
                    a[2] = fmaf(tm, xv.z, a[2]);
                    a[3] = fmaf(tm, xv.w, a[3]);
                }
                *reinterpret_cast<float4 *>(T_s + (32 + ii) * T_LD + j) =
                    make_float4(-a[0], -a[1], -a[2], -a[3]);
            }
            prep_sync();
            // ---- T' = T diag(b gamma), T'' = T diag(b) as hi/lo bf16 tiles (rows t, cols s) ----
            {
                const int t = pt >> 2, qtr = pt & 3;   // 16 columns: chunks 2 qtr, 2 qtr + 1
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int chunk16 = 2 * qtr + cc;
                    float a1[8], a2[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int s = 8 * chunk16 + e;
                        const float tv = (s <= t) ? T_s[t * T_LD + s] : 0.f;
                        a2[e] = tv * beta_s[s];
                        a1[e] = a2[e] * gam_p[s];
                    }
                    const uint32_t off = sw128_chunk(t, chunk16);
                    st_chunk_hilo(sb + OFF_T + off, sb + OFF_T + 8192 + off, a1);
                    st_chunk_hilo(sb + OFF_T + 16384 + off, sb + OFF_T + 24576 + off, a2);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) arrive(x, B_T_FULL);
            // ---- W epilogue ----
            ok = wait_bar(x, B_WU_FULL, ph);
            prep_sync();
            if (*abort_flag) break;
            tc_fence_after();
            {
                float v[32];
                tmem_ld32(tmem_addr(tmem, warp, TM_D1 + 32 * ph2), v);  // W^T row a = r
#pragma unroll
                for (int cc = 0; cc < 4; ++cc)
                    st_shared_bf16x8(sb + OFF_W + sw128_chunk(r, 4 * ph2 + cc), v + 8 * cc);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) arrive(x, B_W_FULL);
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
