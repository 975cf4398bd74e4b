// Chunkwise prefill of the gated delta rule on a thread-block cluster per
// (sequence, value head): one chain CTA and three prep CTAs (bf16 q/k/v, head
// dim 128, chunk 64, fp32 state and accumulation).
//
// Rule and chunk form as in gdn_prefill_tc.cu ("Qwen3-Next", sghael.github.io,
// section "Correcting a memory instead of adding to it"; model card
// "Qwen3-Next-80B-A3B-Instruct", section "Model Overview"):
//   A_ij = b_i exp(G_i - G_j) k_i.k_j (j < i),  T = (I + A)^-1,
//   P_ij = exp(G_i - G_j) q_i.k_j (j <= i),
//   W = T diag(b gamma) K,  U~ = T diag(b) V,  U = U~ - W S0^T,
//   O = diag(gamma) Q S0^T + P U,  S = gamma_L S0 + U^T diag(gamma_L/gamma) K.
//
// Split by dependence on the state:
//   prep CTAs (cluster ranks 1..3) take every third chunk and compute the
//     state-independent part: [Q;K]K^T, A and P, the UT inverse T (blocked
//     16 -> 32 -> 64 on CUDA cores), W and U~ (tcgen05), and ship W (bf16),
//     U~ (fp32) and P (bf16 hi + lo) as one 64 KB block into the chain CTA's
//     shared memory with a bulk DSMEM copy that completes on the chain CTA's
//     mbarrier;
//   the chain CTA (rank 0) walks the chunks in order: D = S0 W^T and S0 Q^T
//     (S0 as a bf16 operand in tensor memory), U = U~ - D, the state update
//     S += (U diag(gamma_L/gamma)) K accumulated in tensor memory after an
//     in-place gamma_L scaling, and the outputs U P^T + gamma_t S0 Q^T, written
//     by dedicated output warps through a small shared-memory transpose.
// Hand-over: the chain CTA re-arms its receive slot and releases the producing
// prep CTA with remote mbarrier arrivals; every wait is bounded (sleeping
// try_wait), and a timeout winds the CTA down and reports GDN_ERR_TIMEOUT.
//
// Precision as in gdn_prefill_tc.cu: exact bf16 q/k/v; T', T'', P, U and
// U diag(gamma_L/gamma) as bf16 hi + lo pairs; U~ crosses in fp32; gamma_t of
// the inter-chunk read-out applied in fp32; only S0 and W are single bf16.
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

constexpr int C = 64;
constexpr int DH = 128;
constexpr int kNumPrep = 3;
constexpr int kClusterSize = 1 + kNumPrep;
constexpr int kThreads = 18 * 32;
// chain CTA roles
constexpr int kCTma = 0, kCMma = 1, kCChain0 = 2, kCNumChain = 8, kCOut0 = 10, kCNumOut = 8;
// prep CTA roles
constexpr int kPCtl = 0, kPWork0 = 1, kPNumWork = 8, kPWorkThreads = kPNumWork * 32;
constexpr uint32_t kWait = 2000;  // sleeping polls (<= ~1 ms each) before a wait gives up

// ---- one chunk's hand-over block (prep staging == chain receive slot) ----
constexpr uint32_t SL_W = 0;        // W, MN-major B operand: 128 rows (a) x 64 (t), 128B swizzle
constexpr uint32_t SL_PH = 16384;   // P hi: 64 rows (t) x 64 (s)
constexpr uint32_t SL_PL = 24576;   // P lo
constexpr uint32_t SL_U = 32768;    // U~ fp32 [i][t], 16-byte chunks xor-swizzled by row
constexpr uint32_t SLOT = 65536;

// ---- chain CTA shared memory ----
constexpr uint32_t C_Q = 0;         // 2 stages x 16 KB (q tile, two atom columns)
constexpr uint32_t C_K = 32768;     // 2 stages x 16 KB
constexpr uint32_t C_R = 65536;     // 2 receive slots x 64 KB
constexpr uint32_t C_TAB = C_R + 2 * SLOT;  // per chain warp gamma_L/gamma, per output warp gamma
constexpr uint32_t C_OST = C_TAB + (kCNumChain + kCNumOut) * 512;  // o tile staging (TMA store)
constexpr uint32_t C_BAR = C_OST + 16384;
// ---- prep CTA shared memory ----
constexpr uint32_t P_QK = 0;        // [atom0: Q | K][atom1: Q | K]
constexpr uint32_t P_V = 32768;
constexpr uint32_t P_T = 49152;     // T' hi, T' lo, T'' hi, T'' lo (4 x 8 KB); A fp32 shares it
constexpr uint32_t A_LD = 68;
constexpr uint32_t P_TF = 81920;    // T fp32 [64][T_LD]
constexpr uint32_t T_LD = 68;
constexpr uint32_t P_X = P_TF + 64 * T_LD * 4;
constexpr uint32_t X_LD = 36;
constexpr uint32_t P_PB = P_X + 32 * X_LD * 4;             // beta, gamma, G
constexpr uint32_t P_ST = 105472;   // staging block (SLOT bytes)
constexpr uint32_t P_BAR = P_ST + SLOT;
constexpr uint32_t SMEM_BYTES = (C_BAR > P_BAR ? C_BAR : P_BAR) + 256 + 1024;
static_assert(P_PB + 3 * 64 * 4 <= P_ST, "prep layout");
static_assert(64 * A_LD * 4 <= 32768, "A fits the T tiles");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(C_OST % 1024 == 0, "128B-swizzled staging tile alignment");

// ---- TMEM columns ----
// chain: D = S0 W^T, S0 Q^T, U P^T, S0 (bf16 A operand), S (fp32), U/Ub hi/lo (bf16 A)
constexpr uint32_t TM_D = 0, TM_Q = 64, TM_O = 128, TM_S0 = 192, TM_S = 256;
constexpr uint32_t TM_UH = 384, TM_UL = 416, TM_BH = 448, TM_BL = 480;
// prep: X then W^T, U~^T
constexpr uint32_t TP_D1 = 0, TP_U = 64;

enum ChainBar {
    CB_QK_FULL0, CB_QK_FULL1, CB_QK_FREE0, CB_QK_FREE1, CB_R_FULL0, CB_R_FULL1, CB_S0_FULL,
    CB_U_MMA, CB_U_FULL, CB_U2_FULL, CB_DS_FULL, CB_O_FULL, CB_Q_FREE, CB_COUNT
};
enum PrepBar { PB_LD_FULL, PB_X_DONE, PB_T_READY, PB_WU_DONE, PB_EPI_DONE, PB_GO, PB_STAGE_FREE,
               PB_COUNT };

struct ClParams {
    const float *g, *beta, *h0;
    const int32_t *cu;
    int64_t T;
    int HK, HV;
    float scale;
    __nv_bfloat16 *o;
    float *hT;
    unsigned int *status;
};

struct Waiter {
    uint64_t *bars;
    volatile int *abort_flag;
    unsigned int *status;
    __device__ bool operator()(int b, uint32_t parity) const {
        for (uint32_t i = 0; i < kWait; ++i) {
            if (mbar_try_wait_sleep(&bars[b], parity, 1000000u)) return true;
            if (*abort_flag) return false;
        }
        *abort_flag = 1;
        atomicExch(status, (unsigned int)GDN_ERR_TIMEOUT);
        return false;
    }
};

__device__ __forceinline__ void local_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void work_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kPWorkThreads) : "memory");
}
__device__ __forceinline__ void out_sync() {
    asm volatile("bar.sync 2, %0;" ::"n"(kCNumOut * 32) : "memory");
}
// fp32 U~ tile [i][t]: byte offset of the 16-byte chunk holding t = 4*tc .. 4*tc+3 of row i
__device__ __forceinline__ uint32_t ut_chunk(uint32_t i, uint32_t tc) {
    return i * 256u + (((tc ^ i) & 15u) << 4);
}

// ============================================================================ chain CTA
__device__ void chain_cta(const CUtensorMap *tm_q, const CUtensorMap *tm_k, const CUtensorMap *tm_o,
                          const ClParams &p,
                          uint8_t *sm, uint32_t sb, uint32_t tmem, const Waiter &wt, int h,
                          int n, int64_t bos, int64_t eos, int nchunks) {
    uint64_t *bars = wt.bars;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int HV = p.HV, cqk = h / (HV / p.HK);
    const size_t sbase = ((size_t)n * HV + h) * (size_t)DH * DH;
    auto chunk_len = [&](int c) {
        const int64_t r = eos - (bos + (int64_t)c * C);
        return (int)(r < C ? r : C);
    };
    if (warp == kCTma) {
        if (lane == 0) {
            tma_prefetch_desc(tm_q);
            tma_prefetch_desc(tm_k);
            for (int c = 0; c < nchunks; ++c) {
                const int st = c & 1;
                const int s0 = (int)(bos + (int64_t)c * C);
                if (c >= 2 && !wt(CB_QK_FREE0 + st, (uint32_t)(((c >> 1) - 1) & 1))) break;
                mbar_arrive_expect_tx(&bars[CB_QK_FULL0 + st], 4 * 8192);
                uint8_t *qd = sm + C_Q + st * 16384, *kd = sm + C_K + st * 16384;
                tma_load_3d(qd, tm_q, &bars[CB_QK_FULL0 + st], 0, cqk, s0);
                tma_load_3d(qd + 8192, tm_q, &bars[CB_QK_FULL0 + st], 64, cqk, s0);
                tma_load_3d(kd, tm_k, &bars[CB_QK_FULL0 + st], 0, cqk, s0);
                tma_load_3d(kd + 8192, tm_k, &bars[CB_QK_FULL0 + st], 64, cqk, s0);
            }
        }
    } else if (warp == kCMma) {
        const uint32_t id_n64_mn = idesc_bf16(128, 64, false, true);
        const uint32_t id_n64 = idesc_bf16(128, 64, false, false);
        const uint32_t id_n128_mn = idesc_bf16(128, 128, false, true);
        auto commit = [&](int b) {
            if (elect_one()) mma_commit(&bars[b]);
            __syncwarp();
        };
        for (int c = 0; c < nchunks; ++c) {
            const uint32_t ph = (uint32_t)(c & 1);
            const int s = c & 1;
            const uint32_t slot = sb + C_R + s * SLOT;
            const uint32_t qst = sb + C_Q + s * 16384, kst = sb + C_K + s * 16384;
            if (!wt(CB_R_FULL0 + s, (uint32_t)((c >> 1) & 1))) break;
            // the bulk copy out of the producing prep CTA's staging block has completed:
            // that block may be refilled
            if (elect_one())
                mbar_arrive_remote_relaxed(mapa_shared(sb + P_BAR + PB_STAGE_FREE * 8, 1 + c % kNumPrep));
            __syncwarp();
            if (!wt(CB_S0_FULL, ph)) break;
            tc_fence_after();
            // D = S0 W^T (A = S0 from TMEM, B = W MN-major from the receive slot)
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint64_t b = sdesc_sw128(slot + SL_W + k * 2048, 8192, 1024);
                if (elect_one()) mma_bf16_ts(tmem + TM_D, tmem + TM_S0 + 8 * k, b, id_n64_mn, k > 0);
                __syncwarp();
            }
            commit(CB_U_MMA);
            // S0 Q^T (its accumulator is free once the output warps read chunk c-1)
            if (c >= 1 && !wt(CB_Q_FREE, (uint32_t)((c - 1) & 1))) break;
            if (!wt(CB_QK_FULL0 + s, (uint32_t)((c >> 1) & 1))) break;
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint64_t b = sdesc_sw128(qst + (k >> 2) * 8192 + (k & 3) * 32, 16, 1024);
                if (elect_one()) mma_bf16_ts(tmem + TM_Q, tmem + TM_S0 + 8 * k, b, id_n64, k > 0);
                __syncwarp();
            }
            if (!wt(CB_U_FULL, ph)) break;
            tc_fence_after();
            // S += (U diag(gamma_L/gamma)) K  (hi + lo)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint64_t b = sdesc_sw128(kst + k * 2048, 8192, 1024);
                if (elect_one()) {
                    mma_bf16_ts(tmem + TM_S, tmem + TM_BH + 8 * k, b, id_n128_mn, 1);
                    mma_bf16_ts(tmem + TM_S, tmem + TM_BL + 8 * k, b, id_n128_mn, 1);
                }
                __syncwarp();
            }
            commit(CB_DS_FULL);
            // U P^T (hi/lo cross terms)
            if (!wt(CB_U2_FULL, ph)) break;
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint64_t ph_d = sdesc_sw128(slot + SL_PH + k * 32, 16, 1024);
                const uint64_t pl_d = sdesc_sw128(slot + SL_PL + k * 32, 16, 1024);
                if (elect_one()) {
                    mma_bf16_ts(tmem + TM_O, tmem + TM_UH + 8 * k, ph_d, id_n64, k > 0);
                    mma_bf16_ts(tmem + TM_O, tmem + TM_UH + 8 * k, pl_d, id_n64, 1);
                    mma_bf16_ts(tmem + TM_O, tmem + TM_UL + 8 * k, ph_d, id_n64, 1);
                }
                __syncwarp();
            }
            commit(CB_O_FULL);
            commit(CB_QK_FREE0 + s);
        }
    } else if (warp < kCOut0) {
        // ------------------------------------------------------------ chain warps
        const int hh = (warp - kCChain0) >> 2;
        const int i = 32 * (warp & 3) + lane;
        float *tab = reinterpret_cast<float *>(sm + C_TAB) + (warp - kCChain0) * 128;  // gamma_L/gamma
        {
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
            uint32_t w[16];
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2) {
#pragma unroll
                for (int j = 0; j < 16; ++j) w[j] = pack_bf16x2(v[32 * q2 + 2 * j], v[32 * q2 + 2 * j + 1]);
                tmem_st16w(tmem_addr(tmem, warp, TM_S0 + 32 * hh + 16 * q2), w);
            }
            if (nchunks > 0) {
                const float2 gp = load_g_pair(p.g, bos, chunk_len(0), HV, h);
                const float gL = expf(__shfl_sync(0xffffffffu, warp_decay_scan(gp.x, gp.y).y, 31));
#pragma unroll
                for (int j = 0; j < 64; ++j) v[j] *= gL;
            }
            tmem_st32f(tmem_addr(tmem, warp, TM_S + 64 * hh), v);
            tmem_st32f(tmem_addr(tmem, warp, TM_S + 64 * hh + 32), v + 32);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) local_arrive(&bars[CB_S0_FULL]);
        }
        float2 gnext = nchunks > 0 ? load_g_pair(p.g, bos, chunk_len(0), HV, h) : make_float2(0.f, 0.f);
        for (int c = 0; c < nchunks; ++c) {
            const uint32_t ph = (uint32_t)(c & 1);
            const int s = c & 1;
            const int64_t s0 = bos + (int64_t)c * C;
            const int L = chunk_len(c);
            {
                const float2 G = warp_decay_scan(gnext.x, gnext.y);
                const float GL = __shfl_sync(0xffffffffu, G.y, 31);
                tab[2 * lane] = __expf(GL - G.x);
                tab[2 * lane + 1] = __expf(GL - G.y);
                __syncwarp();
            }
            if (c + 1 < nchunks) gnext = load_g_pair(p.g, s0 + C, chunk_len(c + 1), HV, h);
            if (!wt(CB_R_FULL0 + s, (uint32_t)((c >> 1) & 1))) break;
            if (!wt(CB_U_MMA, ph)) break;
            tc_fence_after();
            {  // U = U~ - S0 W^T for this thread's 32 tokens t = 32 hh + j of row i
                float u[32];
                tmem_ld32(tmem_addr(tmem, warp, TM_D + 32 * hh), u);
                const uint8_t *ut = sm + C_R + s * SLOT + SL_U;
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4) {
                    const float4 a = *reinterpret_cast<const float4 *>(ut + ut_chunk(i, 8 * hh + q4));
                    u[4 * q4] = a.x - u[4 * q4];
                    u[4 * q4 + 1] = a.y - u[4 * q4 + 1];
                    u[4 * q4 + 2] = a.z - u[4 * q4 + 2];
                    u[4 * q4 + 3] = a.w - u[4 * q4 + 3];
                }
                uint32_t whi[16], wlo[16];
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (32 * hh + j >= L) u[j] = 0.f;
                float ub[32];
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4) {
                    const float4 f = *reinterpret_cast<const float4 *>(tab + 32 * hh + 4 * q4);
                    ub[4 * q4] = u[4 * q4] * f.x;
                    ub[4 * q4 + 1] = u[4 * q4 + 1] * f.y;
                    ub[4 * q4 + 2] = u[4 * q4 + 2] * f.z;
                    ub[4 * q4 + 3] = u[4 * q4 + 3] * f.w;
                }
                split_pack32(ub, whi, wlo);
                tmem_st16w(tmem_addr(tmem, warp, TM_BH + 16 * hh), whi);
                tmem_st16w(tmem_addr(tmem, warp, TM_BL + 16 * hh), wlo);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) local_arrive(&bars[CB_U_FULL]);   // the state update can start
                split_pack32(u, whi, wlo);
                tmem_st16w(tmem_addr(tmem, warp, TM_UH + 16 * hh), whi);
                tmem_st16w(tmem_addr(tmem, warp, TM_UL + 16 * hh), wlo);
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) local_arrive(&bars[CB_U2_FULL]);
            float gLn = 1.f;
            if (c + 1 < nchunks) {
                const float2 Gn = warp_decay_scan(gnext.x, gnext.y);
                gLn = expf(__shfl_sync(0xffffffffu, Gn.y, 31));
            }
            if (!wt(CB_DS_FULL, ph)) break;
            tc_fence_after();
            {  // new state: bf16 copy (next chunk's S0) into TMEM, then scale by its gamma_L
                float v[64];
                tmem_ld32(tmem_addr(tmem, warp, TM_S + 64 * hh), v);
                tmem_ld32(tmem_addr(tmem, warp, TM_S + 64 * hh + 32), v + 32);
                uint32_t w[16];
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2) {
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        w[j] = pack_bf16x2(v[32 * q2 + 2 * j], v[32 * q2 + 2 * j + 1]);
                    tmem_st16w(tmem_addr(tmem, warp, TM_S0 + 32 * hh + 16 * q2), w);
                }
                if (c + 1 < nchunks) {
#pragma unroll
                    for (int j = 0; j < 64; ++j) v[j] *= gLn;
                    tmem_st32f(tmem_addr(tmem, warp, TM_S + 64 * hh), v);
                    tmem_st32f(tmem_addr(tmem, warp, TM_S + 64 * hh + 32), v + 32);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) local_arrive(&bars[CB_S0_FULL]);
        }
        if (!*wt.abort_flag && p.hT) {
            float v[64];
            tmem_ld32(tmem_addr(tmem, warp, TM_S + 64 * hh), v);
            tmem_ld32(tmem_addr(tmem, warp, TM_S + 64 * hh + 32), v + 32);
            float *dst = p.hT + sbase + (size_t)i * DH + hh * 64;
#pragma unroll
            for (int j = 0; j < 64; j += 4)
                *reinterpret_cast<float4 *>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
        }
    } else {
        // ------------------------------------------------------------ output warps
        const int half = (warp - kCOut0) >> 2;   // tokens 32 half .. 32 half + 31
        const int i = 32 * (warp & 3) + lane;    // value row of this thread
        float *tab = reinterpret_cast<float *>(sm + C_TAB) + (warp - kCChain0) * 128;  // gamma
        // o tile [t][i] as two 128B-swizzled 64-column halves, the layout of the store map
        uint8_t *ost = sm + C_OST;
        const uint32_t obase = (uint32_t)(i >> 6) * 8192u + (uint32_t)(i & 7) * 2u;
        const uint32_t ochunk = (uint32_t)((i & 63) >> 3);
        const bool leader = warp == kCOut0 && lane == 0;
        float2 gnext = nchunks > 0 ? load_g_pair(p.g, bos, chunk_len(0), HV, h) : make_float2(0.f, 0.f);
        for (int c = 0; c < nchunks; ++c) {
            const uint32_t ph = (uint32_t)(c & 1);
            const int64_t s0 = bos + (int64_t)c * C;
            const int L = chunk_len(c);
            {
                const float2 G = warp_decay_scan(gnext.x, gnext.y);
                tab[2 * lane] = expf(G.x);
                tab[2 * lane + 1] = expf(G.y);
                __syncwarp();
            }
            if (c + 1 < nchunks) gnext = load_g_pair(p.g, s0 + C, chunk_len(c + 1), HV, h);
            if (!wt(CB_O_FULL, ph)) break;
            tc_fence_after();
            // every MMA reading the receive slot of chunk c has completed: re-arm it
            // and release the prep CTA that produces chunk c + 2 into it
            if (warp == kCOut0 && c + 2 < nchunks) {
                if (lane == 0) {
                    mbar_arrive_expect_tx(&bars[CB_R_FULL0 + (c & 1)], SLOT);
                    mbar_arrive_remote_relaxed(
                        mapa_shared(sb + P_BAR + PB_GO * 8, 1 + (c + 2) % kNumPrep));
                }
                __syncwarp();
            }
            float dq[32], dout[32];
            tmem_ld32(tmem_addr(tmem, warp, TM_Q + 32 * half), dq);
            tmem_ld32(tmem_addr(tmem, warp, TM_O + 32 * half), dout);
            // both accumulators are in registers: the next chunk's MMAs may overwrite them
            tc_fence_before();
            __syncwarp();
            if (lane == 0) local_arrive(&bars[CB_Q_FREE]);
            // the previous chunk's tile store has finished reading the staging tile
            if (leader) bulk_wait_group_read0();
            out_sync();
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4) {
                const float4 gm = *reinterpret_cast<const float4 *>(tab + 32 * half + 4 * q4);
                const float gv[4] = {gm.x, gm.y, gm.z, gm.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = 4 * q4 + e, t = 32 * half + j;
                    const __nv_bfloat16 bv = __float2bfloat16_rn(p.scale * fmaf(gv[e], dq[j], dout[j]));
                    *reinterpret_cast<__nv_bfloat16 *>(ost + obase + t * 128 +
                                                       ((ochunk ^ (uint32_t)(t & 7)) << 4)) = bv;
                }
            }
            fence_proxy_async_smem();
            out_sync();
            if (L == C) {
                if (leader) {
                    tma_store_3d(tm_o, ost, 0, h, (int)s0);
                    tma_store_3d(tm_o, ost + 8192, 64, h, (int)s0);
                    bulk_commit_group();
                }
            } else {
                // short last chunk: the rows past the sequence end belong to the next
                // sequence, so only rows t < L are written, 16 bytes per thread and step
                for (int e = tid - 32 * kCOut0; e < L * 16; e += kCNumOut * 32) {
                    const int t = e >> 4, ch = e & 15;
                    const uint4 val = *reinterpret_cast<const uint4 *>(
                        ost + (ch >> 3) * 8192 + t * 128 + (((ch & 7) ^ (t & 7)) << 4));
                    *reinterpret_cast<uint4 *>(p.o + ((size_t)(s0 + t) * HV + h) * DH + ch * 8) = val;
                }
            }
        }
        // the tile stores complete before the CTA (and its shared memory) goes away
        if (leader) bulk_wait_group0();
    }
}

// ============================================================================ prep CTA
__device__ void prep_cta(const CUtensorMap *tm_q, const CUtensorMap *tm_k, const CUtensorMap *tm_v,
                         const ClParams &p, uint8_t *sm, uint32_t sb, uint32_t tmem,
                         const Waiter &wt, int h, int64_t bos, int64_t eos, int nchunks,
                         int rank) {
    uint64_t *bars = wt.bars;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int HV = p.HV, cqk = h / (HV / p.HK);
    const int first = rank - 1;                                   // chunks first, first+3, ...
    const int nk = nchunks > first ? (nchunks - first + kNumPrep - 1) / kNumPrep : 0;
    auto chunk_of = [&](int k) { return first + kNumPrep * k; };
    auto chunk_len = [&](int c) {
        const int64_t r = eos - (bos + (int64_t)c * C);
        return (int)(r < C ? r : C);
    };
    if (warp == kPCtl) {
        const uint32_t id_x = idesc_bf16(128, 64, false, false);
        const uint32_t id_w = idesc_bf16(128, 64, true, false);
        auto commit = [&](int b) {
            if (elect_one()) mma_commit(&bars[b]);
            __syncwarp();
        };
        auto load = [&](int c) {
            if (lane == 0) {
                const int s0 = (int)(bos + (int64_t)c * C);
                mbar_arrive_expect_tx(&bars[PB_LD_FULL], 6 * 8192);
                tma_load_3d(sm + P_QK, tm_q, &bars[PB_LD_FULL], 0, cqk, s0);
                tma_load_3d(sm + P_QK + 16384, tm_q, &bars[PB_LD_FULL], 64, cqk, s0);
                tma_load_3d(sm + P_QK + 8192, tm_k, &bars[PB_LD_FULL], 0, cqk, s0);
                tma_load_3d(sm + P_QK + 24576, tm_k, &bars[PB_LD_FULL], 64, cqk, s0);
                tma_load_3d(sm + P_V, tm_v, &bars[PB_LD_FULL], 0, h, s0);
                tma_load_3d(sm + P_V + 8192, tm_v, &bars[PB_LD_FULL], 64, h, s0);
            }
            __syncwarp();
        };
        if (nk > 0) {
            if (lane == 0) {
                tma_prefetch_desc(tm_q);
                tma_prefetch_desc(tm_k);
                tma_prefetch_desc(tm_v);
            }
            load(chunk_of(0));
        }
        for (int k = 0; k < nk; ++k) {
            const int c = chunk_of(k);
            const uint32_t ph = (uint32_t)(k & 1);
            if (!wt(PB_LD_FULL, ph)) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                const uint64_t a = sdesc_sw128(sb + P_QK + off, 16, 1024);
                const uint64_t b = sdesc_sw128(sb + P_QK + 8192 + off, 16, 1024);
                if (elect_one()) mma_bf16(tmem + TP_D1, a, b, id_x, kk > 0);
                __syncwarp();
            }
            commit(PB_X_DONE);
            if (!wt(PB_T_READY, ph)) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ka = sdesc_sw128(sb + P_QK + 8192 + kk * 2048, 16384, 1024);
                const uint64_t va = sdesc_sw128(sb + P_V + kk * 2048, 8192, 1024);
                const uint64_t t1h = sdesc_sw128(sb + P_T + kk * 32, 16, 1024);
                const uint64_t t1l = sdesc_sw128(sb + P_T + 8192 + kk * 32, 16, 1024);
                const uint64_t t2h = sdesc_sw128(sb + P_T + 16384 + kk * 32, 16, 1024);
                const uint64_t t2l = sdesc_sw128(sb + P_T + 24576 + kk * 32, 16, 1024);
                if (elect_one()) {
                    mma_bf16(tmem + TP_D1, ka, t1h, id_w, kk > 0);
                    mma_bf16(tmem + TP_D1, ka, t1l, id_w, 1);
                    mma_bf16(tmem + TP_U, va, t2h, id_w, kk > 0);
                    mma_bf16(tmem + TP_U, va, t2l, id_w, 1);
                }
                __syncwarp();
            }
            commit(PB_WU_DONE);
            if (!wt(PB_WU_DONE, ph)) break;   // q/k/v tiles are free again
            if (k + 1 < nk) load(chunk_of(k + 1));
            if (!wt(PB_EPI_DONE, ph)) break;
            if (c >= 2) {
                const int j = first >= 2 ? k : k - 1;   // go arrivals before this chunk
                if (!wt(PB_GO, (uint32_t)(j & 1))) break;
            }
            if (elect_one()) {
                const int s = c & 1;
                const uint32_t mbar = mapa_shared(sb + C_BAR + (CB_R_FULL0 + s) * 8, 0);
                const uint32_t dst = mapa_shared(sb + C_R + s * SLOT, 0);
#pragma unroll
                for (int part = 0; part < 4; ++part)
                    bulk_copy_to_cluster(dst + part * 16384, sb + P_ST + part * 16384, 16384, mbar);
            }
            __syncwarp();
        }
    } else if (warp < kPWork0 + kPNumWork) {
        // ------------------------------------------------------------ prep workers
        const int pt = tid - 32 * kPWork0;                 // 0..255
        const int r = 32 * (warp & 3) + lane;              // TMEM lane of this thread
        const int ph2 = (warp - kPWork0) >> 2;             // column half
        float *beta_s = reinterpret_cast<float *>(sm + P_PB);
        float *gam_p = beta_s + 64;
        float *G_p = gam_p + 64;
        float *A_s = reinterpret_cast<float *>(sm + P_T);
        float *T_s = reinterpret_cast<float *>(sm + P_TF);
        float *X_s = reinterpret_cast<float *>(sm + P_X);
        for (int k = 0; k < nk; ++k) {
            const int c = chunk_of(k);
            const uint32_t ph = (uint32_t)(k & 1);
            const int64_t s0 = bos + (int64_t)c * C;
            const int L = chunk_len(c);
            work_sync();
            if (warp == kPWork0) {
                const float2 gp = load_g_pair(p.g, s0, L, HV, h);
                const float2 Gv = warp_decay_scan(gp.x, gp.y);
                G_p[2 * lane] = Gv.x;
                G_p[2 * lane + 1] = Gv.y;
                gam_p[2 * lane] = expf(Gv.x);
                gam_p[2 * lane + 1] = expf(Gv.y);
            } else if (warp == kPWork0 + 1) {
                const float2 bp = load_g_pair(p.beta, s0, L, HV, h);
                beta_s[2 * lane] = bp.x;
                beta_s[2 * lane + 1] = bp.y;
            }
            bool ok = wt(PB_X_DONE, ph);
            if (ok && k >= 1) ok = wt(PB_STAGE_FREE, (uint32_t)((k - 1) & 1));
            work_sync();
            if (*wt.abort_flag) break;
            tc_fence_after();
            {  // P rows (r < 64) into the staging block, A rows (r >= 64) into A
                float v[32];
                tmem_ld32(tmem_addr(tmem, warp, TP_D1 + 32 * ph2), v);
                const int row = r & 63;
                const float Gi = G_p[row];
                if (r < 64) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int col = 32 * ph2 + j;
                        v[j] = (col <= row) ? __expf(Gi - G_p[col]) * v[j] : 0.f;
                    }
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        const uint32_t off = sw128_chunk(row, 4 * ph2 + cc);
                        st_chunk_hilo(sb + P_ST + SL_PH + off, sb + P_ST + SL_PL + off, v + 8 * cc);
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
            tc_fence_before();
            work_sync();
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
            work_sync();
            // ---- step 2: within each 32x32 half, T10 = -T11 A10 T00 ----
            {
                const int e = pt * 2;
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
            work_sync();
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
            work_sync();
            // ---- step 3: T[32:64][0:32] = -T22 A21 T11 ----
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
            work_sync();
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
            work_sync();
            // ---- T' = T diag(b gamma), T'' = T diag(b) as hi/lo bf16 tiles (A is dead) ----
            {
                const int t = pt >> 2, qtr = pt & 3;
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
                    st_chunk_hilo(sb + P_T + off, sb + P_T + 8192 + off, a1);
                    st_chunk_hilo(sb + P_T + 16384 + off, sb + P_T + 24576 + off, a2);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) local_arrive(&bars[PB_T_READY]);
            // ---- W and U~ epilogues into the staging block ----
            ok = wt(PB_WU_DONE, ph);
            work_sync();
            if (*wt.abort_flag) break;
            tc_fence_after();
            {
                float v[32];
                tmem_ld32(tmem_addr(tmem, warp, TP_D1 + 32 * ph2), v);  // W^T row a = r
#pragma unroll
                for (int cc = 0; cc < 4; ++cc)
                    st_shared_bf16x8(sb + P_ST + SL_W + sw128_chunk(r, 4 * ph2 + cc), v + 8 * cc);
                tmem_ld32(tmem_addr(tmem, warp, TP_U + 32 * ph2), v);   // U~^T row i = r
                uint8_t *ut = sm + P_ST + SL_U;
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4)
                    *reinterpret_cast<float4 *>(ut + ut_chunk(r, 8 * ph2 + q4)) =
                        make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) local_arrive(&bars[PB_EPI_DONE]);
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
prefill_cluster_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_o, const ClParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    const int rank = (int)cluster_ctarank();
    const int h = blockIdx.x / kClusterSize, n = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + (rank == 0 ? C_BAR : P_BAR));
    const int nbars = rank == 0 ? CB_COUNT : PB_COUNT;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + nbars);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + nbars + 1);
    const Waiter wt{bars, abort_flag, p.status};
    int64_t bos, eos;
    if (p.cu) {
        bos = p.cu[n];
        eos = p.cu[n + 1];
    } else {
        bos = (int64_t)n * p.T;
        eos = bos + p.T;
    }
    const int nchunks = (int)((eos - bos + C - 1) / C);
    const uint32_t ncols = rank == 0 ? 512u : 128u;

    if (tid == 0) {
        for (int b = 0; b < nbars; ++b) {
            uint32_t cnt = 1;
            if (rank == 0 && (b == CB_S0_FULL || b == CB_U_FULL || b == CB_U2_FULL)) cnt = kCNumChain;
            if (rank == 0 && b == CB_Q_FREE) cnt = kCNumOut;
            if (rank != 0 && (b == PB_T_READY || b == PB_EPI_DONE)) cnt = kPNumWork;
            mbar_init(&bars[b], cnt);
        }
        *abort_flag = 0;
        if (rank == 0) {
            // receive slots for chunks 0 and 1 expect their bytes from the start
            mbar_arrive_expect_tx(&bars[CB_R_FULL0], SLOT);
            mbar_arrive_expect_tx(&bars[CB_R_FULL1], SLOT);
        }
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(tslot, ncols);
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    cluster_sync_all();   // every CTA's barriers are initialised before any remote traffic

    if (rank == 0)
        chain_cta(&tm_q, &tm_k, &tm_o, p, sm, sb, tmem, wt, h, n, bos, eos, nchunks);
    else
        prep_cta(&tm_q, &tm_k, &tm_v, p, sm, sb, tmem, wt, h, bos, eos, nchunks, rank);

    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, ncols);
    cluster_sync_all();   // no CTA leaves while another may still address its shared memory
}

}  // namespace

bool prefill_cluster_supported(int dk, int dv, int chunk, gdn_dtype dtype) {
    return dtype == GDN_BF16 && dk == DH && dv == DH && chunk == C;
}

cudaError_t launch_prefill_cluster(const PrefillArgs &a, cudaStream_t stream) {
    const int64_t Ttot = a.cu_seqlens ? a.T : (int64_t)a.N * a.T;
    if (Ttot >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    unsigned int *status = static_cast<unsigned int *>(a.workspace);
    cudaError_t err = cudaMemsetAsync(status, 0, sizeof(unsigned int), stream);
    if (err != cudaSuccess) return err;
    CUtensorMap tq, tk, tv, to;
    const uint64_t tok = (uint64_t)(Ttot > 0 ? Ttot : 1);
    uint64_t dq[3] = {(uint64_t)DH, (uint64_t)a.HK, tok};
    uint64_t sq[2] = {(uint64_t)DH * 2, (uint64_t)a.HK * DH * 2};
    uint64_t dv[3] = {(uint64_t)DH, (uint64_t)a.HV, tok};
    uint64_t sv[2] = {(uint64_t)DH * 2, (uint64_t)a.HV * DH * 2};
    uint32_t box[3] = {64, 1, 64};
    if (!encode_bf16_map(&tq, a.q, 3, dq, sq, box) || !encode_bf16_map(&tk, a.k, 3, dq, sq, box) ||
        !encode_bf16_map(&tv, a.v, 3, dv, sv, box) || !encode_bf16_map(&to, a.o, 3, dv, sv, box))
        return cudaErrorInvalidValue;
    err = cudaFuncSetAttribute(prefill_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)SMEM_BYTES);
    if (err != cudaSuccess) return err;
    ClParams prm{a.g, a.beta, a.h0, a.cu_seqlens, a.T, a.HK, a.HV, a.scale,
                 static_cast<__nv_bfloat16 *>(a.o), a.hT, status};
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(kClusterSize * a.HV), (unsigned)a.N, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kClusterSize;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&cfg, prefill_cluster_kernel, tq, tk, tv, to, prm);
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
}

}  // namespace gdn
