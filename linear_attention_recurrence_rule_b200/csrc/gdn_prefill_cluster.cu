// Chunkwise prefill of the gated delta rule on a thread-block cluster per
// (sequence, value head): one chain CTA and three prep CTAs (bf16 q/k/v, head
// dim 128, chunk 64, fp32 state and accumulation).
//
// Rule and chunk form ("Qwen3-Next", sghael.github.io, section "Correcting a
// memory instead of adding to it"; model card "Qwen3-Next-80B-A3B-Instruct",
// section "Model Overview"), with G the chunk-local running sum of g and
// gamma = exp(G):
//   A_ij = b_i exp(G_i - G_j) k_i.k_j (j < i),  T = (I + A)^-1,
//   P_ij = exp(G_i - G_j) q_i.k_j (j <= i),
//   W = T diag(b gamma) K,  U~ = T diag(b) V,  U = U~ - W S0^T,
//   O = diag(gamma) Q S0^T + P U,  S = gamma_L S0 + U^T diag(gamma_L/gamma) K.
//
// Split by dependence on the state:
//   prep CTAs (cluster ranks 1..3) take every third chunk and compute the
//     state-independent part: [Q;K]K^T, A and P, the UT inverse T (blocked
//     16 -> 32 -> 64 on CUDA cores), T' = T diag(b gamma) and T'' = T diag(b) as
//     bf16 hi + lo tiles, W^T = K^T T'^T (tcgen05) and the chunk's decay table.
//     They ship 49 KB per chunk -- -W (the first rows of a K-major [-W;Q]
//     operand), P and T'' (hi + lo) and the table -- from one of two staging
//     blocks into the chain CTA's receive slot with bulk DSMEM copies that
//     complete on the chain CTA's mbarrier, where the chain's own TMA loads of
//     the chunk's Q, K and V also land;
//   the chain CTA (rank 0) walks the chunks in order: U~^T = V^T T''^T goes into
//     the U accumulator ahead of the chunk, then S0 (-W)^T is added to it and
//     S0 Q^T formed (S0 as a bf16 operand in tensor memory), the state update
//     S += (U diag(gamma_L / gamma)) K accumulates in tensor memory after an
//     in-place gamma_L scaling, and the outputs are gamma_t S0 Q^T + U P^T;
//     sixteen epilogue warps share every epilogue (16 tokens or 32 state columns
//     each) and write chunk c's outputs while chunk c + 1's first products run
//     (with the layer's output gate, o * sigmoid(z) before the rounding to bf16,
//     the fp16 factors loaded while the state is rescaled).
// The chain's critical loop hands over between its epilogue warps and the
// MMA-issuing warp through named barriers (no sleeping wake-up on that path);
// tensor-core completions and cross-CTA hand-overs use mbarriers.
//
// Bounded waits: every mbarrier wait gives up after ~2 s of sleeping polls.
// A timeout records GDN_ERR_TIMEOUT, raises an abort flag in all four CTAs,
// and every loop then runs its remaining iterations without work (keeping
// every named barrier matched), after which in-flight loads, copies and MMAs
// are drained (again bounded) before tensor memory is freed.
//
// Precision: exact bf16 q/k/v; T', T'', P, U and U diag(gamma_L/gamma) as bf16
// hi + lo pairs (U~ = T''V is formed from T'' hi + lo with fp32 accumulation);
// gamma_t of the inter-chunk read-out applied in fp32; only S0 and W are single
// bf16.
#include <cuda.h>
#include <cuda_fp16.h>

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
constexpr int kWarps = 17;
constexpr int kThreads = kWarps * 32;
// chain CTA roles: warp 0 issues MMAs, 1..16 epilogue warps (4 per TMEM lane quadrant)
constexpr int kCMma = 0, kCEpi0 = 1, kCNumEpi = 16;
// prep CTA roles: warp 0 loads and issues MMAs, 1..16 workers
constexpr int kPCtl = 0, kPWork0 = 1, kPNumWork = 16, kPWorkThreads = kPNumWork * 32;
constexpr uint32_t kWait = 2000;   // sleeping polls (<= ~1 ms each) before a wait gives up
constexpr uint32_t kDrain = 50;    // polls for a drain of in-flight work after an abort

// named barriers (0 is __syncthreads)
constexpr uint32_t NB_WORK = 1;                       // prep workers
constexpr uint32_t NB_S0 = 1, NB_U = 2, NB_U2 = 3;    // epilogue warps + MMA warp
constexpr uint32_t kChainSync = (kCNumEpi + 1) * 32;

// ---- chain receive slot of one chunk: Q, K, V by TMA, the rest from a prep CTA ----
constexpr uint32_t SL_WQ = 0;       // per 64-column half 16 KB: -W rows (t), then Q rows (t); K-major
constexpr uint32_t SL_K = 32768;    // K as loaded (rows t, two 64-column halves), MN-major B
constexpr uint32_t SL_V = 49152;    // V as loaded (rows t, two 64-column halves), MN-major A
constexpr uint32_t SL_PH = 65536;   // P hi: 64 rows (t) x 64 (s), K-major
constexpr uint32_t SL_PL = 73728;   // P lo
constexpr uint32_t SL_T2H = 81920;  // T'' = T diag(b) hi: 64 rows (t) x 64 (s), K-major
constexpr uint32_t SL_T2L = 90112;  // T'' lo
constexpr uint32_t SL_TAB = 98304;  // fp32: gamma_L/gamma_t [64], gamma_t [64], gamma_L
constexpr uint32_t SLOT = 99328;    // bytes per slot (a multiple of 1024: slots stay swizzle-aligned)
// a prep CTA's staging block (what its bulk copies carry) and where each piece lands
constexpr uint32_t ST_W = 0;        // -W rows, two 64-column halves of 8 KB -> SL_WQ, SL_WQ + 16384
constexpr uint32_t ST_P = 16384;    // P hi, P lo -> SL_PH
constexpr uint32_t ST_T2 = 32768;   // T'' hi, T'' lo -> SL_T2H
constexpr uint32_t ST_TAB = 49152;  // decay table -> SL_TAB
constexpr uint32_t ST_BYTES = 50176;
constexpr uint32_t QKV_BYTES = 6 * 8192;            // Q, K and V tiles loaded by the chain CTA
constexpr uint32_t SLOT_TX = ST_BYTES + QKV_BYTES;  // bytes that complete one receive slot

// ---- chain CTA shared memory ----
constexpr uint32_t C_R = 0;                                 // 2 receive slots
constexpr uint32_t C_OT = C_R + 2 * SLOT;   // per epilogue warp: 16 x 32 bf16 output tile
constexpr uint32_t C_BAR = C_OT + kCNumEpi * 1024;
// ---- prep CTA shared memory ----
// two q/k buffers of 32 KB: [Q half 0 | K half 0][Q half 1 | K half 1]
constexpr uint32_t P_QK = 0, QK_STRIDE = 32768;
constexpr uint32_t P_T = 65536;     // A fp32 [64][A_LD], then T' hi, T' lo (2 x 8 KB)
constexpr uint32_t A_LD = 68;
constexpr uint32_t P_TF = P_T + 64 * A_LD * 4;   // T fp32 [64][T_LD]
constexpr uint32_t T_LD = 68;
constexpr uint32_t P_X = P_TF + 64 * T_LD * 4;
constexpr uint32_t X_LD = 36;
constexpr uint32_t P_PB = P_X + 32 * X_LD * 4;   // beta, gamma, G, 1/|q|, 1/|k|
constexpr uint32_t P_ST = 106496;   // two staging blocks (ST_BYTES each, 1024-aligned)
constexpr uint32_t P_BAR = P_ST + 2 * ST_BYTES;

// CB_Z0 + w: epilogue warp w's gate-logit tile has landed in its output tile (GT)
enum ChainBar { CB_R_FULL0, CB_R_FULL1, CB_U_MMA, CB_DS_FULL, CB_O_FULL, CB_DRAIN, CB_Z0,
                CB_COUNT = CB_Z0 + 16 };
enum PrepBar { PB_LD_FULL0, PB_LD_FULL1, PB_X_DONE, PB_T_READY, PB_W_DONE, PB_EPI_DONE, PB_GO,
               PB_STAGE_FREE0, PB_STAGE_FREE1, PB_DRAIN, PB_COUNT };

// words at the same offset in every CTA: TMEM base, abort flag, slot bookkeeping
constexpr uint32_t AUX_RAW = (C_BAR + CB_COUNT * 8 > P_BAR + PB_COUNT * 8) ? C_BAR + CB_COUNT * 8
                                                                          : P_BAR + PB_COUNT * 8;
constexpr uint32_t AUX = (AUX_RAW + 15) & ~15u;
constexpr uint32_t AUX_TSLOT = AUX, AUX_ABORT = AUX + 4, AUX_ARMED = AUX + 8,
                   AUX_CONSUMED = AUX + 12;
constexpr uint32_t SMEM_BYTES = AUX + 16 + 1024;
static_assert(P_PB + 5 * 64 * 4 <= P_ST, "prep layout");
static_assert(64 * A_LD * 4 >= 16384, "T' tiles fit where A was");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(P_ST % 1024 == 0 && SLOT % 1024 == 0 && ST_BYTES % 1024 == 0 && P_T % 1024 == 0,
              "swizzle alignment");

// ---- TMEM columns ----
// chain: S0 [W;Q]^T (D = S0 W^T, then S0 Q^T), U P^T, S0 (bf16 A operand), S (fp32),
//        U / U diag(gamma_L/gamma) hi and lo (bf16 A operands)
constexpr uint32_t TM_D = 0, TM_Q = 64, TM_O = 128, TM_S0 = 192, TM_S = 256;
constexpr uint32_t TM_UH = 384, TM_UL = 416, TM_BH = 448, TM_BL = 480;
// prep: [Q;K]K^T, then W^T
constexpr uint32_t TP_D1 = 0;

struct ClParams {
    const float *g, *beta, *h0;
    const int32_t *cu;
    int64_t T;
    int HK, HV;
    float scale;
    __nv_bfloat16 *o;
    float *hT;
    unsigned int *status;
    unsigned int prologue;   // GDN_PROLOGUE_* flags
};

struct Waiter {
    uint64_t *bars;
    volatile int *abort_flag;
    unsigned int *status;
    uint32_t abort_saddr;   // shared address of the abort flag (same in every CTA)
    // false once the cluster has aborted: the caller then skips its work
    __device__ bool operator()(int b, uint32_t parity) const {
        if (mbar_test_wait(&bars[b], parity)) return true;   // usually complete already
        if (*abort_flag) return false;
        for (uint32_t i = 0; i < kWait; ++i) {
            if (mbar_try_wait_sleep(&bars[b], parity, 1000000u)) return true;
            if (*abort_flag) return false;
        }
        abort_all();
        return false;
    }
    // teardown: waits (bounded) for in-flight work whether or not the cluster aborted
    __device__ void drain(int b, uint32_t parity) const {
        for (uint32_t i = 0; i < kDrain; ++i)
            if (mbar_try_wait_sleep(&bars[b], parity, 1000000u)) return;
    }
    __device__ void abort_all() const {
        atomicExch(status, (unsigned int)GDN_ERR_TIMEOUT);
        for (uint32_t r = 0; r < (uint32_t)kClusterSize; ++r)
            st_cluster_u32(mapa_shared(abort_saddr, r), 1u);
    }
};

__device__ __forceinline__ void local_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// descriptor of the same operand `bytes` further on (the start-address field holds
// address >> 4; shared addresses stay below 256 KB, so the field cannot overflow)
__device__ __forceinline__ uint64_t desc_add(uint64_t d, uint32_t bytes) { return d + (bytes >> 4); }
// the whole warp agrees (wait results are warp-uniform in practice; this makes it certain)
__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v); }

// ============================================================================ chain CTA
// Q, K and V tiles of chunk c into its receive slot (completing on that slot's mbarrier)
__device__ __forceinline__ void load_qkv_slot(const CUtensorMap *tm_q, const CUtensorMap *tm_k,
                                              const CUtensorMap *tm_v, uint8_t *sm, uint64_t *bars,
                                              int c, int cqk, int h, int64_t bos) {
    const int s = c & 1;
    uint8_t *slot = sm + C_R + s * SLOT;
    uint64_t *bar = &bars[CB_R_FULL0 + s];
    const int s0 = (int)(bos + (int64_t)c * C);
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        tma_load_3d(slot + SL_WQ + hf * 16384 + 8192, tm_q, bar, 64 * hf, cqk, s0);
        tma_load_3d(slot + SL_K + hf * 8192, tm_k, bar, 64 * hf, cqk, s0);
        tma_load_3d(slot + SL_V + hf * 8192, tm_v, bar, 64 * hf, h, s0);
    }
}

// GT: the output gate o <- o * sigmoid(z) is applied in the read-out, before the
// one rounding to bf16, from factors sigmoid(z) precomputed in fp16.  Each
// epilogue warp prefetches its 16 x 32 tile of factors into L2 one chunk ahead,
// TMA-loads it into its output tile while the state is rescaled, and the
// read-out overwrites it in place with the gated outputs.
template <bool GT>
__device__ void chain_cta(const CUtensorMap *tm_q, const CUtensorMap *tm_k, const CUtensorMap *tm_v,
                          const CUtensorMap *tm_o, const CUtensorMap *tm_z, const ClParams &p, uint8_t *sm, uint32_t sb, uint32_t tmem,
                          const Waiter &wt, int h, int n, int64_t bos, int64_t eos, int nchunks) {
    uint64_t *bars = wt.bars;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int HV = p.HV, cqk = h / (HV / p.HK);
    const size_t sbase = ((size_t)n * HV + h) * (size_t)DH * DH;
    volatile int *armed = reinterpret_cast<volatile int *>(sm + AUX_ARMED);
    volatile int *consumed = reinterpret_cast<volatile int *>(sm + AUX_CONSUMED);
    auto chunk_len = [&](int c) {
        const int64_t r = eos - (bos + (int64_t)c * C);
        return (int)(r < C ? r : C);
    };
    if (warp == kCMma) {
        // ------------------------------------------------------------ MMA warp
        const uint32_t id_n64 = idesc_bf16(128, 64, false, false);
        const uint32_t id_wq = idesc_bf16(128, 128, false, false);
        const uint32_t id_s = idesc_bf16(128, 128, false, true);
        const uint32_t id_u = idesc_bf16(128, 64, true, false);
        auto commit = [&](int b) {
            if (elect_one()) mma_commit(&bars[b]);
            __syncwarp();
        };
        // chunk c's receive slot is complete: release the producing prep CTA's
        // staging block, then U~^T = V^T T''^T into the U accumulator (hi + lo), so
        // that chunk c's first product only has to add S0 (-W)^T
        auto take_slot = [&](int c, bool ok_in) -> bool {
            const bool ok = warp_all(ok_in && wt(CB_R_FULL0 + (c & 1), (uint32_t)((c >> 1) & 1)));
            if (!ok) return false;
            const uint32_t slot = sb + C_R + (c & 1) * SLOT;
            if (lane == 0) *consumed = c + 1;
            // the bulk copies out of that staging block have completed
            if (elect_one())
                mbar_arrive_remote_relaxed(mapa_shared(
                    sb + P_BAR + (PB_STAGE_FREE0 + ((c / kNumPrep) & 1)) * 8, 1 + c % kNumPrep));
            __syncwarp();
            tc_fence_after();
            const uint64_t va0 = sdesc_sw128(slot + SL_V, 8192, 1024);
            const uint64_t th0 = sdesc_sw128(slot + SL_T2H, 16, 1024);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                if (elect_one()) {
                    mma_bf16(tmem + TM_D, desc_add(va0, k * 2048), desc_add(th0, k * 32), id_u, k > 0);
                    mma_bf16(tmem + TM_D, desc_add(va0, k * 2048), desc_add(th0, SL_T2L - SL_T2H + k * 32),
                             id_u, 1);
                }
                __syncwarp();
            }
            return true;
        };
        bool ok = nchunks > 0 ? take_slot(0, true) : true;
        for (int c = 0; c < nchunks; ++c) {
            const uint32_t slot = sb + C_R + (c & 1) * SLOT;
            // S0 of chunk c is in tensor memory, and the epilogue warps have read every
            // accumulator of chunk c - 1 that this chunk's MMAs overwrite
            named_sync(NB_S0, kChainSync);
            tc_fence_after();
            if (ok) {
                // [U | S0 Q^T] = [U~ | 0] + S0 [-W;Q]^T in one N = 128 product (A = S0 from
                // TMEM, B K-major from the slot; the epilogue warps zeroed S0 Q^T's columns)
                const uint64_t wq0 = sdesc_sw128(slot + SL_WQ, 16, 1024);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    if (elect_one())
                        mma_bf16_ts(tmem + TM_D, tmem + TM_S0 + 8 * k,
                                    desc_add(wq0, (k >> 2) * 16384 + (k & 3) * 32), id_wq, 1);
                    __syncwarp();
                }
                commit(CB_U_MMA);
            }
            named_sync(NB_U, kChainSync);     // U diag(gamma_L/gamma) (hi, lo) is in TMEM
            tc_fence_after();
            if (ok) {
                // S += (U diag(gamma_L/gamma)) K  (hi + lo; K MN-major from the slot)
                const uint64_t k0 = sdesc_sw128(slot + SL_K, 8192, 1024);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    if (elect_one()) {
                        mma_bf16_ts(tmem + TM_S, tmem + TM_BH + 8 * k, desc_add(k0, k * 2048), id_s, 1);
                        mma_bf16_ts(tmem + TM_S, tmem + TM_BL + 8 * k, desc_add(k0, k * 2048), id_s, 1);
                    }
                    __syncwarp();
                }
                commit(CB_DS_FULL);
            }
            named_sync(NB_U2, kChainSync);    // U (hi, lo) is in TMEM
            tc_fence_after();
            if (ok) {
                // U P^T (hi/lo cross terms)
                const uint64_t p0 = sdesc_sw128(slot + SL_PH, 16, 1024);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint64_t ph_d = desc_add(p0, k * 32), pl_d = desc_add(p0, SL_PL - SL_PH + k * 32);
                    if (elect_one()) {
                        mma_bf16_ts(tmem + TM_O, tmem + TM_UH + 8 * k, ph_d, id_n64, k > 0);
                        mma_bf16_ts(tmem + TM_O, tmem + TM_UH + 8 * k, pl_d, id_n64, 1);
                        mma_bf16_ts(tmem + TM_O, tmem + TM_UL + 8 * k, ph_d, id_n64, 1);
                    }
                    __syncwarp();
                }
                commit(CB_O_FULL);
            }
            // the next chunk's U~ (this chunk's U was read before its second barrier);
            // it runs while this chunk's state update completes
            if (c + 1 < nchunks) ok = take_slot(c + 1, ok);
        }
        // every MMA issued here has completed before tensor memory is released
        commit(CB_DRAIN);
        wt.drain(CB_DRAIN, 0);
    } else {
        // ------------------------------------------------------------ epilogue warps
        // Warp w works on TMEM lane quadrant w % 4 (state rows i) and on part
        // (w - 1) / 4 of the columns: tokens 16 part .. 16 part + 15 of the
        // 64-token products, state columns 32 part .. 32 part + 31.
        const int part = (warp - kCEpi0) >> 2;
        const int i = 32 * (warp & 3) + lane;
        {
            // start state: fp32 (scaled at the start of chunk 0) and its bf16 copy (chunk 0's S0)
            const float *src = p.h0 ? p.h0 + sbase + (size_t)i * DH + 32 * part : nullptr;
            float v[32];
            uint32_t w[16];
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                const float4 v4 = src ? *reinterpret_cast<const float4 *>(src + j)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
                v[j] = v4.x;
                v[j + 1] = v4.y;
                v[j + 2] = v4.z;
                v[j + 3] = v4.w;
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) w[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
            tmem_st16w(tmem_addr(tmem, warp, TM_S0 + 16 * part), w);
            tmem_st32f(tmem_addr(tmem, warp, TM_S + 32 * part), v);
            // chunk 0's S0 Q^T accumulates onto zero
#pragma unroll
            for (int j = 0; j < 16; ++j) w[j] = 0u;
            tmem_st16w(tmem_addr(tmem, warp, TM_Q + 16 * part), w);
            tmem_wait_st();
        }
        tc_fence_before();
        if (nchunks > 0) named_sync(NB_S0, kChainSync);
        bool ok = true;
        float dq[16];            // scale * gamma_t * (S0 q_t) of the previous chunk
        // gate factors of chunk cp for this warp's 16 tokens x 32 value rows, into the
        // warp's output tile once its previous store has been read (tokens past the
        // end of the data read as zero; those of a next sequence are never stored)
        uint32_t zst = 0;   // bit 0: phase of the next gate-logit load; bit 1: one in flight
        auto load_z = [&](int cp) {
            if (lane == 0) {
                uint64_t *zbar = &bars[CB_Z0 + (warp - kCEpi0)];
                bulk_wait_group_read0();
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(zbar, 1024);
                tma_load_3d(sm + C_OT + (warp - kCEpi0) * 1024, tm_z, zbar, 32 * (warp & 3), h,
                            (int)(bos + (int64_t)cp * C + 16 * part));
            }
            __syncwarp();
            zst |= 2u;
        };
        // read-out of chunk cp: o_t = dq + scale (U P^T)_t for this warp's 16 tokens x
        // 32 value rows, put into a per-warp shared tile [t][i] and written by one
        // TMA store of the warp (plain 16-byte stores for tokens of a short last chunk)
        unsigned short *ot = reinterpret_cast<unsigned short *>(sm + C_OT + (warp - kCEpi0) * 1024);
        auto read_out = [&](int cp) -> bool {
            const int64_t ps0 = bos + (int64_t)cp * C;
            const int pL = chunk_len(cp);
            float dout[16];
            tmem_ld16(tmem_addr(tmem, warp, TM_O + 16 * part), dout);
            // the tile's previous store has been read out of shared memory
            if (lane == 0) bulk_wait_group_read0();
            __syncwarp();
            if (GT) {
                // the gate factors are in the tile
                const bool zok = warp_all(wt(CB_Z0 + (warp - kCEpi0), zst & 1u));
                if (zok) zst = (zst & 1u) ^ 1u;
                tmem_wait_ld();
                if (!zok) return false;
            }
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                float out = fmaf(p.scale, dout[j], dq[j]);
                if (GT) out *= __half2float(__ushort_as_half(ot[j * 32 + lane]));
                const __nv_bfloat16 b = __float2bfloat16_rn(out);
                ot[j * 32 + lane] = *reinterpret_cast<const unsigned short *>(&b);
            }
            if (16 * part + 16 <= pL) {
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_3d(tm_o, ot, 32 * (warp & 3), h, (int)(ps0 + 16 * part));
                    bulk_commit_group();
                }
            } else {
                __syncwarp();
#pragma unroll
                for (int pass = 0; pass < 2; ++pass) {
                    const int t = 8 * pass + (lane >> 2), c4 = lane & 3;
                    const uint4 val = *reinterpret_cast<const uint4 *>(ot + t * 32 + c4 * 8);
                    if (16 * part + t < pL)
                        *reinterpret_cast<uint4 *>(p.o + ((size_t)(ps0 + 16 * part + t) * HV + h) * DH +
                                                   32 * (warp & 3) + 8 * c4) = val;
                }
            }
            __syncwarp();
            return true;
        };
        for (int c = 0; c < nchunks; ++c) {
            const uint32_t ph = (uint32_t)(c & 1);
            const int s = c & 1;
            const int L = chunk_len(c);
            const uint8_t *slot = sm + C_R + s * SLOT;
            const float *tab = reinterpret_cast<const float *>(slot + SL_TAB);
            if (GT) {
                // this chunk's gate factors towards L2 a period ahead of their load, and
                // the previous chunk's into the output tile (an L2 hit by now), in
                // flight while the state is rescaled
                if (lane == 0)
                    tma_prefetch_l2_3d(tm_z, 32 * (warp & 3), h, (int)(bos + (int64_t)c * C + 16 * part));
                if (c > 0 && ok) load_z(c - 1);
            }
            ok = warp_all(ok && wt(CB_R_FULL0 + s, (uint32_t)((c >> 1) & 1)));
            if (ok) {
                // scale the fp32 state by this chunk's gamma_L before its update
                const float gL = tab[128];
                float v[32];
                tmem_ld32(tmem_addr(tmem, warp, TM_S + 32 * part), v);
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] *= gL;
                tmem_st32f(tmem_addr(tmem, warp, TM_S + 32 * part), v);
            }
            if (c > 0) {
                // the previous chunk's U P^T is done: every read of its receive slot is
                // over, so re-arm that slot and release the prep CTA that produces chunk
                // c + 1 into it; then write the previous chunk's outputs (its
                // accumulator is overwritten only after this chunk's second barrier)
                ok = warp_all(ok && wt(CB_O_FULL, (uint32_t)((c - 1) & 1)));
                if (ok) {
                    tc_fence_after();
                    if (warp == kCEpi0 && c + 1 < nchunks) {
                        if (lane == 0) {
                            mbar_arrive_expect_tx(&bars[CB_R_FULL0 + ((c + 1) & 1)], SLOT_TX);
                            *armed = c + 2;
                            load_qkv_slot(tm_q, tm_k, tm_v, sm, bars, c + 1, cqk, h, bos);
                            mbar_arrive_remote_relaxed(
                                mapa_shared(sb + P_BAR + PB_GO * 8, 1 + (c + 1) % kNumPrep));
                        }
                        __syncwarp();
                    }
                    ok = read_out(c - 1);
                }
            }
            ok = warp_all(ok && wt(CB_U_MMA, ph));
            float u[16];
            if (ok) {
                tc_fence_after();
                // U = U~ - S0 W^T for tokens t = 16 part + j of row i (formed by the MMAs)
                tmem_ld16(tmem_addr(tmem, warp, TM_D + 16 * part), u);
                tmem_wait_ld();
                if (L < C) {   // tokens past the sequence end (short last chunk)
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (16 * part + j >= L) u[j] = 0.f;
                }
                // U diag(gamma_L/gamma) as hi + lo words
                uint32_t whi[8], wlo[8];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const float4 f = *reinterpret_cast<const float4 *>(tab + 16 * part + 4 * q4);
                    const float b0 = u[4 * q4] * f.x, b1 = u[4 * q4 + 1] * f.y;
                    const float b2 = u[4 * q4 + 2] * f.z, b3 = u[4 * q4 + 3] * f.w;
                    const __nv_bfloat162 h01 = __floats2bfloat162_rn(b0, b1);
                    const __nv_bfloat162 h23 = __floats2bfloat162_rn(b2, b3);
                    const float2 f01 = __bfloat1622float2(h01), f23 = __bfloat1622float2(h23);
                    whi[2 * q4] = *reinterpret_cast<const uint32_t *>(&h01);
                    whi[2 * q4 + 1] = *reinterpret_cast<const uint32_t *>(&h23);
                    wlo[2 * q4] = pack_bf16x2(b0 - f01.x, b1 - f01.y);
                    wlo[2 * q4 + 1] = pack_bf16x2(b2 - f23.x, b3 - f23.y);
                }
                tmem_st8w(tmem_addr(tmem, warp, TM_BH + 8 * part), whi);
                tmem_st8w(tmem_addr(tmem, warp, TM_BL + 8 * part), wlo);
            }
            // (the wait also covers the gamma_L-scaled state)
            tmem_wait_st();
            tc_fence_before();
            named_sync(NB_U, kChainSync);     // the state update can start
            if (ok) {
                uint32_t whi[8], wlo[8];
#pragma unroll
                for (int w = 0; w < 8; ++w) {
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(u[2 * w], u[2 * w + 1]);
                    const float2 hf = __bfloat1622float2(h2);
                    whi[w] = *reinterpret_cast<const uint32_t *>(&h2);
                    wlo[w] = pack_bf16x2(u[2 * w] - hf.x, u[2 * w + 1] - hf.y);
                }
                tmem_st8w(tmem_addr(tmem, warp, TM_UH + 8 * part), whi);
                tmem_st8w(tmem_addr(tmem, warp, TM_UL + 8 * part), wlo);
                tmem_wait_st();
            }
            tc_fence_before();
            named_sync(NB_U2, kChainSync);    // U P^T can start
            const bool more = c + 1 < nchunks;
            ok = warp_all(ok && wt(CB_DS_FULL, ph));
            if (ok) {
                tc_fence_after();
                if (more) {
                    // new state -> bf16 copy in TMEM: the next chunk's S0
                    float v[32];
                    uint32_t w[16];
                    tmem_ld32(tmem_addr(tmem, warp, TM_S + 32 * part), v);
#pragma unroll
                    for (int j = 0; j < 16; ++j) w[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
                    tmem_st16w(tmem_addr(tmem, warp, TM_S0 + 16 * part), w);
                }
                // scale * gamma_t * S0 q_t of this part's tokens, read before the next
                // chunk's MMAs overwrite it (gamma_t from the slot, still held); the
                // columns are zeroed for the next chunk's accumulation
                tmem_ld16(tmem_addr(tmem, warp, TM_Q + 16 * part), dq);
                tmem_wait_ld();
                if (more) {
                    uint32_t z[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) z[j] = 0u;
                    tmem_st16w(tmem_addr(tmem, warp, TM_Q + 16 * part), z);
                }
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const float4 g4 = *reinterpret_cast<const float4 *>(tab + 64 + 16 * part + 4 * q4);
                    dq[4 * q4] *= p.scale * g4.x;
                    dq[4 * q4 + 1] *= p.scale * g4.y;
                    dq[4 * q4 + 2] *= p.scale * g4.z;
                    dq[4 * q4 + 3] *= p.scale * g4.w;
                }
                tmem_wait_st();
            }
            tc_fence_before();
            if (more) named_sync(NB_S0, kChainSync);
        }
        if (nchunks > 0) {
            if (GT && ok) load_z(nchunks - 1);
            ok = warp_all(ok && wt(CB_O_FULL, (uint32_t)((nchunks - 1) & 1)));
            if (ok) {
                tc_fence_after();
                ok = read_out(nchunks - 1);
            }
        }
        // a gate-logit load still in flight (after an abort) lands before the
        // CTA's shared memory is released, and so do this warp's tile stores
        if (GT && (zst & 2u)) wt.drain(CB_Z0 + (warp - kCEpi0), zst & 1u);
        if (lane == 0) bulk_wait_group0();
        __syncwarp();
        if (ok && p.hT) {
            tc_fence_after();
            float v[32];
            tmem_ld32(tmem_addr(tmem, warp, TM_S + 32 * part), v);
            float *dst = p.hT + sbase + (size_t)i * DH + 32 * part;
#pragma unroll
            for (int j = 0; j < 32; j += 4)
                *reinterpret_cast<float4 *>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
        }
    }
}

// ============================================================================ prep CTA
template <bool PRO>
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
        int issued = 0, landed = 0;    // q/k loads issued / waited for (k-th into buffer k & 1)
        auto load = [&](int k) {
            if (lane == 0) {
                const int s0 = (int)(bos + (int64_t)chunk_of(k) * C);
                uint64_t *bar = &bars[PB_LD_FULL0 + (k & 1)];
                uint8_t *buf = sm + P_QK + (k & 1) * QK_STRIDE;
                mbar_arrive_expect_tx(bar, 4 * 8192);
                tma_load_3d(buf, tm_q, bar, 0, cqk, s0);
                tma_load_3d(buf + 16384, tm_q, bar, 64, cqk, s0);
                tma_load_3d(buf + 8192, tm_k, bar, 0, cqk, s0);
                tma_load_3d(buf + 24576, tm_k, bar, 64, cqk, s0);
            }
            __syncwarp();
            ++issued;
        };
        if (nk > 0) {
            if (lane == 0) {
                tma_prefetch_desc(tm_q);
                tma_prefetch_desc(tm_k);
            }
            load(0);
        }
        for (int k = 0; k < nk; ++k) {
            const int c = chunk_of(k);
            const uint32_t ph = (uint32_t)(k & 1);
            const uint32_t qkv = sb + P_QK + (k & 1) * QK_STRIDE;
            if (!warp_all(wt(PB_LD_FULL0 + (k & 1), (uint32_t)((k >> 1) & 1)))) break;
            ++landed;
            // the other buffer's chunk (k - 1) finished its W product: load chunk k + 1
            if (k + 1 < nk) load(k + 1);
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                const uint64_t a = sdesc_sw128(qkv + off, 16, 1024);
                const uint64_t b = sdesc_sw128(qkv + 8192 + off, 16, 1024);
                if (elect_one()) mma_bf16(tmem + TP_D1, a, b, id_x, kk > 0);
                __syncwarp();
            }
            commit(PB_X_DONE);
            if (!warp_all(wt(PB_T_READY, ph))) break;
            tc_fence_after();
            // W^T = K^T T'^T (T' = T diag(b gamma) as hi + lo)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ka = sdesc_sw128(qkv + 8192 + kk * 2048, 16384, 1024);
                const uint64_t t1h = sdesc_sw128(sb + P_T + kk * 32, 16, 1024);
                const uint64_t t1l = sdesc_sw128(sb + P_T + 8192 + kk * 32, 16, 1024);
                if (elect_one()) {
                    mma_bf16(tmem + TP_D1, ka, t1h, id_w, kk > 0);
                    mma_bf16(tmem + TP_D1, ka, t1l, id_w, 1);
                }
                __syncwarp();
            }
            commit(PB_W_DONE);
            if (!warp_all(wt(PB_W_DONE, ph))) break;   // this buffer's q/k tiles are free again
            if (!warp_all(wt(PB_EPI_DONE, ph))) break;
            if (c >= 2) {
                const int j = first >= 2 ? k : k - 1;   // go arrivals before this chunk
                if (!warp_all(wt(PB_GO, (uint32_t)(j & 1)))) break;
            }
            if (elect_one()) {
                const int s = c & 1;
                const uint32_t mbar = mapa_shared(sb + C_BAR + (CB_R_FULL0 + s) * 8, 0);
                const uint32_t dst = mapa_shared(sb + C_R + s * SLOT, 0);
                const uint32_t st = sb + P_ST + (k & 1) * ST_BYTES;
                bulk_copy_to_cluster(dst + SL_WQ, st + ST_W, 8192, mbar);
                bulk_copy_to_cluster(dst + SL_WQ + 16384, st + ST_W + 8192, 8192, mbar);
                bulk_copy_to_cluster(dst + SL_PH, st + ST_P, 16384, mbar);
                bulk_copy_to_cluster(dst + SL_T2H, st + ST_T2, 16384, mbar);
                bulk_copy_to_cluster(dst + SL_TAB, st + ST_TAB, ST_BYTES - ST_TAB, mbar);
            }
            __syncwarp();
        }
        // after an abort: a load still in flight lands, and issued MMAs complete,
        // before this CTA's shared and tensor memory are released
        for (int d = landed; d < issued; ++d) wt.drain(PB_LD_FULL0 + (d & 1), (uint32_t)((d >> 1) & 1));
        commit(PB_DRAIN);
        wt.drain(PB_DRAIN, 0);
    } else if (warp < kPWork0 + kPNumWork) {
        // ------------------------------------------------------------ prep workers
        const int pt = tid - 32 * kPWork0;                 // 0..511
        const int r = 32 * (warp & 3) + lane;              // TMEM lane of this thread
        const int qtr = (warp - kPWork0) >> 2;             // column quarter (16 columns)
        float *beta_s = reinterpret_cast<float *>(sm + P_PB);
        float *gam_p = beta_s + 64;
        float *G_p = gam_p + 64;
        // input prologue: 1/|q_t|, 1/|k_t| (L2-normalised rows), folded into the
        // diagonal scalings below; 1 throughout without it
        float *rq_p = G_p + 64;
        float *rk_p = rq_p + 64;
        const unsigned pro = PRO ? p.prologue : 0u;   // compiled out without the prologue
        const bool norm_qk = PRO && (pro & (GDN_PROLOGUE_NORM_Q | GDN_PROLOGUE_NORM_K)) != 0;
        const bool logits = PRO && (pro & GDN_PROLOGUE_GATE_LOGITS) != 0;
        if (PRO && !norm_qk && pt < 128) (pt < 64 ? rq_p : rk_p)[pt & 63] = 1.f;
        // 1/|q_t|, 1/|k_t| where the prologue normalises, else exactly 1
        auto rq = [&](int t) { return PRO ? rq_p[t] : 1.f; };
        auto rk = [&](int t) { return PRO ? rk_p[t] : 1.f; };
        float *A_s = reinterpret_cast<float *>(sm + P_T);
        float *T_s = reinterpret_cast<float *>(sm + P_TF);
        float *X_s = reinterpret_cast<float *>(sm + P_X);
        bool ok = true;
        for (int k = 0; k < nk; ++k) {
            const int c = chunk_of(k);
            const uint32_t ph = (uint32_t)(k & 1);
            const int64_t s0 = bos + (int64_t)c * C;
            const int L = chunk_len(c);
            const uint32_t stb = P_ST + (k & 1) * ST_BYTES;   // this chunk's staging block
            named_sync(NB_WORK, kPWorkThreads);
            if (warp == kPWork0) {
                float2 gp = load_g_pair(p.g, s0, L, HV, h);
                if (logits) {   // g = log sigmoid(a) for the tokens of the chunk
                    if (2 * lane < L) gp.x = gate_log_sigmoid(gp.x);
                    if (2 * lane + 1 < L) gp.y = gate_log_sigmoid(gp.y);
                }
                const float2 Gv = warp_decay_scan(gp.x, gp.y);
                G_p[2 * lane] = Gv.x;
                G_p[2 * lane + 1] = Gv.y;
                gam_p[2 * lane] = expf(Gv.x);
                gam_p[2 * lane + 1] = expf(Gv.y);
            } else if (warp == kPWork0 + 1) {
                float2 bp = load_g_pair(p.beta, s0, L, HV, h);
                if (logits) {   // beta = sigmoid(b)
                    if (2 * lane < L) bp.x = gate_sigmoid(bp.x);
                    if (2 * lane + 1 < L) bp.y = gate_sigmoid(bp.y);
                }
                beta_s[2 * lane] = bp.x;
                beta_s[2 * lane + 1] = bp.y;
            }
            // the X product is done and this staging block's previous contents (chunk
            // k - 2 of this CTA) have been copied out
            ok = warp_all(ok && wt(PB_X_DONE, ph) &&
                          (k < 2 || wt(PB_STAGE_FREE0 + (k & 1), (uint32_t)(((k >> 1) - 1) & 1))));
            if (norm_qk) {
                // squared norms of the 64 q and 64 k rows of the landed tiles: four
                // threads per row, 64 bytes each (the 128B swizzle only permutes the
                // 16-byte pieces inside a row)
                ok = warp_all(ok && wt(PB_LD_FULL0 + (k & 1), (uint32_t)((k >> 1) & 1)));
                if (ok) {
                    const int qr = pt >> 2, part = pt & 3;
                    const bool isk = qr >= 64;
                    const int t = qr & 63;
                    const uint8_t *rp = sm + P_QK + (k & 1) * QK_STRIDE + (part >> 1) * 16384 +
                                        (isk ? 8192 : 0) + t * 128 + (part & 1) * 64;
                    float ss = 0.f;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint4 w = *reinterpret_cast<const uint4 *>(rp + 16 * i);
                        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f = __bfloat1622float2(
                                *reinterpret_cast<const __nv_bfloat162 *>(&ws[e]));
                            ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
                        }
                    }
                    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
                    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
                    if (part == 0) {
                        const bool on = (pro & (isk ? GDN_PROLOGUE_NORM_K : GDN_PROLOGUE_NORM_Q)) != 0;
                        (isk ? rk_p : rq_p)[t] = t < L ? (on ? inv_l2norm(ss) : 1.f) : 0.f;
                    }
                }
            }
            named_sync(NB_WORK, kPWorkThreads);
            if (ok) {
                tc_fence_after();
                // P rows (r < 64) into the staging block, A rows (r >= 64) into A
                float v[16];
                tmem_ld16(tmem_addr(tmem, warp, TP_D1 + 16 * qtr), v);
                tmem_wait_ld();
                const int row = r & 63;
                const int row0 = 32 * ((warp & 3) & 1);          // first row of this warp
                const bool all_masked = 16 * qtr > row0 + 31;    // every column > every row
                const float Gi = G_p[row];
                const float ri = r < 64 ? rq(row) : rk(row);
                if (r < 64) {
                    if (all_masked) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) v[j] = 0.f;
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int col = 16 * qtr + j;
                            v[j] = (col <= row) ? __expf(Gi - G_p[col]) * (ri * rk(col)) * v[j]
                                                : 0.f;
                        }
                    }
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        const uint32_t off = sw128_chunk(row, 2 * qtr + cc);
                        st_chunk_hilo(sb + stb + ST_P + off, sb + stb + ST_P + 8192 + off, v + 8 * cc);
                    }
                } else {
                    const float bi = beta_s[row] * ri;
                    if (all_masked) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) v[j] = 0.f;
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int col = 16 * qtr + j;
                            v[j] = (col < row) ? bi * __expf(Gi - G_p[col]) * rk(col) * v[j]
                                               : 0.f;
                        }
                    }
                    float4 *dst = reinterpret_cast<float4 *>(A_s + row * A_LD + 16 * qtr);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                }
                // decay table of this chunk for the chain CTA
                if (pt < 64) {
                    float *tb = reinterpret_cast<float *>(sm + stb + ST_TAB);
                    tb[pt] = __expf(G_p[63] - G_p[pt]) * rk(pt);   // gamma_L / gamma_t / |k_t|
                    tb[64 + pt] = gam_p[pt] * rq(pt);              // gamma_t / |q_t|
                    if (pt == 0) tb[128] = gam_p[63];      // gamma_L
                }
            }
            tc_fence_before();
            named_sync(NB_WORK, kPWorkThreads);
            // ---- UT inverse, step 1: 16x16 diagonal blocks (threads 0..63) ----
            if (ok && pt < 64) {
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
            named_sync(NB_WORK, kPWorkThreads);
            // ---- step 2: within each 32x32 half, T10 = -T11 A10 T00 (one entry per thread) ----
            const int hf2 = pt >> 8, ii2 = (pt >> 4) & 15, j2 = pt & 15;
            const int r1 = 32 * hf2 + 16, c0 = 32 * hf2;
            if (ok) {
                float a0 = 0.f;
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    const float t0 = (m >= j2) ? T_s[(c0 + m) * T_LD + c0 + j2] : 0.f;
                    a0 = fmaf(A_s[(r1 + ii2) * A_LD + c0 + m], t0, a0);
                }
                X_s[(16 * hf2 + ii2) * X_LD + j2] = a0;
            }
            named_sync(NB_WORK, kPWorkThreads);
            if (ok) {
                float a0 = 0.f;
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    const float tm = (m <= ii2) ? T_s[(r1 + ii2) * T_LD + r1 + m] : 0.f;
                    a0 = fmaf(tm, X_s[(16 * hf2 + m) * X_LD + j2], a0);
                }
                T_s[(r1 + ii2) * T_LD + c0 + j2] = -a0;
            }
            named_sync(NB_WORK, kPWorkThreads);
            // ---- step 3: T[32:64][0:32] = -T22 A21 T11 (two entries per thread) ----
            const int ii3 = pt >> 4, j3 = (pt & 15) * 2;
            if (ok) {
                float a0 = 0.f, a1 = 0.f;
#pragma unroll 8
                for (int m = 0; m < 32; ++m) {
                    const float am = A_s[(32 + ii3) * A_LD + m];
                    const float2 tv = *reinterpret_cast<const float2 *>(T_s + m * T_LD + j3);
                    a0 = fmaf(am, (m >= j3) ? tv.x : 0.f, a0);
                    a1 = fmaf(am, (m >= j3 + 1) ? tv.y : 0.f, a1);
                }
                *reinterpret_cast<float2 *>(X_s + ii3 * X_LD + j3) = make_float2(a0, a1);
            }
            named_sync(NB_WORK, kPWorkThreads);
            if (ok) {
                float a0 = 0.f, a1 = 0.f;
#pragma unroll 8
                for (int m = 0; m < 32; ++m) {
                    const float tm = (m <= ii3) ? T_s[(32 + ii3) * T_LD + 32 + m] : 0.f;
                    const float2 xv = *reinterpret_cast<const float2 *>(X_s + m * X_LD + j3);
                    a0 = fmaf(tm, xv.x, a0);
                    a1 = fmaf(tm, xv.y, a1);
                }
                *reinterpret_cast<float2 *>(T_s + (32 + ii3) * T_LD + j3) = make_float2(-a0, -a1);
            }
            named_sync(NB_WORK, kPWorkThreads);
            // ---- T' = T diag(b gamma) (for W) and T'' = T diag(b) (shipped) as hi/lo bf16
            //      tiles; A is dead ----
            if (ok) {
                const int t = pt >> 3, chunk16 = pt & 7;
                float a1[8], a2[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int s = 8 * chunk16 + e;
                    const float tv = (s <= t) ? T_s[t * T_LD + s] : 0.f;
                    a2[e] = tv * beta_s[s];
                    a1[e] = a2[e] * gam_p[s] * rk(s);
                }
                const uint32_t off = sw128_chunk(t, chunk16);
                st_chunk_hilo(sb + P_T + off, sb + P_T + 8192 + off, a1);
                st_chunk_hilo(sb + stb + ST_T2 + off, sb + stb + ST_T2 + 8192 + off, a2);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) local_arrive(&bars[PB_T_READY]);
            // ---- -W epilogue into the staging block ----
            ok = warp_all(ok && wt(PB_W_DONE, ph));
            named_sync(NB_WORK, kPWorkThreads);
            if (ok) {
                tc_fence_after();
                float v[16];
                // W^T row a = r, tokens t = 16 qtr + j -> -W rows of the K-major [-W;Q] operand
                tmem_ld16(tmem_addr(tmem, warp, TP_D1 + 16 * qtr), v);
                tmem_wait_ld();
                uint8_t *wq = sm + stb + ST_W + (r >> 6) * 8192 + (r & 7) * 2;
                const uint32_t wc = (uint32_t)((r & 63) >> 3);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int t = 16 * qtr + j;
                    *reinterpret_cast<__nv_bfloat16 *>(wq + t * 128 + ((wc ^ (uint32_t)(t & 7)) << 4)) =
                        __float2bfloat16_rn(-v[j]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) local_arrive(&bars[PB_EPI_DONE]);
        }
    }
}

template <bool PRO, bool GT>
__global__ void __launch_bounds__(kThreads, 1)
prefill_cluster_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_o,
                       const __grid_constant__ CUtensorMap tm_z, const ClParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    const int rank = (int)cluster_ctarank();
    const int h = blockIdx.x / kClusterSize, n = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + (rank == 0 ? C_BAR : P_BAR));
    const int nbars = rank == 0 ? CB_COUNT : PB_COUNT;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + AUX_TSLOT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + AUX_ABORT);
    const Waiter wt{bars, abort_flag, p.status, sb + AUX_ABORT};
    int64_t bos, eos;
    if (p.cu) {
        bos = p.cu[n];
        eos = p.cu[n + 1];
    } else {
        bos = (int64_t)n * p.T;
        eos = bos + p.T;
    }
    const int nchunks = (int)((eos - bos + C - 1) / C);
    const uint32_t ncols = rank == 0 ? 512u : 64u;

    if (tid == 0) {
        for (int b = 0; b < nbars; ++b) {
            uint32_t cnt = 1;
            if (rank != 0 && (b == PB_T_READY || b == PB_EPI_DONE)) cnt = kPNumWork;
            mbar_init(&bars[b], cnt);
        }
        *abort_flag = 0;
        if (rank == 0) {
            // receive slots for chunks 0 and 1 expect their bytes from the start
            const int pre = nchunks < 2 ? nchunks : 2;
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            for (int c = 0; c < pre; ++c) {
                mbar_arrive_expect_tx(&bars[CB_R_FULL0 + c], SLOT_TX);
                load_qkv_slot(&tm_q, &tm_k, &tm_v, sm, bars, c, h / (p.HV / p.HK), h, bos);
            }
            *reinterpret_cast<volatile int *>(sm + AUX_ARMED) = pre;
            *reinterpret_cast<volatile int *>(sm + AUX_CONSUMED) = 0;
        }
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(tslot, ncols);
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    cluster_sync_all();   // every CTA's barriers are initialised before any remote traffic

    if (rank == 0)
        chain_cta<GT>(&tm_q, &tm_k, &tm_v, &tm_o, &tm_z, p, sm, sb, tmem, wt, h, n, bos, eos, nchunks);
    else
        prep_cta<PRO>(&tm_q, &tm_k, &tm_v, p, sm, sb, tmem, wt, h, bos, eos, nchunks, rank);

    tc_fence_before();
    __syncthreads();
    if (rank == 0 && tid == 0) {
        // after an abort: bulk copies already issued into the receive slots land
        // before this CTA's shared memory is released
        const int armed = *reinterpret_cast<volatile int *>(sm + AUX_ARMED);
        for (int d = *reinterpret_cast<volatile int *>(sm + AUX_CONSUMED); d < armed; ++d)
            wt.drain(CB_R_FULL0 + (d & 1), (uint32_t)((d >> 1) & 1));
    }
    if (warp == 0) tmem_dealloc(tmem, ncols);
    cluster_sync_all();   // no CTA leaves while another may still address its shared memory
}

}  // namespace

bool prefill_cluster_supported(int dk, int dv, int chunk, gdn_dtype dtype) {
    return dtype == GDN_BF16 && dk == DH && dv == DH && chunk == C;
}

size_t prefill_cluster_workspace(int, int64_t, int, int, bool) { return 256; }

cudaError_t launch_prefill_cluster(const PrefillArgs &a, cudaStream_t stream) {
    const int64_t Ttot = a.cu_seqlens ? a.T : (int64_t)a.N * a.T;
    if (Ttot >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    unsigned int *status = static_cast<unsigned int *>(a.workspace);
    cudaError_t err = a.keep_status ? cudaSuccess : cudaMemsetAsync(status, 0, sizeof(unsigned int), stream);
    if (err != cudaSuccess) return err;
    CUtensorMap tq, tk, tv, to;
    const uint64_t tok = (uint64_t)(Ttot > 0 ? Ttot : 1);
    uint64_t dq[3] = {(uint64_t)DH, (uint64_t)a.HK, tok};
    uint64_t sq[2] = {(uint64_t)DH * 2, (uint64_t)a.HK * DH * 2};
    uint64_t dv[3] = {(uint64_t)DH, (uint64_t)a.HV, tok};
    uint64_t sv[2] = {(uint64_t)DH * 2, (uint64_t)a.HV * DH * 2};
    uint32_t box[3] = {64, 1, 64};
    if (!encode_bf16_map(&tq, a.q, 3, dq, sq, box) || !encode_bf16_map(&tk, a.k, 3, dq, sq, box) ||
        !encode_bf16_map(&tv, a.v, 3, dv, sv, box))
        return cudaErrorInvalidValue;
    // o: one warp's 16 tokens x 32 value rows per store, unswizzled 64-byte rows
    uint32_t obox[3] = {32, 1, 16};
    if (!encode_bf16_map(&to, a.o, 3, dv, sv, obox, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    // gate factors (fp16, o's layout; copied raw, so the 2-byte map type serves):
    // the same 16 x 32 tiles, loaded into the output tiles
    CUtensorMap tz = to;
    if (a.gate && !encode_bf16_map(&tz, a.gate, 3, dv, sv, obox, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    auto kern = a.gate ? (a.prologue ? prefill_cluster_kernel<true, true> : prefill_cluster_kernel<false, true>)
                    : (a.prologue ? prefill_cluster_kernel<true, false> : prefill_cluster_kernel<false, false>);
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)SMEM_BYTES);
    if (err != cudaSuccess) return err;
    ClParams prm{a.g, a.beta, a.h0, a.cu_seqlens, a.T, a.HK, a.HV, a.scale,
                 static_cast<__nv_bfloat16 *>(a.o), a.hT, status, a.prologue};
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
    err = cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, to, tz, prm);
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
}

}  // namespace gdn
