// Chunkwise prefill of the gated delta rule (bf16 q/k/v, head dim 128, chunk
// 64, fp32 state and accumulation) on a thread-block cluster per (sequence,
// value head): one chain CTA and three prep CTAs, the prep results handed over
// through a small ring of chunk records in the workspace (L2-resident).
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
// Prep CTAs (cluster ranks 1..3) take every third chunk and do all the work
// that does not depend on the state: [Q;K]K^T on tcgen05, the masked A and P,
// the UT inverse (blocked 16 -> 32 -> 64 on CUDA cores), W^T = K^T T'^T and
// U~^T = V^T T''^T on tcgen05 (T' = T diag(b gamma), T'' = T diag(b) as bf16
// hi + lo), and the chunk's decay table.  Each chunk becomes one record of the
// chain's ring in global memory: -W (bf16, the rows of a K-major operand), P
// (bf16 hi + lo), the table, and U~ (fp32, token-major).  The record is
// published with a release arrive on the chain CTA's ring barrier; the chain
// CTA's MMA warp hands the ring slot back once the record has landed in its
// shared memory.
//
// The chain CTA walks the chunks in order, with the warps split by role so that
// the work on the state's dependency chain never waits behind the outputs:
//   warp 0 issues the MMAs (one elected lane): U' = S0 (-W)^T (S0 as one bf16
//     operand in tensor memory), S0 Q^T (S0 as bf16 hi + lo), the state update
//     S += (U diag(gamma_L/gamma)) K (hi + lo) into the fp32 state in tensor
//     memory, and U P^T (hi/lo cross terms) into the columns S0 Q^T held;
//   warp 1 loads each chunk into one of two shared-memory slots: the record by
//     bulk copies, Q and K by TMA (no multicast anywhere);
//   warps 2..9 (the critical epilogue) rescale the state by gamma_L, form
//     U = U~ + U' and its bf16 hi/lo copies U diag(gamma_L/gamma) and U, and
//     copy the new state into the bf16 hi/lo operands of the next chunk;
//   warps 10..17 (the output epilogue) take scale * gamma_t (S0 q_t) out of
//     tensor memory as soon as it is formed, then add scale * (U P^T) and write
//     o by TMA stores (with the layer's output gate, o * sigmoid(z) before the
//     one rounding to bf16, from fp16 factors loaded beside the outputs).
//
// Bounded waits: every mbarrier wait gives up after ~2 s of sleeping polls; a
// timeout records GDN_ERR_TIMEOUT, raises an abort flag in all four CTAs, and
// every loop then runs its remaining iterations without work (keeping every
// named barrier matched), after which in-flight loads, copies, stores and MMAs
// are drained (again bounded) before tensor memory is freed.
//
// Precision: exact bf16 q/k/v; T', T'', P, U and U diag(gamma_L/gamma) as bf16
// hi + lo pairs, U~ accumulated in fp32 and handed over in fp32, S0 as bf16
// hi + lo in the read-out S0 Q^T; gamma_t of the read-out applied in fp32.  Only
// W and the S0 operand of U = U~ - W S0^T enter as single bf16.
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
constexpr int kRing = 6;            // ring records per chain (two per prep CTA)
// chain CTA roles
constexpr int kCMma = 0, kCLoad = 1, kCE0 = 2, kCNumCE = 8, kOE0 = kCE0 + kCNumCE, kCNumOE = 8;
constexpr int kWarps = kOE0 + kCNumOE;   // 18
constexpr int kThreads = kWarps * 32;
// prep CTA roles: warp 0 loads and issues MMAs, 1..16 workers, 17 idle
constexpr int kPCtl = 0, kPWork0 = 1, kPNumWork = 16, kPWorkThreads = kPNumWork * 32;

// named barriers (0 is __syncthreads)
constexpr uint32_t NB_WORK = 1;                 // prep workers
constexpr uint32_t NB_S0 = 1, NB_UD = 2;        // chain: MMA warp + critical epilogue warps
constexpr uint32_t kChainSync = (1 + kCNumCE) * 32;

// ---- ring record of one chunk (global memory, 16-byte aligned pieces) ----
constexpr uint32_t RS_W = 0;         // -W rows (t), K-major, two 64-column halves of 8 KB
constexpr uint32_t RS_P = 16384;     // P hi, P lo: 64 rows (t) x 64 (s), K-major
constexpr uint32_t RS_TAB = 32768;   // fp32: gamma_L/gamma_t [64], gamma_t [64], gamma_L
constexpr uint32_t RS_U = 33792;     // U~ fp32, [value row][token], rows UT_LD floats apart
constexpr uint32_t UT_LD = 68;       // (a padded pitch: 16-byte row reads are conflict-free)
// the parts staged in the prep CTA's shared memory (P and U~ go to the record directly)
constexpr uint32_t ST_W = 0, ST_TAB = 16384, ST_BYTES = 17408;
constexpr uint32_t RSLOT = RS_U + DH * UT_LD * 4;   // 68608
constexpr size_t kRingHeader = 256;  // status word (and padding) before the rings

// ---- chain receive slot of one chunk ----
constexpr uint32_t SL_WQ = 0;       // per 64-column half 16 KB: -W rows (t), then Q rows; K-major
constexpr uint32_t SL_K = 32768;    // K as loaded (rows t, two 64-column halves), MN-major B
constexpr uint32_t SL_P = 49152;    // P hi, P lo
constexpr uint32_t SL_TAB = 65536;  // decay table
constexpr uint32_t SL_U = 66560;    // U~ fp32 [i][t] (pitch UT_LD)
constexpr uint32_t SLOT = SL_U + DH * UT_LD * 4;   // 101376 (a multiple of 1024)

// ---- chain CTA shared memory ----
constexpr uint32_t C_R = 0;                       // 2 receive slots
constexpr uint32_t C_OT = C_R + 2 * SLOT;         // per output warp: 32 x 32 bf16 tile
constexpr uint32_t C_BAR = C_OT + kCNumOE * 2048;
// ---- prep CTA shared memory ----
constexpr uint32_t P_QK = 0, QK_STRIDE = 32768;   // two q/k buffers: [Q h0 | K h0][Q h1 | K h1]
constexpr uint32_t P_V = 65536, V_STRIDE = 16384; // two v buffers: [V h0][V h1]
constexpr uint32_t P_T = 98304;                   // A fp32 [64][A_LD], then T' hi, T' lo
constexpr uint32_t A_LD = 68;
constexpr uint32_t P_TF = P_T + 64 * A_LD * 4;    // T fp32 [64][T_LD]
constexpr uint32_t T_LD = 68;
constexpr uint32_t P_X = P_TF + 64 * T_LD * 4;
constexpr uint32_t X_LD = 36;
constexpr uint32_t P_T2 = 138240;                 // T'' hi, T'' lo (B operand of U~^T)
constexpr uint32_t P_PB = P_T2 + 16384;           // beta, gamma, G, 1/|q|, 1/|k|
constexpr uint32_t P_ST = 156672;                 // two staging blocks (ST_BYTES each)
constexpr uint32_t P_VL = P_ST + 2 * ST_BYTES;    // two v remainder buffers (values given as a pair)
constexpr uint32_t P_BAR = P_VL + 2 * V_STRIDE;

enum ChainBar { CB_FULL0, CB_FULL1, CB_RING0, CB_FREE0 = CB_RING0 + kRing, CB_FREE1,
                CB_U, CB_Q, CB_S, CB_O, CB_QREAD, CB_ODRAIN, CB_DRAIN, CB_Z0,
                CB_COUNT = CB_Z0 + kCNumOE };
enum PrepBar { PB_LD0, PB_LD1, PB_X, PB_XREAD, PB_T, PB_WU, PB_EPI, PB_RFREE0, PB_RFREE1, PB_DRAIN,
               PB_COUNT };

// words at the same offset in every CTA
constexpr uint32_t AUX_RAW = (C_BAR + CB_COUNT * 8 > P_BAR + PB_COUNT * 8) ? C_BAR + CB_COUNT * 8
                                                                          : P_BAR + PB_COUNT * 8;
constexpr uint32_t AUX = (AUX_RAW + 15) & ~15u;
constexpr uint32_t AUX_TSLOT = AUX, AUX_ABORT = AUX + 4, AUX_RING = AUX + 8, AUX_ARMED = AUX + 12,
                   AUX_SEQ = AUX + 16;
constexpr int kOrderMax = 1024;   // packed batches up to this many sequences run longest first
constexpr uint32_t SMEM_BYTES = AUX + 32 + 1024;
static_assert(P_X + 32 * X_LD * 4 <= P_T2, "prep layout");
static_assert(P_PB + 5 * 64 * 4 <= P_ST, "prep layout");
static_assert(64 * A_LD * 4 >= 16384, "T' tiles fit where A was");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(P_ST % 1024 == 0 && SLOT % 1024 == 0 && ST_BYTES % 1024 == 0 && P_VL % 1024 == 0 &&
                  P_T % 1024 == 0 &&
                  P_T2 % 1024 == 0 && P_V % 1024 == 0 && C_OT % 1024 == 0,
              "swizzle alignment");
static_assert(RSLOT % 16 == 0 && RS_U % 16 == 0, "bulk copy alignment");

// ---- TMEM columns ----
// chain: U' = S0 (-W)^T, S0 Q^T then U P^T, S0 hi, S0 lo (bf16 A operands), S (fp32),
//        U diag(gamma_L/gamma) hi/lo and U hi/lo (bf16 A operands)
constexpr uint32_t TM_U = 0, TM_Q = 64, TM_SH = 128, TM_SL = 192, TM_S = 256;
constexpr uint32_t TM_BH = 384, TM_BL = 416, TM_UH = 448, TM_UL = 480;
// prep: [Q;K]K^T, W^T, U~^T
constexpr uint32_t TP_X = 0, TP_W = 64, TP_U = 128;

struct RingParams {
    const float *g, *beta, *h0;
    const int32_t *cu;
    int64_t T;
    int HK, HV;
    float scale;
    __nv_bfloat16 *o;
    float *hT;
    unsigned int *status;
    uint8_t *rings;          // kRing records per SM id
    int nrings;              // SM ids the rings cover
    unsigned int prologue;   // GDN_PROLOGUE_* flags
    bool vpair;              // v comes with bf16 remainders (tm_vl): U~ = T''(V + V_lo)
};

// Release arrive on another cluster CTA's mbarrier: the arriving thread's earlier
// writes (and those it has observed) are visible to a thread that acquires the
// completed phase at cluster scope.
__device__ __forceinline__ void mbar_arrive_remote_release(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}
// Bulk copy from this CTA's shared memory to global memory, tracked by the bulk group.
__device__ __forceinline__ void bulk_store_s2g(void *dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
                 "r"(src), "r"(bytes)
                 : "memory");
}
// two fp32 lanes at once (sm_100 packed arithmetic), each rounded as its scalar op;
// the pairs are packed into 64-bit registers inside the asm so nothing goes to memory
#define GDN_PACKED2(name, op)                                                              \
    __device__ __forceinline__ float2 name(float2 a, float2 b) {                          \
        float2 d;                                                                          \
        asm("{\n\t.reg .b64 pa, pb, pd;\n\tmov.b64 pa, {%2, %3};\n\tmov.b64 pb, {%4, %5};\n\t" \
            op " pd, pa, pb;\n\tmov.b64 {%0, %1}, pd;\n\t}"                               \
            : "=f"(d.x), "=f"(d.y)                                                         \
            : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));                                     \
        return d;                                                                          \
    }
GDN_PACKED2(add2, "add.rn.f32x2")
GDN_PACKED2(mul2, "mul.rn.f32x2")
GDN_PACKED2(sub2, "sub.rn.f32x2")
#undef GDN_PACKED2
// A pair of floats -> its bf16 hi word (round to nearest) and the lo word of the
// remainder (bf16 of x - hi, exact subtraction), element 0 in the low halves.
__device__ __forceinline__ void split_pair(float2 x, uint32_t &hi, uint32_t &lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x.x, x.y);
    hi = *reinterpret_cast<const uint32_t *>(&h);
    const float2 hf = make_float2(__uint_as_float(hi << 16), __uint_as_float(hi & 0xffff0000u));
    const float2 r = sub2(x, hf);
    const __nv_bfloat162 l = __floats2bfloat162_rn(r.x, r.y);
    lo = *reinterpret_cast<const uint32_t *>(&l);
}
// 16 TMEM columns of this thread's lane as 8 pairs (waits for the load)
__device__ __forceinline__ void tmem_ld16p(uint32_t taddr, float2 (&v)[8]) {
    float x[16];
    tmem_ld16(taddr, x);
    tmem_wait_ld();
#pragma unroll
    for (int w = 0; w < 8; ++w) v[w] = make_float2(x[2 * w], x[2 * w + 1]);
}
__device__ __forceinline__ void tmem_st16p(uint32_t taddr, const float2 (&v)[8]) {
    float x[16];
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        x[2 * w] = v[w].x;
        x[2 * w + 1] = v[w].y;
    }
    tmem_st16(taddr, x);
}
// v op= 16 consecutive floats of shared memory (16-byte aligned), as pairs
__device__ __forceinline__ void add_lds16p(float2 (&v)[8], const float *src) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 f = reinterpret_cast<const float4 *>(src)[q];
        v[2 * q] = add2(v[2 * q], make_float2(f.x, f.y));
        v[2 * q + 1] = add2(v[2 * q + 1], make_float2(f.z, f.w));
    }
}
__device__ __forceinline__ void mul_lds16p(float2 (&v)[8], const float *src) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 f = reinterpret_cast<const float4 *>(src)[q];
        v[2 * q] = mul2(v[2 * q], make_float2(f.x, f.y));
        v[2 * q + 1] = mul2(v[2 * q + 1], make_float2(f.z, f.w));
    }
}
// ---- warp-level 16x8x8 TF32 products with fp32 accuracy (x = hi + lo, the three
// products hi*hi + hi*lo + lo*hi), for the small block products of the UT inverse.
// Fragments (lane = 4g + t): A 16x8 row-major {(g,t), (g+8,t), (g,t+4), (g+8,t+4)},
// B 8x8 {(k=t, n=g), (k=t+4, n=g)}, D 16x8 {(g,2t), (g,2t+1), (g+8,2t), (g+8,2t+1)}.
__device__ __forceinline__ uint32_t tf32_rna(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ void split_tf32(float x, uint32_t &hi, uint32_t &lo) {
    hi = tf32_rna(x);
    lo = tf32_rna(x - __uint_as_float(hi));
}
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// d += M[r0.., c0..] (16 x 8 of a row-major fp32 matrix, leading dimension ld) *
//      N[k0.., n0..] (8 x 8), entries where keep_a(row, col) / keep_b(k, n) is false
//      taken as zero
template <typename KA, typename KB>
__device__ __forceinline__ void mma3_smem(float (&d)[4], const float *M, int ld, int r0, int c0,
                                          const float *N, int ldn, int k0, int n0, KA keep_a,
                                          KB keep_b) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int ar[4] = {r0 + g, r0 + g + 8, r0 + g, r0 + g + 8};
    const int ac[4] = {c0 + t, c0 + t, c0 + t + 4, c0 + t + 4};
    uint32_t ah[4], al[4], bh[2], bl[2];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        split_tf32(keep_a(ar[i], ac[i]) ? M[ar[i] * ld + ac[i]] : 0.f, ah[i], al[i]);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int kk = k0 + t + 4 * i, nn = n0 + g;
        split_tf32(keep_b(kk, nn) ? N[kk * ldn + nn] : 0.f, bh[i], bl[i]);
    }
    mma_tf32(d, ah, bh);
    mma_tf32(d, ah, bl);
    mma_tf32(d, al, bh);
}
// D fragment (times s) into a row-major fp32 matrix at (r0, c0)
__device__ __forceinline__ void store_d(float *M, int ld, int r0, int c0, const float (&d)[4], float s) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    *reinterpret_cast<float2 *>(M + (r0 + g) * ld + c0 + 2 * t) = make_float2(s * d[0], s * d[1]);
    *reinterpret_cast<float2 *>(M + (r0 + g + 8) * ld + c0 + 2 * t) = make_float2(s * d[2], s * d[3]);
}

__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t cluster_addr) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t smid() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(r));
    return r;
}

__device__ __forceinline__ bool mbar_try_wait_acq_cluster(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_try_wait_plain(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded waits: try_wait without a suspend hint (the waiting warp is suspended by
// the hardware for a short, implementation-defined time and woken ~100 cycles
// after the phase completes), given up after kWaitCycles of the SM clock
// (~2 s); the drain after an abort gives up after kDrainCycles.
constexpr long long kWaitCycles = 4000000000LL, kDrainCycles = 100000000LL;
struct Waiter {
    uint64_t *bars;
    volatile int *abort_flag;
    unsigned int *status;
    uint32_t abort_saddr;   // shared address of the abort flag (same in every CTA)
    // false once the cluster has aborted: the caller then skips its work
    __device__ bool operator()(int b, uint32_t parity) const {
        if (mbar_try_wait_plain(&bars[b], parity)) return true;
        const long long t0 = clock64();
        for (;;) {
            if (*abort_flag) return false;
            if (mbar_try_wait_plain(&bars[b], parity)) return true;
            if (clock64() - t0 > kWaitCycles) break;
        }
        abort_all();
        return false;
    }
    // the same for a phase completed by another CTA's release arrive
    __device__ bool acquire(int b, uint32_t parity) const {
        const long long t0 = clock64();
        for (;;) {
            if (*abort_flag) return false;
            if (mbar_try_wait_acq_cluster(&bars[b], parity)) return true;
            if (clock64() - t0 > kWaitCycles) break;
        }
        abort_all();
        return false;
    }
    // teardown: waits (bounded) for in-flight work whether or not the cluster aborted
    __device__ void drain(int b, uint32_t parity) const {
        const long long t0 = clock64();
        while (!mbar_try_wait_plain(&bars[b], parity))
            if (clock64() - t0 > kDrainCycles) return;
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
template <bool GT>
__device__ void chain_cta(const CUtensorMap *tm_q, const CUtensorMap *tm_k, const CUtensorMap *tm_o,
                          const CUtensorMap *tm_z, const RingParams &p, uint8_t *sm, uint32_t sb,
                          uint32_t tmem, const Waiter &wt, int h, int n, int64_t bos, int64_t eos,
                          int nchunks, uint8_t *ring) {
    uint64_t *bars = wt.bars;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int HV = p.HV, cqk = h / (HV / p.HK);
    const size_t sbase = ((size_t)n * HV + h) * (size_t)DH * DH;
    auto chunk_len = [&](int c) {
        const int64_t r = eos - (bos + (int64_t)c * C);
        return (int)(r < C ? r : C);
    };
    if (warp == kCMma) {
        // ------------------------------------------------------------ MMA warp
        const uint32_t id_n64 = idesc_bf16(128, 64, false, false);
        const uint32_t id_s = idesc_bf16(128, 128, false, true);
        auto commit = [&](int b) {
            if (elect_one()) mma_commit(&bars[b]);
            __syncwarp();
        };
        bool ok = true;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c & 1;
            const uint32_t slot = sb + C_R + s * SLOT;
            ok = warp_all(ok && wt(CB_FULL0 + s, (uint32_t)((c >> 1) & 1)));
            if (ok) {
                // the record has landed: its ring slot goes back to the prep CTA
                if (elect_one())
                    mbar_arrive_remote_relaxed(mapa_shared(
                        sb + P_BAR + (PB_RFREE0 + ((c / kNumPrep) & 1)) * 8, 1 + c % kNumPrep));
                __syncwarp();
            }
            // S0 (hi, lo) of chunk c is in tensor memory
            named_sync(NB_S0, kChainSync);
            tc_fence_after();
            const uint64_t wq0 = sdesc_sw128(slot + SL_WQ, 16, 1024);
            const uint64_t q0 = sdesc_sw128(slot + SL_WQ + 8192, 16, 1024);
            if (ok) {
                // U' = S0 (-W)^T (the critical product first)
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    if (elect_one())
                        mma_bf16_ts(tmem + TM_U, tmem + TM_SH + 8 * k,
                                    desc_add(wq0, (k >> 2) * 16384 + (k & 3) * 32), id_n64, k > 0);
                    __syncwarp();
                }
                commit(CB_U);
            }
            // the previous chunk's outputs have been read out of the S0 Q^T columns
            if (c > 0) ok = warp_all(ok && wt(CB_ODRAIN, (uint32_t)((c - 1) & 1)));
            if (ok) {
                // S0 Q^T with S0 as hi + lo
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint64_t qd = desc_add(q0, (k >> 2) * 16384 + (k & 3) * 32);
                    if (elect_one()) {
                        mma_bf16_ts(tmem + TM_Q, tmem + TM_SH + 8 * k, qd, id_n64, k > 0);
                        mma_bf16_ts(tmem + TM_Q, tmem + TM_SL + 8 * k, qd, id_n64, 1);
                    }
                    __syncwarp();
                }
                commit(CB_Q);
            }
            // U diag(gamma_L/gamma) and U (hi, lo) are in TMEM, the state is rescaled
            named_sync(NB_UD, kChainSync);
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
                commit(CB_S);
            }
            // S0 Q^T has been read out: U P^T takes its columns
            ok = warp_all(ok && wt(CB_QREAD, (uint32_t)(c & 1)));
            if (ok) {
                tc_fence_after();
                const uint64_t p0 = sdesc_sw128(slot + SL_P, 16, 1024);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint64_t ph_d = desc_add(p0, k * 32), pl_d = desc_add(p0, 8192 + k * 32);
                    if (elect_one()) {
                        mma_bf16_ts(tmem + TM_Q, tmem + TM_UH + 8 * k, ph_d, id_n64, k > 0);
                        mma_bf16_ts(tmem + TM_Q, tmem + TM_UH + 8 * k, pl_d, id_n64, 1);
                        mma_bf16_ts(tmem + TM_Q, tmem + TM_UL + 8 * k, ph_d, id_n64, 1);
                    }
                    __syncwarp();
                }
                commit(CB_O);
                commit(CB_FREE0 + s);   // every read of this slot is issued before this point
            }
        }
        // every MMA issued here has completed before tensor memory is released
        commit(CB_DRAIN);
        wt.drain(CB_DRAIN, 0);
    } else if (warp == kCLoad) {
        // ------------------------------------------------------------ loader warp
        volatile int *armed = reinterpret_cast<volatile int *>(sm + AUX_ARMED);
        bool ok = true;
        if (lane == 0) {
            tma_prefetch_desc(tm_q);
            tma_prefetch_desc(tm_k);
        }
        for (int c = 0; c < nchunks && ok; ++c) {
            const int s = c & 1;
            // the slot's previous chunk (c - 2) has been read by every MMA
            if (c >= 2) ok = warp_all(wt(CB_FREE0 + s, (uint32_t)(((c >> 1) - 1) & 1)));
            if (!ok) break;
            uint8_t *slot = sm + C_R + s * SLOT;
            uint64_t *full = &bars[CB_FULL0 + s];
            const int s0 = (int)(bos + (int64_t)c * C);
            if (lane == 0) {
                mbar_arrive_expect_tx(full, SLOT);
                *armed = c + 1;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    tma_load_3d(slot + SL_WQ + hf * 16384 + 8192, tm_q, full, 64 * hf, cqk, s0);
                    tma_load_3d(slot + SL_K + hf * 8192, tm_k, full, 64 * hf, cqk, s0);
                }
                // the q/k tiles of chunk c + 2 into L2 ahead of their load
                if (c + 2 < nchunks) {
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        tma_prefetch_l2_3d(tm_q, 64 * hf, cqk, s0 + 2 * C);
                        tma_prefetch_l2_3d(tm_k, 64 * hf, cqk, s0 + 2 * C);
                    }
                }
            }
            __syncwarp();
            // the prep CTA has published chunk c's record
            ok = warp_all(wt.acquire(CB_RING0 + c % kRing, (uint32_t)((c / kRing) & 1)));
            if (!ok) break;
            if (lane == 0) {
                fence_proxy_async_global();
                const uint8_t *rec = ring + (size_t)(c % kRing) * RSLOT;
                bulk_load_g2s(slot + SL_WQ, rec + RS_W, 8192, full);
                bulk_load_g2s(slot + SL_WQ + 16384, rec + RS_W + 8192, 8192, full);
                bulk_load_g2s(slot + SL_P, rec + RS_P, RS_U - RS_P, full);   // P hi, P lo, table
                bulk_load_g2s(slot + SL_U, rec + RS_U, RSLOT - RS_U, full);
            }
            __syncwarp();
        }
    } else if (warp < kOE0) {
        // ------------------------------------------------------------ critical epilogue
        // Warp w works on TMEM lane quadrant w % 4 (state rows i) and half hf of the
        // columns: tokens 32 hf .. 32 hf + 31 of the 64-token products, state
        // columns 64 hf .. 64 hf + 63.
        const int hf = (warp - kCE0) >> 2;
        const int i = 32 * (warp & 3) + lane;
        // the fp32 state (64 columns) -> its S0 hi/lo copies in tensor memory
        auto split_copy = [&]() {
#pragma unroll
            for (int part = 0; part < 4; ++part) {
                float2 v[8];
                uint32_t whi[8], wlo[8];
                tmem_ld16p(tmem_addr(tmem, warp, TM_S + 64 * hf + 16 * part), v);
#pragma unroll
                for (int w = 0; w < 8; ++w) split_pair(v[w], whi[w], wlo[w]);
                tmem_st8w(tmem_addr(tmem, warp, TM_SH + 32 * hf + 8 * part), whi);
                tmem_st8w(tmem_addr(tmem, warp, TM_SL + 32 * hf + 8 * part), wlo);
            }
        };
        // the state scaled in place by gamma_L of the chunk about to start: that
        // chunk's update accumulates onto it (its first products read only the copies)
        auto scale_state = [&](float gL) {
            const float2 g2 = make_float2(gL, gL);
#pragma unroll
            for (int part = 0; part < 4; ++part) {
                float2 v[8];
                tmem_ld16p(tmem_addr(tmem, warp, TM_S + 64 * hf + 16 * part), v);
#pragma unroll
                for (int w = 0; w < 8; ++w) v[w] = mul2(v[w], g2);
                tmem_st16p(tmem_addr(tmem, warp, TM_S + 64 * hf + 16 * part), v);
            }
        };
        auto gamma_L = [&](int c) {
            return reinterpret_cast<const float *>(sm + C_R + (c & 1) * SLOT + SL_TAB)[128];
        };
        bool ok = true;
        {
            // start state into tensor memory with its bf16 hi/lo copy (chunk 0's S0),
            // then scaled by chunk 0's gamma_L
            const float *src = p.h0 ? p.h0 + sbase + (size_t)i * DH + 64 * hf : nullptr;
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                float v[32];
                uint32_t whi[16], wlo[16];
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    const float4 v4 = src ? *reinterpret_cast<const float4 *>(src + 32 * part + j)
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
                    v[j] = v4.x;
                    v[j + 1] = v4.y;
                    v[j + 2] = v4.z;
                    v[j + 3] = v4.w;
                }
                split_pack32(v, whi, wlo);
                tmem_st32f(tmem_addr(tmem, warp, TM_S + 64 * hf + 32 * part), v);
                tmem_st16w(tmem_addr(tmem, warp, TM_SH + 32 * hf + 16 * part), whi);
                tmem_st16w(tmem_addr(tmem, warp, TM_SL + 32 * hf + 16 * part), wlo);
            }
            tmem_wait_st();
            tc_fence_before();
            if (nchunks > 0) {
                named_sync(NB_S0, kChainSync);
                ok = warp_all(wt(CB_FULL0, 0u));
                if (ok) scale_state(gamma_L(0));
            }
        }
        for (int c = 0; c < nchunks; ++c) {
            const int s = c & 1;
            const uint8_t *slot = sm + C_R + s * SLOT;
            const float *tab = reinterpret_cast<const float *>(slot + SL_TAB);
            const float *ut = reinterpret_cast<const float *>(slot + SL_U);
            // U' of this chunk is formed (and, issued before it by the same thread, the
            // previous chunk's U P^T has read its U (hi, lo) operand)
            ok = warp_all(ok && wt(CB_U, (uint32_t)(c & 1)));
            if (ok) {
                tc_fence_after();
                // U diag(gamma_L/gamma) = (U~ - S0 W^T) diag(gamma_L/gamma) for tokens
                // t = 32 hf + j of row i, as hi and lo words (U is exactly zero for the
                // tokens past the end of a short last chunk: their beta is zero, so
                // their rows of T are unit rows and those of W and U~ vanish)
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    const int t0 = 32 * hf + 16 * part;
                    float2 u[8];
                    uint32_t whi[8], wlo[8];
                    tmem_ld16p(tmem_addr(tmem, warp, TM_U + t0), u);
                    add_lds16p(u, ut + i * UT_LD + t0);
                    mul_lds16p(u, tab + t0);
#pragma unroll
                    for (int w = 0; w < 8; ++w) split_pair(u[w], whi[w], wlo[w]);
                    tmem_st8w(tmem_addr(tmem, warp, TM_BH + t0 / 2), whi);
                    tmem_st8w(tmem_addr(tmem, warp, TM_BL + t0 / 2), wlo);
                }
            }
            // (the wait also covers the gamma_L-scaled state)
            tmem_wait_st();
            tc_fence_before();
            named_sync(NB_UD, kChainSync);
            const bool more = c + 1 < nchunks;
            ok = warp_all(ok && wt(CB_S, (uint32_t)(c & 1)));
            if (ok && more) {
                tc_fence_after();
                split_copy();
                tmem_wait_st();
            }
            tc_fence_before();
            if (more) {
                named_sync(NB_S0, kChainSync);
                // the next chunk's slot (its gamma_L) has landed: the MMA warp waited
                // for it before the barrier
                ok = warp_all(ok && wt(CB_FULL0 + ((c + 1) & 1), (uint32_t)(((c + 1) >> 1) & 1)));
                if (ok) scale_state(gamma_L(c + 1));
            }
        }
        if (ok && p.hT) {
            tc_fence_after();
            float *dst = p.hT + sbase + (size_t)i * DH + 64 * hf;
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                float v[32];
                tmem_ld32(tmem_addr(tmem, warp, TM_S + 64 * hf + 32 * part), v);
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    *reinterpret_cast<float4 *>(dst + 32 * part + j) =
                        make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
            }
        }
    } else {
        // ------------------------------------------------------------ output epilogue
        // Warp w reads lane quadrant w % 4 (value rows i) for tokens 32 hf .. 32 hf + 31.
        const int ow = warp - kOE0;
        const int hf = ow >> 2;
        unsigned short *ot = reinterpret_cast<unsigned short *>(sm + C_OT + ow * 2048);
        uint64_t *zbar = &bars[CB_Z0 + ow];
        uint32_t zph = 0;
        bool zflight = false;
        bool ok = true;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c & 1;
            const int64_t ps0 = bos + (int64_t)c * C;
            const int L = chunk_len(c);
            const float *tab = reinterpret_cast<const float *>(sm + C_R + s * SLOT + SL_TAB);
            if (GT && ok) {
                // this chunk's gate factors into the output tile, once its previous
                // store has been read (an L2 prefetch of the next chunk's tile first)
                if (lane == 0) {
                    if (c + 1 < nchunks)
                        tma_prefetch_l2_3d(tm_z, 32 * (warp & 3), h, (int)(ps0 + C + 32 * hf));
                    bulk_wait_group_read0();
                    fence_proxy_async_smem();
                    mbar_arrive_expect_tx(zbar, 2048);
                    tma_load_3d(ot, tm_z, zbar, 32 * (warp & 3), h, (int)(ps0 + 32 * hf));
                }
                __syncwarp();
                zflight = true;
            }
            // U = U~ - S0 W^T as bf16 hi/lo (the A operand of U P^T; its previous
            // reader, the last chunk's U P^T, completed before U' was formed), then
            // scale * gamma_t * (S0 q_t), read before U P^T takes its columns
            float dq[32];
            ok = warp_all(ok && wt(CB_FULL0 + s, (uint32_t)((c >> 1) & 1)) && wt(CB_U, (uint32_t)(c & 1)));
            if (ok) {
                tc_fence_after();
                const int i = 32 * (warp & 3) + lane;
                const float *utr = reinterpret_cast<const float *>(sm + C_R + s * SLOT + SL_U) + i * UT_LD;
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    const int t0 = 32 * hf + 16 * part;
                    float2 u[8];
                    uint32_t whi[8], wlo[8];
                    tmem_ld16p(tmem_addr(tmem, warp, TM_U + t0), u);
                    add_lds16p(u, utr + t0);
#pragma unroll
                    for (int w = 0; w < 8; ++w) split_pair(u[w], whi[w], wlo[w]);
                    tmem_st8w(tmem_addr(tmem, warp, TM_UH + t0 / 2), whi);
                    tmem_st8w(tmem_addr(tmem, warp, TM_UL + t0 / 2), wlo);
                }
            }
            ok = warp_all(ok && wt(CB_Q, (uint32_t)(c & 1)));
            if (ok) {
                tc_fence_after();
                tmem_ld32(tmem_addr(tmem, warp, TM_Q + 32 * hf), dq);
#pragma unroll
                for (int j = 0; j < 32; ++j) dq[j] *= p.scale * tab[64 + 32 * hf + j];
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) local_arrive(&bars[CB_QREAD]);
            float o32[32];
            ok = warp_all(ok && wt(CB_O, (uint32_t)(c & 1)));
            if (ok) {
                tc_fence_after();
                tmem_ld32(tmem_addr(tmem, warp, TM_Q + 32 * hf), o32);
#pragma unroll
                for (int j = 0; j < 32; ++j) dq[j] = fmaf(p.scale, o32[j], dq[j]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) local_arrive(&bars[CB_ODRAIN]);
            if (!ok) continue;
            if (GT) {
                ok = warp_all(wt(CB_Z0 + ow, zph));
                if (!ok) continue;
                zph ^= 1u;
                zflight = false;
            } else {
                // the tile's previous store has been read out of shared memory
                if (lane == 0) bulk_wait_group_read0();
                __syncwarp();
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                float out = dq[j];
                if (GT) out *= __half2float(__ushort_as_half(ot[j * 32 + lane]));
                const __nv_bfloat16 b = __float2bfloat16_rn(out);
                ot[j * 32 + lane] = *reinterpret_cast<const unsigned short *>(&b);
            }
            if (32 * hf + 32 <= L) {
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_3d(tm_o, ot, 32 * (warp & 3), h, (int)(ps0 + 32 * hf));
                    bulk_commit_group();
                }
            } else {
                __syncwarp();
#pragma unroll
                for (int pass = 0; pass < 4; ++pass) {
                    const int t = 8 * pass + (lane >> 2), c4 = lane & 3;
                    const uint4 val = *reinterpret_cast<const uint4 *>(ot + t * 32 + c4 * 8);
                    if (32 * hf + t < L)
                        *reinterpret_cast<uint4 *>(p.o + ((size_t)(ps0 + 32 * hf + t) * HV + h) * DH +
                                                   32 * (warp & 3) + 8 * c4) = val;
                }
            }
            __syncwarp();
        }
        // a gate-factor load still in flight (after an abort) lands before the CTA's
        // shared memory is released, and so do this warp's tile stores
        if (GT && zflight) wt.drain(CB_Z0 + ow, zph);
        if (lane == 0) bulk_wait_group0();
        __syncwarp();
    }
}

// ============================================================================ prep CTA
template <bool PRO>
__device__ void prep_cta(const CUtensorMap *tm_q, const CUtensorMap *tm_k, const CUtensorMap *tm_v,
                         const CUtensorMap *tm_vl, const RingParams &p, uint8_t *sm, uint32_t sb, uint32_t tmem,
                         const Waiter &wt, int h, int64_t bos, int64_t eos, int nchunks, int rank,
                         uint8_t *ring) {
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
        int issued = 0, landed = 0;    // q/k/v loads issued / waited for (k-th into buffer k & 1)
        bool stored = false;           // a bulk store of the staging block may be in flight
        auto load = [&](int k) {
            if (lane == 0) {
                const int s0 = (int)(bos + (int64_t)chunk_of(k) * C);
                uint64_t *bar = &bars[PB_LD0 + (k & 1)];
                uint8_t *buf = sm + P_QK + (k & 1) * QK_STRIDE;
                uint8_t *vb = sm + P_V + (k & 1) * V_STRIDE;
                mbar_arrive_expect_tx(bar, (p.vpair ? 8 : 6) * 8192);
                if (p.vpair) {
                    uint8_t *vl = sm + P_VL + (k & 1) * V_STRIDE;
                    tma_load_3d(vl, tm_vl, bar, 0, h, s0);
                    tma_load_3d(vl + 8192, tm_vl, bar, 64, h, s0);
                }
                tma_load_3d(buf, tm_q, bar, 0, cqk, s0);
                tma_load_3d(buf + 16384, tm_q, bar, 64, cqk, s0);
                tma_load_3d(buf + 8192, tm_k, bar, 0, cqk, s0);
                tma_load_3d(buf + 24576, tm_k, bar, 64, cqk, s0);
                tma_load_3d(vb, tm_v, bar, 0, h, s0);
                tma_load_3d(vb + 8192, tm_v, bar, 64, h, s0);
            }
            __syncwarp();
            ++issued;
        };
        // [Q;K]K^T of chunk k into TP_X once its tiles have landed
        auto x_product = [&](int k) -> bool {
            if (!warp_all(wt(PB_LD0 + (k & 1), (uint32_t)((k >> 1) & 1)))) return false;
            ++landed;
            tc_fence_after();
            const uint32_t qkv = sb + P_QK + (k & 1) * QK_STRIDE;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                const uint64_t a = sdesc_sw128(qkv + off, 16, 1024);
                const uint64_t b = sdesc_sw128(qkv + 8192 + off, 16, 1024);
                if (elect_one()) mma_bf16(tmem + TP_X, a, b, id_x, kk > 0);
                __syncwarp();
            }
            commit(PB_X);
            return true;
        };
        bool ok = nk > 0;
        if (nk > 0) {
            if (lane == 0) {
                tma_prefetch_desc(tm_q);
                tma_prefetch_desc(tm_k);
                tma_prefetch_desc(tm_v);
                if (p.vpair) tma_prefetch_desc(tm_vl);
            }
            load(0);
            if (nk > 1) load(1);
            ok = x_product(0);
        }
        for (int k = 0; k < nk && ok; ++k) {
            const int c = chunk_of(k);
            const uint32_t ph = (uint32_t)(k & 1);
            const uint32_t qkv = sb + P_QK + (k & 1) * QK_STRIDE;
            const uint32_t vb = sb + P_V + (k & 1) * V_STRIDE;
            // the workers have read chunk k's [Q;K]K^T: chunk k + 1's goes into its columns
            if (!warp_all(wt(PB_XREAD, ph))) break;
            if (k + 1 < nk && !x_product(k + 1)) break;
            if (!warp_all(wt(PB_T, ph))) break;
            tc_fence_after();
            // W^T = K^T T'^T and U~^T = V^T T''^T (T', T'' as hi + lo; V as V + V_lo
            // when the values come as a pair)
            const uint32_t vlb = sb + P_VL + (k & 1) * V_STRIDE;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ka = sdesc_sw128(qkv + 8192 + kk * 2048, 16384, 1024);
                const uint64_t va = sdesc_sw128(vb + kk * 2048, 8192, 1024);
                const uint64_t val = sdesc_sw128(vlb + kk * 2048, 8192, 1024);
                const uint64_t t1h = sdesc_sw128(sb + P_T + kk * 32, 16, 1024);
                const uint64_t t1l = sdesc_sw128(sb + P_T + 8192 + kk * 32, 16, 1024);
                const uint64_t t2h = sdesc_sw128(sb + P_T2 + kk * 32, 16, 1024);
                const uint64_t t2l = sdesc_sw128(sb + P_T2 + 8192 + kk * 32, 16, 1024);
                if (elect_one()) {
                    mma_bf16(tmem + TP_W, ka, t1h, id_w, kk > 0);
                    mma_bf16(tmem + TP_W, ka, t1l, id_w, 1);
                    mma_bf16(tmem + TP_U, va, t2h, id_w, kk > 0);
                    mma_bf16(tmem + TP_U, va, t2l, id_w, 1);
                    if (p.vpair) mma_bf16(tmem + TP_U, val, t2h, id_w, 1);
                }
                __syncwarp();
            }
            commit(PB_WU);
            // workers: -W, P and the table staged, U~ written into the ring record
            if (!warp_all(wt(PB_EPI, ph))) break;
            // chunk k + 2's tiles into chunk k's buffers (every product reading them
            // has completed), then chunk k's hand-over
            if (k + 2 < nk) load(k + 2);
            if (lane == 0) {
                uint8_t *rec = ring + (size_t)(c % kRing) * RSLOT;
                const uint32_t stg = sb + P_ST + (k & 1) * ST_BYTES;
                fence_proxy_async_smem();
                bulk_store_s2g(rec + RS_W, stg + ST_W, 16384);
                bulk_store_s2g(rec + RS_TAB, stg + ST_TAB, ST_BYTES - ST_TAB);
                bulk_commit_group();
                bulk_wait_group0();
                fence_proxy_async_global();
                mbar_arrive_remote_release(mapa_shared(sb + C_BAR + (CB_RING0 + c % kRing) * 8, 0));
            }
            stored = true;
            __syncwarp();
        }
        // after an abort: a load still in flight lands, issued MMAs complete and
        // bulk stores have read the staging blocks before this CTA's memory is released
        for (int d = landed; d < issued; ++d) wt.drain(PB_LD0 + (d & 1), (uint32_t)((d >> 1) & 1));
        if (stored && lane == 0) bulk_wait_group0();
        __syncwarp();
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
        auto rq = [&](int t) { return PRO ? rq_p[t] : 1.f; };
        auto rk = [&](int t) { return PRO ? rk_p[t] : 1.f; };
        float *A_s = reinterpret_cast<float *>(sm + P_T);
        float *T_s = reinterpret_cast<float *>(sm + P_TF);
        float *X_s = reinterpret_cast<float *>(sm + P_X);
        bool ok = true;
        // g (worker warp 0) and beta (worker warp 1) of a chunk are loaded one chunk
        // ahead: their strided reads come from DRAM
        float2 gb_next = make_float2(0.f, 0.f);
        auto load_gb = [&](int k) {
            const int c = chunk_of(k);
            const float *src = warp == kPWork0 ? p.g : p.beta;
            return load_g_pair(src, bos + (int64_t)c * C, chunk_len(c), HV, h);
        };
        if (nk > 0 && warp <= kPWork0 + 1) gb_next = load_gb(0);
        for (int k = 0; k < nk; ++k) {
            const int c = chunk_of(k);
            const uint32_t ph = (uint32_t)(k & 1);
            const int L = chunk_len(c);
            const uint32_t stb = P_ST + (k & 1) * ST_BYTES;   // this chunk's staging block
            uint8_t *rec = ring + (size_t)(c % kRing) * RSLOT;     // and its ring record
            named_sync(NB_WORK, kPWorkThreads);
            float2 gb = gb_next;
            if (warp <= kPWork0 + 1 && k + 1 < nk) gb_next = load_gb(k + 1);
            if (warp == kPWork0) {
                float2 gp = gb;
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
                float2 bp = gb;
                if (logits) {   // beta = sigmoid(b)
                    if (2 * lane < L) bp.x = gate_sigmoid(bp.x);
                    if (2 * lane + 1 < L) bp.y = gate_sigmoid(bp.y);
                }
                beta_s[2 * lane] = bp.x;
                beta_s[2 * lane + 1] = bp.y;
            }
            // the X product is done (this staging block's previous contents, chunk k - 2,
            // were stored before chunk k's X product began), and the chain has taken
            // chunk c - kRing out of this ring record
            ok = warp_all(ok && wt(PB_X, ph));
            if (k >= 2) ok = warp_all(ok && wt(PB_RFREE0 + (k & 1), (uint32_t)(((k >> 1) - 1) & 1)));
            if (norm_qk) {
                // squared norms of the 64 q and 64 k rows of the landed tiles: four
                // threads per row, 64 bytes each (the 128B swizzle only permutes the
                // 16-byte pieces inside a row)
                ok = warp_all(ok && wt(PB_LD0 + (k & 1), (uint32_t)((k >> 1) & 1)));
                if (ok) {
                    const int qr = pt >> 2, part = pt & 3;
                    const bool isk = qr >= 64;
                    const int t = qr & 63;
                    const uint8_t *rp = sm + P_QK + (k & 1) * QK_STRIDE + (part >> 1) * 16384 +
                                        (isk ? 8192 : 0) + t * 128 + (part & 1) * 64;
                    float ss = 0.f;
#pragma unroll
                    for (int ii = 0; ii < 4; ++ii) {
                        const uint4 w = *reinterpret_cast<const uint4 *>(rp + 16 * ii);
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
                tmem_ld16(tmem_addr(tmem, warp, TP_X + 16 * qtr), v);
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
                        // P hi and lo into the record, as the chain CTA's swizzled operand image
                        const uint32_t off = sw128_chunk(row, 2 * qtr + cc);
                        uint32_t hw[4], lw[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            split_pair(make_float2(v[8 * cc + 2 * e], v[8 * cc + 2 * e + 1]), hw[e], lw[e]);
                        *reinterpret_cast<uint4 *>(rec + RS_P + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                        *reinterpret_cast<uint4 *>(rec + RS_P + 8192 + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
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
            // [Q;K]K^T has been read: the control warp may form the next chunk's
            tc_fence_before();
            __syncwarp();
            if (lane == 0) local_arrive(&bars[PB_XREAD]);
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
            // ---- step 2: within each 32x32 half h, T10 = -T11 (A10 T00) (16 x 16 blocks
            //      at rows 32h + 16, columns 32h); worker warp 2h + j owns columns 8j..8j+7
            //      of the block: Y = A10 T00 into the block's place in T, then -T11 Y over
            //      it (the warp reads its columns of Y before writing them) ----
            const int wi = warp - kPWork0;
            const auto all = [](int, int) { return true; };
            if (ok && wi < 4) {
                const int hh = wi >> 1, nt = wi & 1, r1 = 32 * hh + 16, c0 = 32 * hh;
                float d[4] = {0.f, 0.f, 0.f, 0.f};
                // T00 is lower triangular: k-steps below the tile's first column vanish
                for (int kk = nt; kk < 2; ++kk)
                    mma3_smem(d, A_s, A_LD, r1, c0 + 8 * kk, T_s, T_LD, c0 + 8 * kk, c0 + 8 * nt, all, all);
                store_d(T_s, T_LD, r1, c0 + 8 * nt, d, 1.f);
                __syncwarp();
                float e[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int kk = 0; kk < 2; ++kk)
                    mma3_smem(e, T_s, T_LD, r1, r1 + 8 * kk, T_s, T_LD, r1 + 8 * kk, c0 + 8 * nt, all, all);
                __syncwarp();
                store_d(T_s, T_LD, r1, c0 + 8 * nt, e, -1.f);
            }
            named_sync(NB_WORK, kPWorkThreads);
            // ---- step 3: T[32:64][0:32] = -T22 (A21 T11); worker warp w < 8 owns the 16 x 8
            //      tile (rows 16 (w >> 2), columns 8 (w & 3)) of X = A21 T11, then of the
            //      result.  The blocks above the diagonal that no step wrote (T11 rows
            //      0..15 x columns 16..31, T22 rows 32..47 x columns 48..63) are masked:
            //      T11[k][n] = 0 for k < n, T22[m][k] = 0 for k > m ----
            if (ok && wi < 8) {
                const int mt = wi >> 2, nt = wi & 3;
                float d[4] = {0.f, 0.f, 0.f, 0.f};
                for (int kk = nt; kk < 4; ++kk)
                    mma3_smem(d, A_s, A_LD, 32 + 16 * mt, 8 * kk, T_s, T_LD, 8 * kk, 8 * nt, all,
                              [](int k, int n) { return k >= n; });
                store_d(X_s, X_LD, 16 * mt, 8 * nt, d, 1.f);
            }
            named_sync(NB_WORK, kPWorkThreads);
            if (ok && wi < 8) {
                const int mt = wi >> 2, nt = wi & 3;
                float d[4] = {0.f, 0.f, 0.f, 0.f};
                for (int kk = 0; kk <= 2 * mt + 1; ++kk)
                    mma3_smem(d, T_s, T_LD, 32 + 16 * mt, 32 + 8 * kk, X_s, X_LD, 8 * kk, 8 * nt,
                              [](int m, int k) { return k <= m; }, all);
                store_d(T_s, T_LD, 32 + 16 * mt, 8 * nt, d, -1.f);
            }
            named_sync(NB_WORK, kPWorkThreads);
            // ---- T' = T diag(b gamma) (for W) and T'' = T diag(b) (for U~) as hi/lo
            //      bf16 tiles; A is dead ----
            if (ok) {
                const int t = pt >> 3, chunk16 = pt & 7;
                float a1[8], a2[8];
#pragma unroll
                for (int h4 = 0; h4 < 2; ++h4) {
                    const int s4 = 8 * chunk16 + 4 * h4;
                    const float4 tv = *reinterpret_cast<const float4 *>(T_s + t * T_LD + s4);
                    const float4 bv = *reinterpret_cast<const float4 *>(beta_s + s4);
                    const float4 gv = *reinterpret_cast<const float4 *>(gam_p + s4);
                    const float tt[4] = {tv.x, tv.y, tv.z, tv.w}, bb[4] = {bv.x, bv.y, bv.z, bv.w};
                    const float gg[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int sidx = s4 + e;
                        a2[4 * h4 + e] = (sidx <= t ? tt[e] : 0.f) * bb[e];
                        a1[4 * h4 + e] = a2[4 * h4 + e] * gg[e] * rk(sidx);
                    }
                }
                const uint32_t off = sw128_chunk(t, chunk16);
                st_chunk_hilo(sb + P_T + off, sb + P_T + 8192 + off, a1);
                st_chunk_hilo(sb + P_T2 + off, sb + P_T2 + 8192 + off, a2);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) local_arrive(&bars[PB_T]);
            // ---- -W into the staging block, U~ into the ring record ----
            ok = warp_all(ok && wt(PB_WU, ph));
            if (ok) {
                tc_fence_after();
                float v[16], u16[16];
                // W^T row a = r, tokens t = 16 qtr + j -> -W rows of the K-major [-W;Q] operand
                tmem_ld16(tmem_addr(tmem, warp, TP_W + 16 * qtr), v);
                tmem_ld16(tmem_addr(tmem, warp, TP_U + 16 * qtr), u16);
                tmem_wait_ld();
                uint8_t *wq = sm + stb + ST_W + (r >> 6) * 8192 + (r & 7) * 2;
                const uint32_t wc = (uint32_t)((r & 63) >> 3);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int t = 16 * qtr + j;
                    *reinterpret_cast<__nv_bfloat16 *>(wq + t * 128 + ((wc ^ (uint32_t)(t & 7)) << 4)) =
                        __float2bfloat16_rn(-v[j]);
                }
                // U~^T row i = r, tokens t = 16 qtr + j -> U~[i][t] (64 contiguous bytes per thread)
                float4 *ur = reinterpret_cast<float4 *>(rec + RS_U + ((size_t)r * UT_LD + 16 * qtr) * 4);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    ur[j] = make_float4(u16[4 * j], u16[4 * j + 1], u16[4 * j + 2], u16[4 * j + 3]);
                // for the chain's bulk copy of the record (the control thread's release
                // arrive publishes these writes)
                fence_proxy_async_global();
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) local_arrive(&bars[PB_EPI]);
        }
    }
}

// TMO: a test-only instance whose first wait -- before any load, copy or MMA is
// issued -- has a limit of zero polls on a barrier nothing arrives on, so the
// timeout path (status word, abort flags in every CTA, every loop running its
// iterations without work, the drains) runs without a real hang.
template <bool PRO, bool GT, bool TMO = false>
__global__ void __launch_bounds__(kThreads, 1)
prefill_ring_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_vl,
                    const __grid_constant__ CUtensorMap tm_o, const __grid_constant__ CUtensorMap tm_z,
                    const RingParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    const int rank = (int)cluster_ctarank();
    const int h = blockIdx.x / kClusterSize;
    const int tid = threadIdx.x, warp = tid >> 5;
    // Packed batches run longest sequence first: row r of the grid (dispatched after
    // rows 0..r-1) takes the sequence of rank r by decreasing length (ties by index),
    // so the long chains start in the first wave and the short ones fill the tail.
    // Every CTA of a cluster derives the same permutation from cu_seqlens.
    int n = blockIdx.y;
    if (p.cu && gridDim.y > 1 && gridDim.y <= (unsigned)kOrderMax) {
        const int N = (int)gridDim.y;
        volatile int *seq = reinterpret_cast<volatile int *>(sm + AUX_SEQ);
        if (tid == 0) *seq = n;
        __syncthreads();
        for (int m = tid; m < N; m += kThreads) {
            const int lm = p.cu[m + 1] - p.cu[m];
            int rk = 0;
            for (int j = 0; j < N; ++j) {
                const int lj = p.cu[j + 1] - p.cu[j];
                rk += (lj > lm || (lj == lm && j < m)) ? 1 : 0;
            }
            if (rk == n) *seq = m;
        }
        __syncthreads();
        n = *seq;
    }
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
    const uint32_t ncols = rank == 0 ? 512u : 256u;

    if (tid == 0) {
        for (int b = 0; b < nbars; ++b) {
            uint32_t cnt = 1;
            if (rank != 0 && (b == PB_T || b == PB_EPI || b == PB_XREAD)) cnt = kPNumWork;
            if (rank == 0 && (b == CB_ODRAIN || b == CB_QREAD)) cnt = kCNumOE;
            mbar_init(&bars[b], cnt);
        }
        *abort_flag = 0;
        *reinterpret_cast<volatile int *>(sm + AUX_ARMED) = 0;
        // the chain CTA's SM id selects the ring the cluster uses (one chain CTA per SM
        // at a time: the shared-memory footprint allows a single CTA per SM)
        if (rank == 0) *reinterpret_cast<volatile int *>(sm + AUX_RING) = (int)smid();
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(tslot, ncols);
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    cluster_sync_all();   // every CTA's barriers are initialised before any remote traffic

    if (TMO) {
        // the drain barrier completes only at teardown: a zero-limit wait on it gives up
        if (rank == 0 && tid == 0 && !mbar_test_wait(&bars[CB_DRAIN], 0u)) wt.abort_all();
        cluster_sync_all();   // every CTA sees the abort flags before any work starts
    }
    const int ring_id = (int)ld_cluster_u32(mapa_shared(sb + AUX_RING, 0));
    const bool ring_ok = ring_id >= 0 && ring_id < p.nrings;
    if (!ring_ok && rank == 0 && tid == 0) atomicExch(p.status, (unsigned int)GDN_ERR_CUDA);
    uint8_t *ring = p.rings + (size_t)(ring_ok ? ring_id : 0) * kRing * RSLOT;
    // after an abort (only the test instance can have one here) no work is issued
    const int nwork = (ring_ok && !(TMO && *abort_flag)) ? nchunks : 0;

    if (rank == 0)
        chain_cta<GT>(&tm_q, &tm_k, &tm_o, &tm_z, p, sm, sb, tmem, wt, h, n, bos, eos, nwork, ring);
    else
        prep_cta<PRO>(&tm_q, &tm_k, &tm_v, &tm_vl, p, sm, sb, tmem, wt, h, bos, eos, nwork, rank, ring);

    tc_fence_before();
    __syncthreads();
    if (rank == 0 && tid == 0) {
        // after an abort: loads already issued into the receive slots land before
        // this CTA's shared memory is released (the loader arms a slot's barrier
        // for every chunk it started; the MMA warp consumed the rest)
        const int armed = *reinterpret_cast<volatile int *>(sm + AUX_ARMED);
        for (int d = armed - 2 > 0 ? armed - 2 : 0; d < armed; ++d)
            wt.drain(CB_FULL0 + (d & 1), (uint32_t)((d >> 1) & 1));
    }
    if (warp == 0) tmem_dealloc(tmem, ncols);
    cluster_sync_all();   // no CTA leaves while another may still address its shared memory
}

int device_sm_count() {
    int dev = 0, nsm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || nsm <= 0) {
        cudaGetLastError();   // clear a sticky "no device" from the query
        return 0;
    }
    return nsm;
}

}  // namespace

bool prefill_ring_supported(int dk, int dv, int chunk, gdn_dtype dtype) {
    return dtype == GDN_BF16 && dk == DH && dv == DH && chunk == C;
}

size_t prefill_ring_workspace(int, int64_t, int, int, bool) {
    // one ring per SM id; 148 SMs on a B200 when no device can be queried
    const int nsm = device_sm_count();
    const size_t nrings = (size_t)(nsm > 0 ? nsm : 148);
    return kRingHeader + nrings * kRing * RSLOT;
}

cudaError_t launch_prefill_ring(const PrefillArgs &a, cudaStream_t stream, bool timeout_test) {
    const int64_t Ttot = a.cu_seqlens ? a.T : (int64_t)a.N * a.T;
    if (Ttot >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    if (a.workspace_bytes < kRingHeader + (size_t)kRing * RSLOT) return cudaErrorInvalidValue;
    unsigned int *status = static_cast<unsigned int *>(a.workspace);
    cudaError_t err = a.keep_status ? cudaSuccess : cudaMemsetAsync(status, 0, sizeof(unsigned int), stream);
    if (err != cudaSuccess) return err;
    CUtensorMap tq, tk, tv, tvl, to;
    const uint64_t tok = (uint64_t)(Ttot > 0 ? Ttot : 1);
    uint64_t dq[3] = {(uint64_t)DH, (uint64_t)a.HK, tok};
    uint64_t sq[2] = {(uint64_t)DH * 2, (uint64_t)a.HK * DH * 2};
    uint64_t dv[3] = {(uint64_t)DH, (uint64_t)a.HV, tok};
    uint64_t sv[2] = {(uint64_t)DH * 2, (uint64_t)a.HV * DH * 2};
    uint32_t box[3] = {64, 1, 64};
    if (!encode_bf16_map(&tq, a.q, 3, dq, sq, box) || !encode_bf16_map(&tk, a.k, 3, dq, sq, box) ||
        !encode_bf16_map(&tv, a.v, 3, dv, sv, box))
        return cudaErrorInvalidValue;
    tvl = tv;
    if (a.v_lo && !encode_bf16_map(&tvl, a.v_lo, 3, dv, sv, box)) return cudaErrorInvalidValue;
    // o: one output warp's 32 tokens x 32 value rows per store, unswizzled 64-byte rows
    uint32_t obox[3] = {32, 1, 32};
    if (!encode_bf16_map(&to, a.o, 3, dv, sv, obox, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    // gate factors (fp16, o's layout; copied raw, so the 2-byte map type serves)
    CUtensorMap tz = to;
    if (a.gate && !encode_bf16_map(&tz, a.gate, 3, dv, sv, obox, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    auto kern = a.gate ? (a.prologue ? prefill_ring_kernel<true, true> : prefill_ring_kernel<false, true>)
                       : (a.prologue ? prefill_ring_kernel<true, false> : prefill_ring_kernel<false, false>);
    if (timeout_test) kern = prefill_ring_kernel<false, false, true>;
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (err != cudaSuccess) return err;
    RingParams prm{a.g, a.beta, a.h0, a.cu_seqlens, a.T, a.HK, a.HV, a.scale,
                   static_cast<__nv_bfloat16 *>(a.o), a.hT, status,
                   static_cast<uint8_t *>(a.workspace) + kRingHeader,
                   (int)((a.workspace_bytes - kRingHeader) / ((size_t)kRing * RSLOT)), a.prologue,
                   a.v_lo != nullptr};
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
    err = cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, tvl, to, tz, prm);
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
}

}  // namespace gdn
