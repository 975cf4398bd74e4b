// Chunkwise prefill of the gated delta rule on CUDA cores (fp32 arithmetic).
//
// This path serves every (dtype, head dim, chunk) the tensor-core path does not
// (fp32 inputs in particular: TF32 operands would not meet an fp32 tolerance).
//
// Chunk algebra (derived from the recurrence S_t = a_t S_{t-1}(I - b_t k_t k_t^T)
// + b_t v_t k_t^T, "Qwen3-Next", sghael.github.io, section "Correcting a memory
// instead of adding to it").  Inside a chunk of L tokens that starts from S0,
// with G the chunk-local running sum of g and gamma_i = exp(G_i):
//   u_i = b_i (v_i - a_i S_{i-1} k_i)   so that   S_i = a_i S_{i-1} + u_i k_i^T
//   (I + A) U = Y,  A_ij = b_i exp(G_i - G_j) k_i.k_j (j < i),
//                   Y_i  = b_i (v_i - gamma_i S0 k_i)
//   o_i  = gamma_i S0 q_i + sum_{j<=i} exp(G_i - G_j) (q_i.k_j) u_j
//   S_L  = gamma_L S0 + sum_j exp(G_L - G_j) u_j k_j^T
// U is obtained by forward substitution on the unit-lower-triangular system,
// which is the same result as applying the UT inverse T = (I + A)^-1 to Y.
//
// Work split: one CTA per (value tile of BV state rows, value head, sequence).
// State rows are independent, so each CTA carries BV rows of S in shared
// memory through the sequential loop over chunks; the key-key and query-key
// products of a chunk are recomputed by each value tile.
#include <cuda_fp16.h>

#include <type_traits>

#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kSimtThreads = 256;

template <int DK, int BV, int C>
struct SimtSmem {
    static constexpr int KP = DK + 1;  // padded rows: conflict-free column walks
    static constexpr int CP = C + 1;
    static constexpr size_t floats = 2 * (size_t)C * KP   // K, Q
                                     + (size_t)BV * KP    // S rows
                                     + 2 * (size_t)C * CP // A, P
                                     + 3 * (size_t)C * BV // Y/U, K S^T, Q S^T
                                     + 2 * (size_t)C;     // G, beta
    static constexpr size_t bytes = floats * sizeof(float);
};

template <typename Tin, int DK, int BV, int C>
__global__ void __launch_bounds__(kSimtThreads)
prefill_simt_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k,
                    const Tin *__restrict__ v, const float *__restrict__ g,
                    const float *__restrict__ beta, const float *__restrict__ h0,
                    const int32_t *__restrict__ cu, int64_t T, int HK, int HV, int dv,
                    float scale, Tin *__restrict__ o, float *__restrict__ hT, unsigned pro,
                    const void *__restrict__ gate) {
    using L_ = SimtSmem<DK, BV, C>;
    constexpr int KP = L_::KP, CP = L_::CP, NT = kSimtThreads;
    const int tid = threadIdx.x;
    const int e0 = blockIdx.x * BV;
    const int h = blockIdx.y;
    const int n = blockIdx.z;
    const int c = h / (HV / HK);
    int64_t bos, eos;
    if (cu) {
        bos = cu[n];
        eos = cu[n + 1];
    } else {
        bos = (int64_t)n * T;
        eos = bos + T;
    }

    extern __shared__ float sm[];
    float *Ks = sm;
    float *Qs = Ks + C * KP;
    float *Ss = Qs + C * KP;
    float *As = Ss + BV * KP;
    float *Ps = As + C * CP;
    float *Ys = Ps + C * CP;
    float *KSs = Ys + C * BV;
    float *QSs = KSs + C * BV;
    float *Gs = QSs + C * BV;
    float *Bs = Gs + C;

    const size_t state_base = ((size_t)n * HV + h) * (size_t)dv * DK;
    for (int idx = tid; idx < BV * DK; idx += NT) {
        const int e = idx / DK, a = idx - e * DK;
        Ss[e * KP + a] = h0 ? h0[state_base + (size_t)(e0 + e) * DK + a] : 0.f;
    }

    for (int64_t s0 = bos; s0 < eos; s0 += C) {
        const int L = (int)((eos - s0) < C ? (eos - s0) : C);
        __syncthreads();  // previous chunk fully consumed
        // ---- load the chunk (rows >= L are zero) ----
        for (int idx = tid; idx < C * (DK / 4); idx += NT) {
            const int i = idx / (DK / 4), a = (idx - i * (DK / 4)) * 4;
            float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), qv = kv;
            if (i < L) {
                const size_t off = ((size_t)(s0 + i) * HK + c) * DK + a;
                kv = load4(k + off);
                qv = load4(q + off);
            }
            float *kr = Ks + i * KP + a, *qr = Qs + i * KP + a;
            kr[0] = kv.x; kr[1] = kv.y; kr[2] = kv.z; kr[3] = kv.w;
            qr[0] = qv.x; qr[1] = qv.y; qr[2] = qv.z; qr[3] = qv.w;
        }
        for (int idx = tid; idx < C * BV; idx += NT) {
            const int i = idx / BV, e = idx - i * BV;
            Ys[idx] = i < L ? to_f32(v[((size_t)(s0 + i) * HV + h) * dv + e0 + e]) : 0.f;
        }
        if (tid < C) {
            // with gate logits: g = log sigmoid(a), beta = sigmoid(b); padding stays 0
            const bool logits = (pro & GDN_PROLOGUE_GATE_LOGITS) != 0;
            const float gv = tid < L ? g[(s0 + tid) * HV + h] : 0.f;
            const float bv = tid < L ? beta[(s0 + tid) * HV + h] : 0.f;
            Gs[tid] = (logits && tid < L) ? gate_log_sigmoid(gv) : gv;
            Bs[tid] = (logits && tid < L) ? gate_sigmoid(bv) : bv;
        }
        __syncthreads();
        // ---- chunk-local running sum of the log decay ----
        if (tid == 0) {
            float run = 0.f;
            for (int i = 0; i < L; ++i) { run += Gs[i]; Gs[i] = run; }
        }
        // ---- input prologue: L2-normalised q / k rows (one thread per row) ----
        if (pro & (GDN_PROLOGUE_NORM_Q | GDN_PROLOGUE_NORM_K)) {
            for (int idx = tid; idx < 2 * L; idx += NT) {
                const bool is_k = idx >= L;
                if (!(pro & (is_k ? GDN_PROLOGUE_NORM_K : GDN_PROLOGUE_NORM_Q))) continue;
                float *row = (is_k ? Ks : Qs) + (idx - (is_k ? L : 0)) * KP;
                float ss = 0.f;
                for (int a = 0; a < DK; ++a) ss = fmaf(row[a], row[a], ss);
                const float r = inv_l2norm(ss);
                for (int a = 0; a < DK; ++a) row[a] *= r;
            }
        }
        __syncthreads();
        // ---- A (strictly lower) and P (lower incl. diagonal) ----
        for (int idx = tid; idx < C * C; idx += NT) {
            const int i = idx / C, j = idx - i * C;
            float av = 0.f, pv = 0.f;
            if (i < L && j <= i) {
                float kk = 0.f, qk = 0.f;
#pragma unroll 8
                for (int a = 0; a < DK; ++a) {
                    const float kj = Ks[j * KP + a];
                    kk = fmaf(Ks[i * KP + a], kj, kk);
                    qk = fmaf(Qs[i * KP + a], kj, qk);
                }
                const float gam = expf(Gs[i] - Gs[j]);
                if (j < i) av = Bs[i] * gam * kk;
                pv = gam * qk;
            }
            As[i * CP + j] = av;
            Ps[i * CP + j] = pv;
        }
        // ---- K S0^T and Q S0^T for this tile's rows ----
        for (int idx = tid; idx < C * BV; idx += NT) {
            const int i = idx / BV, e = idx - i * BV;
            float ks = 0.f, qs = 0.f;
            if (i < L) {
#pragma unroll 8
                for (int a = 0; a < DK; ++a) {
                    const float s = Ss[e * KP + a];
                    ks = fmaf(Ks[i * KP + a], s, ks);
                    qs = fmaf(Qs[i * KP + a], s, qs);
                }
            }
            KSs[idx] = ks;
            QSs[idx] = qs;
        }
        __syncthreads();
        // ---- Y_i = b_i (v_i - gamma_i S0 k_i) ----
        for (int idx = tid; idx < C * BV; idx += NT) {
            const int i = idx / BV;
            Ys[idx] = i < L ? Bs[i] * (Ys[idx] - expf(Gs[i]) * KSs[idx]) : 0.f;
        }
        __syncthreads();
        // ---- forward substitution: U_i = Y_i - sum_{j<i} A_ij U_j ----
        for (int i = 1; i < L; ++i) {
            for (int e = tid; e < BV; e += NT) {
                float acc = Ys[i * BV + e];
                for (int j = 0; j < i; ++j) acc = fmaf(-As[i * CP + j], Ys[j * BV + e], acc);
                Ys[i * BV + e] = acc;
            }
            __syncthreads();
        }
        // ---- o_i = gamma_i S0 q_i + sum_{j<=i} P_ij u_j ----
        for (int idx = tid; idx < L * BV; idx += NT) {
            const int i = idx / BV, e = idx - i * BV;
            float acc = 0.f;
            for (int j = 0; j <= i; ++j) acc = fmaf(Ps[i * CP + j], Ys[j * BV + e], acc);
            acc = fmaf(expf(Gs[i]), QSs[idx], acc);
            const size_t oi = ((size_t)(s0 + i) * HV + h) * dv + e0 + e;
            float out = scale * acc;
            if (gate)   // output gate, before the one rounding: fp32 factors for fp32, else fp16
                out *= std::is_same<Tin, float>::value ? static_cast<const float *>(gate)[oi]
                                                       : __half2float(static_cast<const __half *>(gate)[oi]);
            o[oi] = from_f32<Tin>(out);
        }
        __syncthreads();
        // ---- S_L = gamma_L S0 + sum_j exp(G_L - G_j) u_j k_j^T ----
        const float GL = Gs[L - 1];
        for (int idx = tid; idx < L * BV; idx += NT) {
            const int j = idx / BV, e = idx - j * BV;
            Ys[idx] *= expf(GL - Gs[j]);
        }
        __syncthreads();
        const float gL = expf(GL);
        for (int idx = tid; idx < BV * DK; idx += NT) {
            const int e = idx / DK, a = idx - e * DK;
            float acc = gL * Ss[e * KP + a];
            for (int j = 0; j < L; ++j) acc = fmaf(Ys[j * BV + e], Ks[j * KP + a], acc);
            Ss[e * KP + a] = acc;
        }
    }
    __syncthreads();
    if (hT) {
        for (int idx = tid; idx < BV * DK; idx += NT) {
            const int e = idx / DK, a = idx - e * DK;
            hT[state_base + (size_t)(e0 + e) * DK + a] = Ss[e * KP + a];
        }
    }
}

template <typename Tin, int DK, int BV, int C>
cudaError_t launch_shape(const PrefillArgs &a, cudaStream_t stream) {
    constexpr size_t smem = SimtSmem<DK, BV, C>::bytes;
    auto kern = prefill_simt_kernel<Tin, DK, BV, C>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
    if (err != cudaSuccess) return err;
    const dim3 grid(a.dv / BV, a.HV, a.N), block(kSimtThreads);
    kern<<<grid, block, smem, stream>>>(
        static_cast<const Tin *>(a.q), static_cast<const Tin *>(a.k),
        static_cast<const Tin *>(a.v), a.g, a.beta, a.h0, a.cu_seqlens, a.T, a.HK, a.HV, a.dv,
        a.scale, static_cast<Tin *>(a.o), a.hT, a.prologue, a.gate);
    return cudaGetLastError();
}

template <typename Tin, int DK>
cudaError_t launch_dk(const PrefillArgs &a, cudaStream_t stream) {
    switch (a.chunk) {
        case 16: return launch_shape<Tin, DK, 32, 16>(a, stream);
        case 32: return launch_shape<Tin, DK, 32, 32>(a, stream);
        case 64: return launch_shape<Tin, DK, 32, 64>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

template <typename Tin>
cudaError_t launch_typed(const PrefillArgs &a, cudaStream_t stream) {
    switch (a.dk) {
        case 32: return launch_dk<Tin, 32>(a, stream);
        case 64: return launch_dk<Tin, 64>(a, stream);
        case 128: return launch_dk<Tin, 128>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool prefill_simt_supported(int dk, int dv, int chunk) {
    return (dk == 32 || dk == 64 || dk == 128) && (dv == 32 || dv == 64 || dv == 128) &&
           (chunk == 16 || chunk == 32 || chunk == 64);
}

cudaError_t launch_prefill_simt(const PrefillArgs &a, cudaStream_t stream) {
    if (a.N == 0) return cudaSuccess;
    return a.dtype == GDN_BF16 ? launch_typed<__nv_bfloat16>(a, stream)
                               : launch_typed<float>(a, stream);
}

}  // namespace gdn
