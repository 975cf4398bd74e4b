// Self-test of the tcgen05 / TMA building blocks on one CTA.
//
// Runs the four operand patterns the tensor-core prefill uses and returns the
// fp32 accumulators, so a test can compare them with a plain matrix product:
//   D1 = X  * Y^T   X [128x128], Y [64x128]   both K-major, loaded by TMA
//   D2 = Z^T * R^T  Z [64x128] (MN-major A from TMA), R [64x64] (K-major B,
//                   written by threads with the 128B swizzle)
//   D3 = U  * Z     U [128x64] (K-major A, thread-written), Z as MN-major B
//   D4 = D0 - S * W S [128x128] (K-major A, thread-written, negated),
//                   W [128x64] (MN-major B, thread-written), D0 [128x64]
//                   stored into TMEM by tcgen05.st before accumulating.
//   D5 = U  * Z     as D3 but with U packed into TMEM (A operand from TMEM).
// All inputs are row-major bf16 (D0 fp32); outputs row-major fp32.
#include <cuda.h>

#include "gdn.h"
#include "gdn_internal.h"
#include "gdn_selftest.h"
#include "tc_primitives.cuh"
#include "tma_host.h"

namespace gdn {
namespace {

using namespace tc;

constexpr uint32_t kWait = 2000;   // sleeping polls of at most ~1 ms each

constexpr uint32_t OFF_X = 0;          // 2 atom cols x 128 rows = 32 KB
constexpr uint32_t OFF_Y = 32768;      // 2 x 64 rows = 16 KB
constexpr uint32_t OFF_Z = 49152;      // 2 x 64 rows = 16 KB
constexpr uint32_t OFF_R = 65536;      // 64 rows = 8 KB
constexpr uint32_t OFF_U = 73728;      // 128 rows = 16 KB
constexpr uint32_t OFF_S = 90112;      // 2 x 128 rows = 32 KB
constexpr uint32_t OFF_W = 122880;     // 128 rows = 16 KB
constexpr uint32_t OFF_BAR = 139264;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 64 + 1024;

__device__ __forceinline__ void load_row64(const __nv_bfloat16 *src, float *f) {
#pragma unroll
    for (int e = 0; e < 64; ++e) f[e] = __bfloat162float(src[e]);
}

__global__ void __launch_bounds__(128, 1)
umma_selftest_kernel(const __grid_constant__ CUtensorMap tm_x,
                     const __grid_constant__ CUtensorMap tm_y,
                     const __grid_constant__ CUtensorMap tm_z, const __nv_bfloat16 *R,
                     const __nv_bfloat16 *U, const __nv_bfloat16 *S, const __nv_bfloat16 *W,
                     const float *D0, float *D1, float *D2, float *D3, float *D4, float *D5,
                     int *status) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bar_tma = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint64_t *bar_mma = bar_tma + 1;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar_tma + 2);
    const int tid = threadIdx.x, warp = tid >> 5;

    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(tslot, 512);
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;

    if (tid == 0) {
        mbar_arrive_expect_tx(bar_tma, 32768 + 16384 + 16384);
        tma_load_2d(sm + OFF_X, &tm_x, bar_tma, 0, 0);
        tma_load_2d(sm + OFF_X + 16384, &tm_x, bar_tma, 64, 0);
        tma_load_2d(sm + OFF_Y, &tm_y, bar_tma, 0, 0);
        tma_load_2d(sm + OFF_Y + 8192, &tm_y, bar_tma, 64, 0);
        tma_load_2d(sm + OFF_Z, &tm_z, bar_tma, 0, 0);
        tma_load_2d(sm + OFF_Z + 8192, &tm_z, bar_tma, 64, 0);
    }
    // thread-written operands
    {
        float f[64];
        const int i = tid;
        if (i < 64) {
            load_row64(R + i * 64, f);
            st_row64_sw128(sbase + OFF_R, i, f);
        }
        load_row64(U + i * 64, f);
        st_row64_sw128(sbase + OFF_U, i, f);
        load_row64(S + i * 128, f);
        st_row64_sw128(sbase + OFF_S, i, f);
        load_row64(S + i * 128 + 64, f);
        st_row64_sw128(sbase + OFF_S + 16384, i, f);
        load_row64(W + i * 64, f);
        st_row64_sw128(sbase + OFF_W, i, f);
        // D0 row i -> TMEM columns 256..319 (this warp's lane quadrant)
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = D0[i * 64 + p * 16 + j];
            tmem_st16(tmem_addr(tmem, warp, 256 + p * 16), v);
        }
        // U row i packed two bf16 per column -> TMEM columns 448..479
        uint32_t w[32];
#pragma unroll
        for (int c = 0; c < 32; ++c)
            w[c] = pack_bf16x2(__bfloat162float(U[i * 64 + 2 * c]),
                               __bfloat162float(U[i * 64 + 2 * c + 1]));
        tmem_st32(tmem_addr(tmem, warp, 448), w);
        tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    bool ok = mbar_wait(bar_tma, 0, kWait);
    if (tid == 0) {
        tc_fence_after();
        if (ok) {
            // D1 = X * Y^T: M=128, N=64, K=128 (both K-major)
            const uint32_t id1 = idesc_bf16(128, 64, false, false);
            for (int k = 0; k < 8; ++k) {
                const uint32_t ko = (k & 3) * 32;
                uint64_t a = sdesc_sw128(sbase + OFF_X + (k >> 2) * 16384 + ko, 16, 1024);
                uint64_t b = sdesc_sw128(sbase + OFF_Y + (k >> 2) * 8192 + ko, 16, 1024);
                mma_bf16(tmem + 0, a, b, id1, k > 0);
            }
            // D2 = Z^T * R^T: A = Z^T MN-major (M=128 cols of Z, K=64 rows), B = R K-major
            const uint32_t id2 = idesc_bf16(128, 64, true, false);
            for (int k = 0; k < 4; ++k) {
                uint64_t a = sdesc_sw128(sbase + OFF_Z + k * 2048, 8192, 1024);
                uint64_t b = sdesc_sw128(sbase + OFF_R + k * 32, 16, 1024);
                mma_bf16(tmem + 64, a, b, id2, k > 0);
            }
            // D3 = U * Z: A = U K-major, B = Z MN-major (K=64 rows, N=128 cols)
            const uint32_t id3 = idesc_bf16(128, 128, false, true);
            for (int k = 0; k < 4; ++k) {
                uint64_t a = sdesc_sw128(sbase + OFF_U + k * 32, 16, 1024);
                uint64_t b = sdesc_sw128(sbase + OFF_Z + k * 2048, 8192, 1024);
                mma_bf16(tmem + 128, a, b, id3, k > 0);
            }
            // D4 = D0 - S * W: A = S K-major (negated), B = W MN-major (K=128 rows, N=64)
            const uint32_t id4 = idesc_bf16(128, 64, false, true, true);
            for (int k = 0; k < 8; ++k) {
                uint64_t a = sdesc_sw128(sbase + OFF_S + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
                uint64_t b = sdesc_sw128(sbase + OFF_W + k * 2048, 8192, 1024);
                mma_bf16(tmem + 256, a, b, id4, 1);
            }
            // D5 = U(TMEM) * Z: A from TMEM, 8 columns per K step of 16
            for (int k = 0; k < 4; ++k) {
                uint64_t b = sdesc_sw128(sbase + OFF_Z + k * 2048, 8192, 1024);
                mma_bf16_ts(tmem + 320, tmem + 448 + k * 8, b, id3, k > 0);
            }
        }
        mma_commit(bar_mma);
    }
    __syncwarp();
    ok = mbar_wait(bar_mma, 0, kWait) && ok;
    tc_fence_after();
    if (!ok && tid == 0) atomicExch(status, (int)GDN_ERR_TIMEOUT);
    {
        const int i = tid;
        float v[16];
        for (int p = 0; p < 4; ++p) {
            tmem_ld16(tmem_addr(tmem, warp, p * 16), v);
            tmem_wait_ld();
            for (int j = 0; j < 16; ++j) D1[i * 64 + p * 16 + j] = v[j];
            tmem_ld16(tmem_addr(tmem, warp, 64 + p * 16), v);
            tmem_wait_ld();
            for (int j = 0; j < 16; ++j) D2[i * 64 + p * 16 + j] = v[j];
            tmem_ld16(tmem_addr(tmem, warp, 256 + p * 16), v);
            tmem_wait_ld();
            for (int j = 0; j < 16; ++j) D4[i * 64 + p * 16 + j] = v[j];
        }
        for (int p = 0; p < 8; ++p) {
            tmem_ld16(tmem_addr(tmem, warp, 128 + p * 16), v);
            tmem_wait_ld();
            for (int j = 0; j < 16; ++j) D3[i * 128 + p * 16 + j] = v[j];
            tmem_ld16(tmem_addr(tmem, warp, 320 + p * 16), v);
            tmem_wait_ld();
            for (int j = 0; j < 16; ++j) D5[i * 128 + p * 16 + j] = v[j];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

bool map2d(CUtensorMap *m, const void *p, uint64_t cols, uint64_t rows, uint32_t box_rows) {
    uint64_t dims[2] = {cols, rows};
    uint64_t strides[1] = {cols * 2};
    uint32_t box[2] = {64, box_rows};
    return encode_bf16_map(m, p, 2, dims, strides, box);
}

}  // namespace
}  // namespace gdn

extern "C" int gdn_selftest_umma(const void *X, const void *Y, const void *Z, const void *R,
                                 const void *U, const void *S, const void *W, const float *D0,
                                 float *D1, float *D2, float *D3, float *D4, float *D5,
                                 int *status, gdn_stream_t stream) {
    using namespace gdn;
    CUtensorMap tx, ty, tz;
    if (!map2d(&tx, X, 128, 128, 128) || !map2d(&ty, Y, 128, 64, 64) ||
        !map2d(&tz, Z, 128, 64, 64))
        return GDN_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaFuncSetAttribute(umma_selftest_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SMEM_BYTES) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return GDN_ERR_CUDA;
    umma_selftest_kernel<<<1, 128, SMEM_BYTES, s>>>(
        tx, ty, tz, static_cast<const __nv_bfloat16 *>(R), static_cast<const __nv_bfloat16 *>(U),
        static_cast<const __nv_bfloat16 *>(S), static_cast<const __nv_bfloat16 *>(W), D0, D1, D2,
        D3, D4, D5, status);
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// Test-only tensor-core prefill whose first on-device wait gives up at once (see
// gdn_selftest.h): the library's timeout path, exercised without a real hang.
extern "C" int gdn_selftest_prefill_timeout(const void *q, const void *k, const void *v,
                                            const float *g, const float *beta, int N, int64_t T,
                                            int HK, int HV, void *o, float *hT, void *workspace,
                                            size_t workspace_bytes, gdn_stream_t stream) {
    if (!q || !k || !v || !g || !beta || !o || !workspace) return GDN_ERR_INVALID_ARG;
    if (N <= 0 || T <= 0 || HK <= 0 || HV <= 0 || HV % HK) return GDN_ERR_INVALID_ARG;
    gdn::PrefillArgs a{q, k, v, g, beta, nullptr, nullptr, N, T, HK, HV, 128, 128, 64,
                       1.0f, GDN_BF16, o, hT, workspace, workspace_bytes};
    if (workspace_bytes < gdn::prefill_workspace_bytes(a)) return GDN_ERR_WORKSPACE;
    const cudaError_t err = gdn::launch_prefill_ring(a, reinterpret_cast<cudaStream_t>(stream), true);
    return err == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// Test-only update-vector verify streaming kernel whose first wait gives up at once
// (see gdn_selftest.h).
extern "C" int gdn_selftest_verify_timeout(const void *v, const float *state, int N, int K, int HV,
                                           void *o, float *u_out, void *workspace,
                                           size_t workspace_bytes, gdn_stream_t stream) {
    if (!v || !state || !o || !workspace) return GDN_ERR_INVALID_ARG;
    if (N <= 0 || K <= 0 || K > 4 || HV <= 0) return GDN_ERR_INVALID_ARG;
    if (workspace_bytes < gdn_recurrent_verify_workspace_size(N, K, HV, 128)) return GDN_ERR_WORKSPACE;
    gdn::VerifyArgs a{nullptr, nullptr, v, nullptr, nullptr, state, nullptr, u_out, N, K, 1, HV, 128, 128,
                      1.0f, GDN_BF16, o, 0u, workspace, workspace_bytes};
    const cudaError_t err = gdn::launch_verify_wy_timeout_test(a, reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// Test-only tensor-core update-vector verify kernel whose first wait gives up at
// once (see gdn_selftest.h).
extern "C" int gdn_selftest_verify_tc_timeout(const void *v, const float *state, int N, int K,
                                              int HV, void *o, float *u_out, void *workspace,
                                              size_t workspace_bytes, gdn_stream_t stream) {
    if (!v || !state || !o || !workspace) return GDN_ERR_INVALID_ARG;
    if (N <= 0 || K <= 0 || K > 8 || HV <= 0) return GDN_ERR_INVALID_ARG;
    if (workspace_bytes < gdn_recurrent_verify_workspace_size(N, K, HV, 128)) return GDN_ERR_WORKSPACE;
    gdn::VerifyArgs a{nullptr, nullptr, v, nullptr, nullptr, state, nullptr, u_out, N, K, 1, HV, 128, 128,
                      1.0f, GDN_BF16, o, 0u, workspace, workspace_bytes};
    const cudaError_t err = gdn::launch_verify_tc_timeout_test(a, reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}
