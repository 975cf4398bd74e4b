// Prefill entry point for callers that cannot allocate device memory.
//
// gdn_chunk_prefill needs a small caller-provided device workspace (the status
// word of its on-device waits).  Some callers cannot make that allocation: a
// plugin or serving loop that runs under a fixed, pre-reserved memory budget,
// code that must not call cudaMalloc on its hot path because the call can
// synchronise the device and stall other streams, or a host API that offers
// no workspace at all.  gdn_chunk_prefill_noalloc serves them by keeping that
// scratch in a fixed-size array inside the library instead.
#include <cuda_runtime.h>

#include <mutex>

#include "gdn.h"
#include "gdn_internal.h"

namespace {

// The library's own scratch: every device that loads the library holds these
// bytes until the process exits.  Every call on a device uses the same array.
constexpr size_t kNoAllocScratchBytes = 256;
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Host code cannot pass g_noalloc_scratch itself to a kernel (in host code the
// name is only a stand-in for the device array); its device address is looked
// up once per device, with that device current.
constexpr int kMaxDevices = 64;
std::once_flag g_once[kMaxDevices];
void *g_scratch_addr[kMaxDevices];
cudaError_t g_scratch_err[kMaxDevices];

cudaError_t scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::call_once(g_once[dev], [dev]() {
        g_scratch_err[dev] = cudaGetSymbolAddress(&g_scratch_addr[dev], g_noalloc_scratch);
    });
    if (g_scratch_err[dev] != cudaSuccess) return g_scratch_err[dev];
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" gdn_status gdn_chunk_prefill_noalloc(const void *q, const void *k, const void *v,
                                                const float *g, const float *beta,
                                                const float *h0, const int32_t *cu_seqlens,
                                                int N, int64_t T, int HK, int HV, int dk, int dv,
                                                int chunk, float scale, gdn_dtype dtype, void *o,
                                                float *hT, gdn_stream_t stream) {
    const size_t need = gdn_chunk_prefill_workspace_size(N, T, HK, HV, dk, dv, chunk, dtype,
                                                         cu_seqlens != nullptr);
    if (need > kNoAllocScratchBytes) return GDN_ERR_WORKSPACE;
    void *scratch = nullptr;
    if (need > 0 && scratch_address(&scratch) != cudaSuccess) return GDN_ERR_CUDA;
    // the prefill clears the status word it relies on before its kernel runs
    return gdn_chunk_prefill(q, k, v, g, beta, h0, cu_seqlens, N, T, HK, HV, dk, dv, chunk,
                             scale, dtype, o, hT, scratch, need > 0 ? kNoAllocScratchBytes : 0,
                             stream);
}
