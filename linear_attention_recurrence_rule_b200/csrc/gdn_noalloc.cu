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
// up with that device current, once per device (a failed lookup is not kept:
// the next call tries again).  A cached address belongs to the device's primary
// context: after cudaDeviceReset the next call must not reuse it, which the
// header states.
constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices];

cudaError_t scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

namespace gdn {

// The status word of the library array (the waits of the last workspace-free
// prefill on the current device): GDN_OK, GDN_ERR_TIMEOUT, or GDN_ERR_CUDA.
gdn_status noalloc_read_status(cudaStream_t stream) {
    void *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return GDN_ERR_CUDA;
    unsigned int word = 0;
    if (cudaMemcpyAsync(&word, scratch, sizeof(word), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return GDN_ERR_CUDA;
    return word == 0 ? GDN_OK : GDN_ERR_TIMEOUT;
}

}  // namespace gdn

extern "C" gdn_status gdn_chunk_prefill_noalloc(const void *q, const void *k, const void *v,
                                                const float *g, const float *beta,
                                                const float *h0, const int32_t *cu_seqlens,
                                                int N, int64_t T, int HK, int HV, int dk, int dv,
                                                int chunk, float scale, gdn_dtype dtype, void *o,
                                                float *hT, gdn_stream_t stream) {
    // on the tensor-core path: the kernel whose only scratch is the status word of
    // its bounded waits (the default prefill also needs a ring of chunk records)
    gdn::PrefillArgs a{q, k, v, g, beta, h0, cu_seqlens, N, T, HK, HV, dk, dv, chunk,
                       scale, dtype, o, hT, nullptr, 0};
    a.status_only = true;
    const size_t need = gdn::prefill_workspace_bytes(a);
    if (need > kNoAllocScratchBytes) return GDN_ERR_WORKSPACE;
    if (need > 0) {
        void *scratch = nullptr;
        if (scratch_address(&scratch) != cudaSuccess) return GDN_ERR_CUDA;
        a.workspace = scratch;
        a.workspace_bytes = kNoAllocScratchBytes;
    }
    // the prefill clears the status word it relies on before its kernel runs
    return gdn::enqueue_prefill(a, reinterpret_cast<cudaStream_t>(stream));
}
