// C ABI entry points (declared in include/gdn.h): argument validation, workspace
// sizing and dispatch to the kernels.  No allocation, no synchronisation, no
// global state; every launch goes to the caller's stream.
#include <cuda_runtime.h>

#include "gdn.h"
#include "gdn_internal.h"

namespace {

bool aligned16(const void *p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool tc_path(int dk, int dv, int chunk, gdn_dtype dt) {
    return gdn::prefill_cluster_supported(dk, dv, chunk, dt);
}

gdn_status check_prefill(const gdn::PrefillArgs &a) {
    if (!a.q || !a.k || !a.v || !a.g || !a.beta || !a.o) return GDN_ERR_INVALID_ARG;
    if (a.N < 0 || a.T < 0 || a.HK <= 0 || a.HV <= 0 || a.dk <= 0 || a.dv <= 0 || a.chunk <= 0)
        return GDN_ERR_INVALID_ARG;
    if (a.HV % a.HK != 0) return GDN_ERR_INVALID_ARG;
    if (a.dtype != GDN_F32 && a.dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (a.cu_seqlens == nullptr && a.N > 0 && a.T > 0 && (int64_t)a.N * a.T > (int64_t)1 << 40)
        return GDN_ERR_INVALID_ARG;
    if (!gdn::prefill_simt_supported(a.dk, a.dv, a.chunk) && !tc_path(a.dk, a.dv, a.chunk, a.dtype))
        return GDN_ERR_UNSUPPORTED;
    if (!aligned16(a.q) || !aligned16(a.k) || !aligned16(a.v) || !aligned16(a.o) ||
        !aligned16(a.h0) || !aligned16(a.hT))
        return GDN_ERR_ALIGNMENT;
    return GDN_OK;
}

}  // namespace

extern "C" {

const char *gdn_status_string(gdn_status s) {
    switch (s) {
        case GDN_OK: return "ok";
        case GDN_ERR_INVALID_ARG: return "invalid argument";
        case GDN_ERR_UNSUPPORTED: return "unsupported shape, chunk or dtype";
        case GDN_ERR_ALIGNMENT: return "buffer not 16-byte aligned";
        case GDN_ERR_CUDA: return "CUDA error";
        case GDN_ERR_TIMEOUT: return "on-device wait timed out";
        case GDN_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

int gdn_version(void) { return 100; }

int gdn_chunk_prefill_path(int dk, int dv, int chunk, gdn_dtype dtype) {
    if (tc_path(dk, dv, chunk, dtype)) return 1;
    if ((dtype == GDN_F32 || dtype == GDN_BF16) && gdn::prefill_simt_supported(dk, dv, chunk))
        return 0;
    return -1;
}

size_t gdn_chunk_prefill_workspace_size(int N, int64_t T, int HK, int HV, int dk, int dv,
                                        int chunk, gdn_dtype dtype, int varlen) {
    if (N < 0 || T < 0 || HK <= 0 || HV <= 0 || HV % HK || chunk <= 0) return 0;
    if (tc_path(dk, dv, chunk, dtype)) return gdn::prefill_cluster_workspace(N, T, HV, chunk, varlen != 0);
    return 0;
}

gdn_status gdn_chunk_prefill(const void *q, const void *k, const void *v, const float *g,
                             const float *beta, const float *h0, const int32_t *cu_seqlens,
                             int N, int64_t T, int HK, int HV, int dk, int dv, int chunk,
                             float scale, gdn_dtype dtype, void *o, float *hT, void *workspace,
                             size_t workspace_bytes, gdn_stream_t stream) {
    gdn::PrefillArgs a{q, k, v, g, beta, h0, cu_seqlens, N, T, HK, HV, dk, dv, chunk,
                       scale, dtype, o, hT, workspace, workspace_bytes};
    gdn_status st = check_prefill(a);
    if (st != GDN_OK) return st;
    if (N == 0) return GDN_OK;
    cudaError_t err;
    if (tc_path(dk, dv, chunk, dtype)) {
        const size_t need = gdn::prefill_cluster_workspace(N, T, HV, chunk, cu_seqlens != nullptr);
        if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return GDN_ERR_WORKSPACE;
        if (!aligned16(workspace)) return GDN_ERR_ALIGNMENT;
        err = gdn::launch_prefill_cluster(a, reinterpret_cast<cudaStream_t>(stream));
    } else {
        err = gdn::launch_prefill_simt(a, reinterpret_cast<cudaStream_t>(stream));
    }
    return err == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status gdn_recurrent_step(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, float *state, int N, int HK, int HV, int dk,
                              int dv, float scale, gdn_dtype dtype, void *o,
                              gdn_stream_t stream) {
    if (!q || !k || !v || !g || !beta || !state || !o) return GDN_ERR_INVALID_ARG;
    if (N < 0 || HK <= 0 || HV <= 0 || dk <= 0 || dv <= 0 || HV % HK) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if ((int64_t)N * HV > 0x7fffffff) return GDN_ERR_UNSUPPORTED;
    if (!gdn::decode_supported(dk, dv)) return GDN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(state))
        return GDN_ERR_ALIGNMENT;
    if (N == 0) return GDN_OK;
    gdn::StepArgs a{q, k, v, g, beta, state, N, HK, HV, dk, dv, scale, dtype, o};
    const cudaError_t err = gdn::launch_decode(a, reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status gdn_read_status(const void *workspace, size_t workspace_bytes, gdn_stream_t stream) {
    if (workspace == nullptr || workspace_bytes < sizeof(unsigned int)) return GDN_OK;
    unsigned int word = 0;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return GDN_ERR_CUDA;
    return word == 0 ? GDN_OK : GDN_ERR_TIMEOUT;
}

}  // extern "C"
