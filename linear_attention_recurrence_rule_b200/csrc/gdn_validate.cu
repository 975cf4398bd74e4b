// Opt-in check of a device cu_seqlens array (gdn_chunk_prefill treats its
// contents as a precondition): starts at 0, never decreases, ends at T.
#include <cuda_runtime.h>

#include "gdn.h"

namespace {

// result: 0 when valid, else 1 + the smallest offending index i (entry i breaks
// the rules: i = 0 not zero, i = N not T, otherwise cu[i] < cu[i - 1]).
__global__ void validate_cu_kernel(const int32_t *cu, int N, int64_t T, int *result) {
    __shared__ int first;
    if (threadIdx.x == 0) first = 0x7fffffff;
    __syncthreads();
    for (int i = threadIdx.x; i <= N; i += blockDim.x) {
        bool bad;
        if (i == 0) bad = cu[0] != 0;
        else bad = cu[i] < cu[i - 1];
        if (i == N && (int64_t)cu[N] != T) bad = true;
        if (bad) atomicMin(&first, i);
    }
    __syncthreads();
    if (threadIdx.x == 0) *result = first == 0x7fffffff ? 0 : first + 1;
}

}  // namespace

extern "C" gdn_status gdn_validate_cu_seqlens(const int32_t *cu_seqlens, int N, int64_t T,
                                              int *result, gdn_stream_t stream) {
    if (!cu_seqlens || !result || N < 0 || T < 0) return GDN_ERR_INVALID_ARG;
    validate_cu_kernel<<<1, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(cu_seqlens, N, T,
                                                                            result);
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}
