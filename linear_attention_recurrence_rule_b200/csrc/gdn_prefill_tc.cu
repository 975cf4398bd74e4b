// tcgen05 tensor-core prefill (bf16, dk = dv = 128, chunk 64).
#include "gdn_internal.h"

namespace gdn {

bool prefill_tc_supported(int, int, int, gdn_dtype) { return false; }
size_t prefill_tc_workspace(int, int64_t, int, int, bool) { return 0; }
cudaError_t launch_prefill_tc(const PrefillArgs &, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace gdn
