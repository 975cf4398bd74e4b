// Internal launch interface between the C ABI (gdn_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "gdn.h"

namespace gdn {

struct PrefillArgs {
    const void *q, *k, *v;
    const float *g, *beta, *h0;
    const int32_t *cu_seqlens;
    int N;
    int64_t T;       // tokens per sequence (no cu_seqlens) or packed total
    int HK, HV, dk, dv, chunk;
    float scale;
    gdn_dtype dtype;
    void *o;
    float *hT;
    void *workspace;
    size_t workspace_bytes;
    bool keep_status = false;   // leave the workspace status word as earlier calls left it
    unsigned prologue = 0;      // GDN_PROLOGUE_* flags
    const void *gate = nullptr; // output gate factors sigmoid(z), o's layout: fp16 for
                                // bf16 calls, fp32 for fp32 calls
    bool status_only = false;   // tensor-core path: the kernel whose only scratch is the
                                // status word (the workspace-free entry point)
    const void *v_lo = nullptr; // bf16 remainders of v (v + v_lo carries it to ~2^-17;
                                // tensor-core path, the layer prefill's convolved values)
};

struct StepArgs {
    const void *q, *k, *v;
    const float *g, *beta;
    float *state;
    int N, HK, HV, dk, dv;
    float scale;
    gdn_dtype dtype;
    void *o;
    unsigned prologue = 0;
    // layer steps (gdn_recurrent_step_layer): short convolution on v, gate on o
    const float *conv_w = nullptr, *conv_b = nullptr;   // [HV*dv][conv_width], [HV*dv]
    void *conv_state = nullptr;                          // [N][conv_width-1][HV*dv], dtype
    int conv_width = 0;                                  // 0: no convolution
    bool conv_silu = false;
    const void *z = nullptr;                             // gate logits [N][HV][dv], dtype
};

struct VerifyArgs {
    const void *q, *k, *v;
    const float *g, *beta, *state;
    float *states, *u;
    int N, K, HK, HV, dk, dv;
    float scale;
    gdn_dtype dtype;
    void *o;
    unsigned prologue = 0;
    void *workspace = nullptr;   // update-vector form: per (sequence, value head) tables
    size_t workspace_bytes = 0;
    // fused commit-then-verify (prev_K > 0): the previous round's kept drafts
    const void *prev_k = nullptr;
    const float *prev_g = nullptr, *prev_u = nullptr;
    const int32_t *accepted = nullptr;
    int prev_K = 0;
};

// fp32 words of the update-vector form's workspace (gdn_verify.cu); prev_K > 0 adds
// the fused commit's tables
size_t verify_workspace_floats(int N, int K, int HV, int dk, int prev_K = 0);


// decode (gdn_decode.cu)
bool decode_supported(int dk, int dv);
cudaError_t launch_decode(const StepArgs &a, cudaStream_t stream);
cudaError_t launch_verify(const VerifyArgs &a, cudaStream_t stream);
// test-only: the update-vector verify's streaming kernel with a first wait that gives up
cudaError_t launch_verify_wy_timeout_test(const VerifyArgs &a, cudaStream_t stream);
cudaError_t launch_verify_tc_timeout_test(const VerifyArgs &a, cudaStream_t stream);

// Largest draft count of the verify kernels (GDN_VERIFY_MAX_DRAFTS in gdn.h).
constexpr int kVerifyMaxDrafts = 16;

struct CommitDeltasArgs {
    const void *k;
    const float *g, *u;
    const int32_t *accepted;
    float *state;
    int N, K, HK, HV, dk, dv;
    gdn_dtype dtype;
    unsigned prologue = 0;
};
cudaError_t launch_commit_deltas(const CommitDeltasArgs &a, cudaStream_t stream);
cudaError_t launch_commit(const float *states, const int32_t *accepted, float *state, int N, int K,
                          int HV, int dv, int dk, cudaStream_t stream);

// short convolution on the values and output gate (gdn_layer.cu)
struct ConvArgs {
    const void *x;
    const float *weight, *bias;   // [C][width], [C] or null
    void *conv_state;             // [N][width-1][C] dtype, in/out, or null (zeros, not kept)
    const int32_t *cu_seqlens;
    int N;
    int64_t T;                    // tokens per sequence (no cu_seqlens) or packed total
    int C, width;
    bool silu;
    gdn_dtype dtype;
    void *y;
    void *y_lo = nullptr;         // bf16 only: y_lo = y_exact - y, a second output
    const void *z = nullptr;      // gate logits in x's layout [tokens][C] (layer prefill) or null
    void *f = nullptr;            // their factors sigmoid(z): fp16 for bf16, fp32 for fp32
};
constexpr int kConvMaxWidth = 8;
int conv_vector_channels(gdn_dtype dtype);   // channels per 16-byte vector
cudaError_t launch_short_conv(const ConvArgs &a, cudaStream_t stream);
cudaError_t launch_output_gate(void *o, const void *z, int64_t elems, gdn_dtype dtype,
                               cudaStream_t stream);
// sigmoid(z) -> fp16 factors (the layer prefill's gate)
cudaError_t launch_gate_factor(const void *z, void *factors, int64_t elems, gdn_dtype dtype,
                               cudaStream_t stream);

// CUDA-core chunked prefill (gdn_prefill_simt.cu)
bool prefill_simt_supported(int dk, int dv, int chunk);
cudaError_t launch_prefill_simt(const PrefillArgs &a, cudaStream_t stream);

// one decay per value row (GDN_ROW_DECAY): the recurrence token by token, one lane
// group per state row (gdn_prefill_rows.cu)
bool prefill_rows_supported(int dk, int dv);
cudaError_t launch_prefill_rows(const PrefillArgs &a, cudaStream_t stream);


// cluster (1 chain CTA + 3 prep CTAs per value head) tensor-core prefill
// (gdn_prefill_cluster.cu)
bool prefill_cluster_supported(int dk, int dv, int chunk, gdn_dtype dtype);
// device workspace the cluster prefill needs: the status word of its bounded waits
size_t prefill_cluster_workspace(int N, int64_t T, int HV, int chunk, bool varlen);
cudaError_t launch_prefill_cluster(const PrefillArgs &a, cudaStream_t stream);

// tensor-core prefill with the prep results handed over through a ring of chunk
// records in the workspace (gdn_prefill_ring.cu): the default tensor-core path
bool prefill_ring_supported(int dk, int dv, int chunk, gdn_dtype dtype);
// device workspace: the status word and one ring of chunk records per SM id
size_t prefill_ring_workspace(int N, int64_t T, int HV, int chunk, bool varlen);
// timeout_test: the test-only instance whose first on-device wait gives up at once
cudaError_t launch_prefill_ring(const PrefillArgs &a, cudaStream_t stream, bool timeout_test = false);

// validation, workspace check and dispatch of one prefill call (gdn_api.cu)
gdn_status enqueue_prefill(const PrefillArgs &a, cudaStream_t stream);
// workspace bytes of one prefill call (0: none needed)
size_t prefill_workspace_bytes(const PrefillArgs &a);
// status word of the workspace-free prefill's library array (gdn_noalloc.cu)
gdn_status noalloc_read_status(cudaStream_t stream);

}  // namespace gdn
