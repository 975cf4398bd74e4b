/*
 * gdn_selftest.h -- self-test entry point of the tensor-core building blocks.
 *
 * Not part of the gated delta rule itself (the pages have no counterpart): it
 * checks on one CTA that the library's shared-memory descriptors, TMA tile
 * loads, tcgen05 MMAs and TMEM loads/stores compute plain matrix products, in
 * exactly the operand layouts the tensor-core prefill relies on.
 */
#ifndef GDN_B200_SELFTEST_H
#define GDN_B200_SELFTEST_H

#include "gdn.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * All pointers are device pointers; inputs row-major bf16 unless noted:
 *   X [128][128], Y [64][128], Z [64][128], R [64][64], U [128][64],
 *   S [128][128], W [128][64], D0 [128][64] fp32.
 * Outputs (row-major fp32):
 *   D1 [128][64]  = X Y^T          D2 [128][64] = Z^T R^T
 *   D3 [128][128] = U Z            D4 [128][64] = D0 - S W
 *   D5 [128][128] = U Z with U read from tensor memory (A operand in TMEM)
 * status (device int) is set to GDN_ERR_TIMEOUT if an on-device wait gave up.
 * X, Y, Z must be 16-byte aligned.  Returns a gdn_status; asynchronous.
 */
GDN_API int gdn_selftest_umma(const void *X, const void *Y, const void *Z, const void *R,
                              const void *U, const void *S, const void *W, const float *D0,
                              float *D1, float *D2, float *D3, float *D4, float *D5,
                              int *status, gdn_stream_t stream);

/*
 * Test-only instance of the tensor-core prefill (bf16, dk = dv = 128, chunk 64;
 * same layouts as gdn_chunk_prefill, h0 = 0, scale 1) whose first on-device
 * wait -- before any load, copy or MMA is issued -- has a limit of zero polls
 * on a barrier that nothing arrives on.  It exercises the library's timeout
 * path without a real hang: the wait gives up, the status word in `workspace`
 * becomes GDN_ERR_TIMEOUT (read it with gdn_read_status), every CTA of each
 * cluster winds down without work, and the kernel returns.  o and hT are then
 * undefined.  workspace: gdn_chunk_prefill_workspace_size(...) bytes.  Returns
 * GDN_OK once enqueued, GDN_ERR_INVALID_ARG / GDN_ERR_WORKSPACE / GDN_ERR_CUDA.
 */
GDN_API int gdn_selftest_prefill_timeout(const void *q, const void *k, const void *v,
                                         const float *g, const float *beta, int N, int64_t T,
                                         int HK, int HV, void *o, float *hT, void *workspace,
                                         size_t workspace_bytes, gdn_stream_t stream);

/*
 * Test-only instance of the update-vector verify's streaming kernel (dk = dv = 128,
 * K <= 4 drafts, bf16 v/o): its first on-device wait, before any copy is issued,
 * has a limit of zero polls on a barrier nothing arrives on, so the kernel records
 * a timeout in the workspace status word (gdn_read_status then returns
 * GDN_ERR_TIMEOUT) and returns with nothing in flight.  v [N][K][HV][128] bf16,
 * state [N][HV][128][128] fp32 (only read), o, u_out as gdn_recurrent_verify (left
 * unwritten); workspace: gdn_recurrent_verify_workspace_size(N, K, HV, 128) bytes.
 */
GDN_API int gdn_selftest_verify_timeout(const void *v, const float *state, int N, int K, int HV,
                                        void *o, float *u_out, void *workspace,
                                        size_t workspace_bytes, gdn_stream_t stream);

/*
 * The same for the tensor-core form of the update-vector verify (bf16 v/o,
 * dk = dv = 128, K <= 8 drafts; the form gdn_recurrent_verify runs for those
 * shapes): before any copy or MMA is issued, its first wait has a limit of zero
 * polls on a barrier nothing arrives on; the status word records the timeout, the
 * CTA frees its tensor memory and returns.  Arguments as gdn_selftest_verify_timeout
 * (state 16-byte aligned); 1 <= K <= 8.
 */
GDN_API int gdn_selftest_verify_tc_timeout(const void *v, const float *state, int N, int K,
                                           int HV, void *o, float *u_out, void *workspace,
                                           size_t workspace_bytes, gdn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GDN_B200_SELFTEST_H */
