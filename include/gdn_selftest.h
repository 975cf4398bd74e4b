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

#ifdef __cplusplus
}
#endif

#endif /* GDN_B200_SELFTEST_H */
