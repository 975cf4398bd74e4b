/*
 * gdn.h -- C ABI of the B200 (sm_100a) gated delta rule library.
 *
 * The operation (sources: "Qwen3-Next", sghael.github.io, section "Correcting
 * a memory instead of adding to it"; model card "Qwen3-Next-80B-A3B-Instruct",
 * section "Model Overview", Gated DeltaNet heads; "The Evolving Transformer /
 * Qwen3-Next", section 01 GatedDeltaNet, for the state orientation and the
 * read-out after the update):
 *
 *   For every sequence n and value head h (reading query/key head
 *   c = floor(h / (HV / HK))), with S a dv x dk fp32 matrix (row = value
 *   index, column = key index) starting at h0[n][h] (or zero):
 *
 *     S_t = alpha_t * S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *     o_t = scale * S_t q_t            alpha_t = exp(g_t)
 *
 *   i.e. the old memory is first shrunk by the decay, then corrected along the
 *   current key by the write strength beta_t (the page's scalar example:
 *   6 -> 3 -> 3 + 0.5 * (10 - 3) = 6.5).  q and k are expected to be
 *   L2-normalised by the caller; the library does not renormalise.
 *
 * Conventions shared by every call
 *   - All pointers are DEVICE pointers of the current CUDA device unless a
 *     comment says otherwise (gdn_chunk_prefill_host takes host buffers).  The
 *     caller owns every buffer; the library keeps no allocation and no global
 *     state, never synchronises the stream, and returns as soon as the work is
 *     enqueued.
 *   - Tensors are dense, row-major, with the last dimension contiguous.
 *   - dtype selects the element type of q, k, v and o: GDN_F32 (float) or
 *     GDN_BF16 (__nv_bfloat16).  g, beta, h0, hT and the decode state are
 *     always fp32.  Internal accumulation and the recurrent state are fp32.
 *   - Host-checkable problems (NULL where a buffer is required, HV % HK != 0,
 *     an unsupported shape/dtype/chunk combination, a misaligned base pointer,
 *     a short workspace) return an error before anything is enqueued.  A failed
 *     kernel launch returns GDN_ERR_CUDA.  There is no fallback to another
 *     implementation or to the CPU.
 *   - The contents of cu_seqlens are a precondition (see below) and are not
 *     checked on the host.
 */
#ifndef GDN_B200_H
#define GDN_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GDN_API __attribute__((visibility("default")))
#else
#define GDN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t.  NULL selects the legacy default stream. */
typedef struct CUstream_st *gdn_stream_t;

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,   /* NULL buffer, non-positive size, HV % HK != 0 ... */
    GDN_ERR_UNSUPPORTED = 2,   /* valid but not implemented: head dim, chunk, dtype */
    GDN_ERR_ALIGNMENT = 3,     /* a base pointer is not 16-byte aligned            */
    GDN_ERR_CUDA = 4,          /* a CUDA runtime/driver call or launch failed       */
    GDN_ERR_TIMEOUT = 5,       /* a bounded on-device wait gave up (reported through
                                  the workspace status word, see gdn_read_status)   */
    GDN_ERR_WORKSPACE = 6      /* workspace missing or smaller than required        */
} gdn_status;

typedef enum { GDN_F32 = 0, GDN_BF16 = 1 } gdn_dtype;

/* Short English description of a status code (static storage, never NULL). */
GDN_API const char *gdn_status_string(gdn_status s);

/* Library version, major * 10000 + minor * 100 + patch. */
GDN_API int gdn_version(void);

/*
 * Bytes of device workspace gdn_chunk_prefill needs for this problem.
 * N: number of sequences; T: tokens per sequence without cu_seqlens, else the
 * packed total; varlen: nonzero when cu_seqlens will be passed.  Returns 0 for
 * arguments gdn_chunk_prefill would reject.  On the tensor-core path (bf16,
 * dk = dv = 128, chunk 64) the workspace holds a status word and, per SM of the
 * current device, a ring of six 65 KB chunk records through which the kernel's
 * prep CTAs hand their results to its chain CTA (~59 MB on a 148-SM B200,
 * independent of N and T); the size is computed for the device current at the
 * time of the query.
 */
GDN_API size_t gdn_chunk_prefill_workspace_size(int N, int64_t T, int HK, int HV, int dk, int dv,
                                        int chunk, gdn_dtype dtype, int varlen);

/*
 * Input prologue flags (bitwise OR; 0 = the inputs are already prepared).
 * They fuse the layer steps just before the rule into the kernels ("The
 * Evolving Transformer / Qwen3-Next", section 01 GatedDeltaNet: keys are
 * L2-normalised, the write strength and the forget gate are sigmoids of their
 * logits; queries are normalised like keys in the model):
 *   GDN_PROLOGUE_NORM_Q       each q row (per QK head, over dk) is replaced by
 *                             q / max(|q|, 1e-12), computed in fp32 from the
 *                             stored values
 *   GDN_PROLOGUE_NORM_K       the same for k
 *   GDN_PROLOGUE_GATE_LOGITS  `g` holds forget logits a and `beta` write logits
 *                             b: alpha = sigmoid(a) (g = log sigmoid(a)) and
 *                             beta = sigmoid(b)
 * No normalised copy is written: the norms are folded into the scalings the
 * kernels already apply.
 */
#define GDN_PROLOGUE_NORM_Q 1u
#define GDN_PROLOGUE_NORM_K 2u
#define GDN_PROLOGUE_GATE_LOGITS 4u
#define GDN_PROLOGUE_ALL 7u

/*
 * GDN_ROW_DECAY (same flag word): one decay per value row instead of one per
 * head -- the teaching code's per-channel forget gate, which scales the rows of
 * the state ("The Evolving Transformer / Qwen3-Next", section 01 GatedDeltaNet).
 * `g` (or, with GDN_PROLOGUE_GATE_LOGITS, its logits) then has one entry per
 * value row: [N][HV][dv] for gdn_recurrent_step_ex, [N][K][HV][dv] for
 * gdn_recurrent_verify and gdn_state_commit_deltas.  Each row i of a state
 * decays by its own alpha_i before the correction.  Supported by the decode
 * step, by verify when states_out is given, by both commits, and by the
 * prefill (`g` [B][T][HV][dv]) for every supported shape, which then runs the
 * recurrence token by token on CUDA cores, one lane group per state row (the
 * rows never mix under this rule; the tensor-core path's per-head triangular
 * inverse would become one per row, so it is not used; `chunk` is checked but
 * does not shape that computation).  The update-vector-only verify and the fused
 * commit-then-verify take it too: their one-pass kernel mixes the drafts per
 * head, which row decays would make per row, so with GDN_ROW_DECAY the verify
 * runs the per-draft kernel without writing states, and the fused call runs the
 * deltas commit and then that verify (two passes over the states).
 */
#define GDN_ROW_DECAY 8u
#define GDN_FLAGS_VALID 15u

/*
 * 1 when gdn_chunk_prefill runs this (head dims, chunk, dtype) combination on
 * the tcgen05 tensor-core path, 0 when it runs on the CUDA-core path, -1 when
 * the combination is unsupported.  Pure host query.
 */
GDN_API int gdn_chunk_prefill_path(int dk, int dv, int chunk, gdn_dtype dtype);

/*
 * Chunkwise prefill: runs the rule over whole sequences.
 *
 * The sequence is cut into chunks of `chunk` tokens (the last one may be
 * short; chunks restart at every sequence start).  Within a chunk the tokens
 * are processed in the WY/UT form derived from the recurrence: a chunk-local
 * running sum G of g, the unit-lower-triangular system (I + A) with
 * A_ij = beta_i exp(G_i - G_j) k_i.k_j (j < i), intra-chunk products on the
 * tensor cores, and a sequential pass over chunks that carries the fp32 state.
 * The result equals the token-by-token recurrence up to rounding.
 *
 * Layouts (B = N without cu_seqlens; with cu_seqlens everything is packed as a
 * single batch row of Ttot = T tokens):
 *   q, k   [B][T][HK][dk]  dtype          v, o   [B][T][HV][dv]  dtype
 *   g      [B][T][HV] fp32 (log decay, g <= 0 expected; alpha = exp(g))
 *   beta   [B][T][HV] fp32 (write strength, expected in [0, 1])
 *   h0     [N][HV][dv][dk] fp32, or NULL for a zero start state
 *   hT     [N][HV][dv][dk] fp32 final states, or NULL to skip; may alias h0
 *   cu_seqlens  NULL, or N+1 int32 device offsets with cu_seqlens[0] = 0,
 *               non-decreasing, cu_seqlens[N] = T (precondition, unchecked)
 * Supported: HV % HK == 0; dtype GDN_BF16 or GDN_F32; dk, dv in {32, 64, 128};
 * chunk in {16, 32, 64}.  (bf16, dk = dv = 128, chunk = 64 runs on the
 * tcgen05 tensor-core path; other combinations run on the CUDA-core path.)
 * Alignment: q, k, v, o, h0, hT must be 16-byte aligned.
 * workspace: device buffer of at least gdn_chunk_prefill_workspace_size(...)
 * bytes (may be NULL when that size is 0); its contents need no initialisation
 * and are scratch after the call.  Calls that share a workspace must be
 * ordered on the device (same stream or synchronised).
 */
GDN_API gdn_status gdn_chunk_prefill(const void *q, const void *k, const void *v, const float *g,
                             const float *beta, const float *h0, const int32_t *cu_seqlens,
                             int N, int64_t T, int HK, int HV, int dk, int dv, int chunk,
                             float scale, gdn_dtype dtype, void *o, float *hT,
                             void *workspace, size_t workspace_bytes, gdn_stream_t stream);

/*
 * gdn_chunk_prefill with the input prologue fused (`prologue`: GDN_PROLOGUE_*
 * flags; 0 is exactly gdn_chunk_prefill).  With GDN_PROLOGUE_GATE_LOGITS, g
 * and beta hold the logits (any real values).  Unknown flag bits return
 * GDN_ERR_INVALID_ARG; with GDN_ROW_DECAY (g [B][T][HV][dv]) the call runs on the
 * CUDA-core path.
 */
GDN_API gdn_status gdn_chunk_prefill_ex(const void *q, const void *k, const void *v,
                                        const float *g, const float *beta, const float *h0,
                                        const int32_t *cu_seqlens, int N, int64_t T, int HK,
                                        int HV, int dk, int dv, int chunk, float scale,
                                        gdn_dtype dtype, void *o, float *hT, void *workspace,
                                        size_t workspace_bytes, unsigned prologue,
                                        gdn_stream_t stream);

/*
 * gdn_chunk_prefill without a caller-provided workspace.  (The source pages
 * have no counterpart: this is a library convenience, not part of the rule.)
 *
 * For callers that cannot allocate device memory -- code running under a
 * fixed, pre-reserved memory budget, a hot path that must not call cudaMalloc
 * (it can synchronise the device and stall other streams), or a host API that
 * offers no workspace.  Same arguments and layouts as gdn_chunk_prefill;
 * the scratch it needs lives in a 256-byte array inside the
 * library that every device loading the library keeps until the process exits.
 *   - Problems needing more than 256 bytes of workspace (see
 *     gdn_chunk_prefill_workspace_size) return GDN_ERR_WORKSPACE.
 *   - The first call on a device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *   - All calls on a device share the array and leave their contents in it:
 *     calls whose work overlaps on the GPU (different streams, not ordered)
 *     race on it.  Order them on one stream, or use gdn_chunk_prefill with
 *     separate workspaces.
 *   - Whether the on-device waits of the last call completed: gdn_read_status
 *     with a NULL workspace reads the array's status word.
 *   - The looked-up address belongs to the device's primary context: after
 *     cudaDeviceReset, do not call it again in the same process.
 *   - It allocates nothing and calls no allocating routine.
 *   - On the tensor-core path it runs the cluster kernel whose only scratch is
 *     that status word (gdn_chunk_prefill runs the faster kernel that also needs
 *     a ring of chunk records in its workspace); its results agree with
 *     gdn_chunk_prefill's within the bf16 tolerance, not bit for bit.
 */
GDN_API gdn_status gdn_chunk_prefill_noalloc(const void *q, const void *k, const void *v,
                                             const float *g, const float *beta, const float *h0,
                                             const int32_t *cu_seqlens, int N, int64_t T, int HK,
                                             int HV, int dk, int dv, int chunk, float scale,
                                             gdn_dtype dtype, void *o, float *hT,
                                             gdn_stream_t stream);

/*
 * Opt-in check of a device cu_seqlens array before gdn_chunk_prefill (which
 * takes its contents as a precondition): one small kernel on `stream` writes to
 * the DEVICE int *result 0 when cu_seqlens[0] = 0, the entries never decrease
 * and cu_seqlens[N] = T, else 1 + the first offending index.  Returns
 * GDN_ERR_INVALID_ARG for NULL pointers or negative sizes, GDN_ERR_CUDA if the
 * launch fails.
 */
GDN_API gdn_status gdn_validate_cu_seqlens(const int32_t *cu_seqlens, int N, int64_t T,
                                           int *result, gdn_stream_t stream);

/*
 * Bytes of device workspace gdn_chunk_prefill_host needs (0 for arguments it
 * would reject).  segment: tokens per segment, 0 selects the default (4096).
 */
GDN_API size_t gdn_chunk_prefill_host_workspace_size(int N, int64_t T, int HK, int HV, int dk,
                                                     int dv, int chunk, gdn_dtype dtype,
                                                     int64_t segment);

/*
 * gdn_chunk_prefill for inputs and outputs in HOST memory, streamed.  (The
 * source pages have no counterpart: a library convenience for prefills whose
 * data lives on the host.)
 *
 * The N sequences of T tokens are processed in segments of `segment` tokens:
 * while segment s runs on `stream`, the inputs of segment s + 1 are copied in on
 * `copy_in` and the outputs of segment s - 1 are copied out on `copy_out`; the
 * state goes from one segment to the next in device memory.  The result equals
 * gdn_chunk_prefill over the whole sequences (chunks restart at every segment
 * start, which does not change the result; segments that are multiples of
 * `chunk` give bit-identical results).
 *   q, k, v, g, beta, o  HOST pointers, layouts as gdn_chunk_prefill without
 *                        cu_seqlens ([N][T][H][d]); page-locked memory lets the
 *                        copies overlap the computation, pageable memory works
 *                        but serialises them.  16-byte aligned.
 *   h0, hT               DEVICE pointers [N][HV][dv][dk] fp32, or NULL (zero start
 *                        state / final state not wanted); hT may alias h0.
 *   workspace            device buffer of at least
 *                        gdn_chunk_prefill_host_workspace_size(...) bytes,
 *                        256-byte aligned; scratch after the call, and the status
 *                        word of gdn_read_status (sticky over all segments).
 *   stream, copy_in, copy_out  three caller-owned streams (they may coincide, at
 *                        the price of overlap).  The call orders itself after work
 *                        already queued on `stream`, and every copy and kernel it
 *                        enqueues completes before later work on `stream`.
 * It creates and destroys 7 CUDA events per call, whatever the number of
 * segments (released by the runtime once they complete), does not synchronise,
 * and allocates no memory.
 * Errors as gdn_chunk_prefill; GDN_ERR_CUDA if an enqueue fails part way (the
 * work already enqueued then still runs).
 */
GDN_API gdn_status gdn_chunk_prefill_host(const void *q, const void *k, const void *v,
                                          const float *g, const float *beta, const float *h0,
                                          int N, int64_t T, int HK, int HV, int dk, int dv,
                                          int chunk, float scale, gdn_dtype dtype, void *o,
                                          float *hT, void *workspace, size_t workspace_bytes,
                                          int64_t segment, gdn_stream_t stream,
                                          gdn_stream_t copy_in, gdn_stream_t copy_out);

/*
 * Fused single-token decode step for N independent sequences: applies one
 * token of the rule to each sequence's state in place and writes its output.
 * Every state element is read once and written once (one pass through HBM).
 *
 * Layouts:
 *   q, k   [N][HK][dk] dtype      v, o [N][HV][dv] dtype
 *   g, beta [N][HV] fp32          state [N][HV][dv][dk] fp32, updated in place
 * Supported: HV % HK == 0; dtype GDN_BF16 or GDN_F32; dk in {32, 64, 128};
 * 1 <= dv <= 256.  Alignment: q, k, v, o, state 16-byte aligned.
 * o must not overlap state.
 */
GDN_API gdn_status gdn_recurrent_step(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, float *state, int N, int HK, int HV, int dk,
                              int dv, float scale, gdn_dtype dtype, void *o,
                              gdn_stream_t stream);

/*
 * gdn_recurrent_step with the input prologue fused (`prologue`: GDN_PROLOGUE_*
 * flags, and GDN_ROW_DECAY for one decay per value row with g [N][HV][dv];
 * 0 is exactly gdn_recurrent_step).  Unknown flag bits return
 * GDN_ERR_INVALID_ARG.
 */
GDN_API gdn_status gdn_recurrent_step_ex(const void *q, const void *k, const void *v,
                                         const float *g, const float *beta, float *state, int N,
                                         int HK, int HV, int dk, int dv, float scale,
                                         gdn_dtype dtype, void *o, unsigned prologue,
                                         gdn_stream_t stream);

/* Largest number of draft tokens gdn_recurrent_verify takes per sequence. */
#define GDN_VERIFY_MAX_DRAFTS 16

/*
 * Multi-token verify step for speculative decoding (Qwen3-Next, section "Speed
 * depends on the serving software": drafted tokens are verified together and
 * only an accepted prefix is kept).  For each of N sequences, K draft tokens
 * are run through the recurrence of gdn_recurrent_step one after another,
 * starting from `state`, which is only read (once, from HBM, for all K
 * tokens).  Every token's output is written; for rolling back to the last
 * accepted draft the call also writes, when the pointer is not NULL:
 *   states_out  the state AFTER every token (pair with gdn_state_commit), or
 *   u_out       every token's update vector u_t = beta_t (v_t - alpha_t S_{t-1} k_t),
 *               with which S_t = alpha_t S_{t-1} + u_t k_t^T (pair with
 *               gdn_state_commit_deltas: K*dv floats per head instead of K
 *               states, the cheaper form in HBM traffic).
 *
 * Layouts (token t of sequence n is row n*K + t):
 *   q, k   [N][K][HK][dk] dtype      v, o [N][K][HV][dv] dtype
 *   g, beta [N][K][HV] fp32          state [N][HV][dv][dk] fp32 (read)
 *   states_out [N][K][HV][dv][dk] fp32   u_out [N][K][HV][dv] fp32
 * prologue: GDN_PROLOGUE_* flags applied to every draft (0 = prepared inputs);
 * GDN_ROW_DECAY: g [N][K][HV][dv]; without states_out it runs the per-draft
 * kernel writing no states (the workspace is checked but not used).
 * workspace: device scratch of at least gdn_recurrent_verify_workspace_size()
 * bytes, 16-byte aligned, needed when states_out is NULL (the update-vector
 * form builds per (sequence, value head) tables there; ignored otherwise, may
 * be NULL); missing or too small returns GDN_ERR_WORKSPACE.
 * Precision: the update-vector form with bf16 inputs, dk = dv = 128 and K <= 8
 * (no row decays) takes the products of the fp32 state with its mixed key and
 * query vectors on tensor cores, both factors split into bf16 hi + lo parts
 * (each term exact up to ~2^-17 relative, the order of fp32 accumulation);
 * every other form accumulates in fp32 on CUDA cores.
 * Supported: as gdn_recurrent_step, and 1 <= K <= GDN_VERIFY_MAX_DRAFTS.
 * Alignment: q, k, v, o, state, states_out 16-byte aligned, u_out 4-byte.
 * No output may overlap an input.  K > GDN_VERIFY_MAX_DRAFTS returns
 * GDN_ERR_UNSUPPORTED.  N == 0 is an empty batch (GDN_OK, nothing launched;
 * pointers may be NULL).
 */
GDN_API gdn_status gdn_recurrent_verify(const void *q, const void *k, const void *v,
                                        const float *g, const float *beta, const float *state,
                                        int N, int K, int HK, int HV, int dk, int dv, float scale,
                                        gdn_dtype dtype, void *o, float *states_out, float *u_out,
                                        unsigned prologue, void *workspace,
                                        size_t workspace_bytes, gdn_stream_t stream);

/*
 * Bytes of device workspace gdn_recurrent_verify needs when states_out is NULL:
 * (2 K dk + 2 K^2) fp32 words per (sequence, value head), rounded up to 16
 * bytes.  0 for invalid sizes.  Pure host query.
 */
GDN_API size_t gdn_recurrent_verify_workspace_size(int N, int K, int HV, int dk);

/*
 * One speculative-decoding round in one pass over the states: first keeps the
 * previous round's accepted drafts (exactly gdn_state_commit_deltas with prev_k,
 * prev_g, prev_u, accepted), writing `state` in place for every sequence that kept
 * at least one draft, then verifies this round's K drafts from the committed
 * state (exactly gdn_recurrent_verify in its update-vector form: o and u_out, the
 * latter for the next round's commit).  Each state element is read once, and
 * written once where a draft was kept -- against three passes for the two calls.
 *
 * Layouts: prev_k [N][prev_K][HK][dk] dtype, prev_g [N][prev_K][HV] fp32,
 * prev_u [N][prev_K][HV][dv] fp32, accepted [N] int32 (device; 0 or out of range
 * = nothing kept); the rest as gdn_recurrent_verify.  `prologue` applies to both
 * rounds' drafts; with GDN_ROW_DECAY (prev_g and g with a trailing dv axis) the
 * call runs gdn_state_commit_deltas and then the verify, two passes.
 * workspace: at least gdn_recurrent_commit_verify_workspace_size() bytes,
 * 16-byte aligned; its first word is the status of the call's bounded waits
 * (gdn_read_status).  Supported: as gdn_recurrent_verify, 1 <= prev_K <= 16.
 */
GDN_API gdn_status gdn_recurrent_commit_verify(const void *prev_k, const float *prev_g,
                                               const float *prev_u, const int32_t *accepted,
                                               int prev_K, const void *q, const void *k,
                                               const void *v, const float *g, const float *beta,
                                               float *state, int N, int K, int HK, int HV, int dk,
                                               int dv, float scale, gdn_dtype dtype, void *o,
                                               float *u_out, unsigned prologue, void *workspace,
                                               size_t workspace_bytes, gdn_stream_t stream);

/* Workspace bytes of gdn_recurrent_commit_verify (0 for invalid sizes). */
GDN_API size_t gdn_recurrent_commit_verify_workspace_size(int N, int prev_K, int K, int HV,
                                                          int dk);

/*
 * Keeps the accepted drafts after gdn_recurrent_verify (states_out form): for
 * each sequence n, state[n] <- states[n][accepted[n] - 1] when
 * 1 <= accepted[n] <= K; state[n] is left unchanged when accepted[n] is 0 (or
 * out of range, which is not an error: nothing was accepted).  accepted is a
 * DEVICE array of N int32, so the acceptance decided on the GPU needs no round
 * trip through the host.
 * Layouts: states [N][K][HV][dv][dk] fp32, state [N][HV][dv][dk] fp32.
 * Alignment: states, state 16-byte aligned, accepted 4-byte aligned; dv*dk a
 * multiple of 4.  N == 0 is an empty batch (GDN_OK; pointers may be NULL).
 */
GDN_API gdn_status gdn_state_commit(const float *states, const int32_t *accepted, float *state,
                                    int N, int K, int HV, int dk, int dv, gdn_stream_t stream);

/*
 * Keeps the accepted drafts after gdn_recurrent_verify (u_out form), updating
 * `state` (the verify call's input state) in place: with a = accepted[n],
 *   S <- (prod_{t<a} alpha_t) S + sum_{t<a} (prod_{t<s<a} alpha_s) u_t k_t^T,
 * alpha_t = exp(g_t): the recurrence unrolled over the kept tokens.  Each
 * state element is read and written once.  a == 0 or out of range leaves the
 * state unchanged.  k and g are the verify call's inputs, u its u_out, and
 * `prologue` the verify call's flags (its NORM_K and GATE_LOGITS bits apply).
 * Layouts: k [N][K][HK][dk] dtype, g [N][K][HV] fp32, u [N][K][HV][dv] fp32,
 * accepted [N] int32 (device), state [N][HV][dv][dk] fp32.
 * Supported: as gdn_recurrent_verify.  Alignment: k, state 16-byte aligned,
 * u, accepted 4-byte.  N == 0 is an empty batch (GDN_OK; pointers may be NULL).
 */
GDN_API gdn_status gdn_state_commit_deltas(const void *k, const float *g, const float *u,
                                           const int32_t *accepted, float *state, int N, int K,
                                           int HK, int HV, int dk, int dv, gdn_dtype dtype,
                                           unsigned prologue, gdn_stream_t stream);

/*
 * ---- The layer steps around the rule -------------------------------------
 * "Qwen3-Next" (sghael.github.io), section "Linear attention with gated delta
 * rule", names two further layer steps: the values are mixed with their
 * recent predecessors by a short convolution before the rule, and its read-out
 * is scaled by a gate.  The page gives neither the width nor the gate's form.
 * Reading used here:
 *   - a causal depthwise convolution along time, one kernel of `width` taps
 *     (2..8) per value channel c = h * dv + i (C = HV * dv channels):
 *       y_t[c] = act(bias[c] + sum_{j<width} weight[c][j] * x_{t-(width-1)+j}[c])
 *     within each sequence; the inputs before a sequence's first token come
 *     from its carried convolution state (its last width-1 inputs, raw) or are
 *     zero; act = identity, or SiLU (x * sigmoid(x)) with GDN_CONV_SILU;
 *   - an elementwise sigmoid gate on the read-out: o <- o * sigmoid(z), one
 *     logit per output element.
 * Convolution state layout: [N][width-1][C] in the call's dtype, row m = the
 * input width-1-m tokens before the next token (row width-2 the most recent).
 */
#define GDN_CONV_SILU 16u
#define GDN_CONV_MAX_WIDTH 8

/*
 * Short causal convolution over N sequences of C channels.
 * x, y [B][T][C] dtype (or packed [T_total][C] with cu_seqlens, as in
 * gdn_chunk_prefill; T is then the packed total); weight [C][width] fp32;
 * bias [C] fp32 or NULL; conv_state as above or NULL (zero history, nothing
 * kept).  When given, conv_state is read as each sequence's history and then
 * overwritten with its last width-1 inputs (taken from the old state where a
 * sequence is shorter than width-1; an empty sequence keeps its state).
 * flags: 0 or GDN_CONV_SILU.  Supported: 2 <= width <= GDN_CONV_MAX_WIDTH, C a
 * multiple of 8 (bf16) or 4 (fp32).  Alignment: x, y, conv_state, weight
 * 16-byte; bias 4-byte.
 * y must not overlap x or conv_state.  Two launches (the convolution, then the
 * state update when conv_state is given).  N == 0: GDN_OK, nothing launched;
 * no tokens: only the state update runs (and keeps every state).
 */
GDN_API gdn_status gdn_short_conv(const void *x, const float *weight, const float *bias,
                                  void *conv_state, const int32_t *cu_seqlens, int N, int64_t T,
                                  int C, int width, unsigned flags, gdn_dtype dtype, void *y,
                                  gdn_stream_t stream);

/*
 * Output gate in place: o <- o * sigmoid(z) over rows x C elements (o and z
 * the same dtype and layout, e.g. [B][T][HV][dv] with C = HV * dv).
 * Supported: rows * C a multiple of 8 (bf16) or 4 (fp32).  Alignment: o, z
 * 16-byte.  rows == 0: GDN_OK, nothing launched.
 */
GDN_API gdn_status gdn_output_gate(void *o, const void *z, int64_t rows, int C, gdn_dtype dtype,
                                   gdn_stream_t stream);

/*
 * gdn_recurrent_step_ex with the layer steps fused into the same kernel: the
 * token's v is convolved with each sequence's carried inputs (conv_state
 * [N][conv_width-1][HV*dv] dtype, updated in place) before the rule, and the
 * output is gated by sigmoid(z) (z [N][HV][dv] dtype) after it.  conv_weight
 * [HV*dv][conv_width] fp32 (NULL: no convolution, conv_width ignored),
 * conv_bias [HV*dv] fp32 or NULL; z NULL: no gate.  flags: GDN_PROLOGUE_*,
 * GDN_ROW_DECAY and GDN_CONV_SILU.  Supported and aligned as
 * gdn_recurrent_step_ex, plus 2 <= conv_width <= GDN_CONV_MAX_WIDTH when
 * conv_weight is given; conv_state, z 2-byte (bf16) or 4-byte (fp32) aligned.
 */
GDN_API gdn_status gdn_recurrent_step_layer(const void *q, const void *k, const void *v,
                                            const float *g, const float *beta, float *state,
                                            const float *conv_weight, const float *conv_bias,
                                            void *conv_state, int conv_width, const void *z,
                                            int N, int HK, int HV, int dk, int dv, float scale,
                                            gdn_dtype dtype, void *o, unsigned flags,
                                            gdn_stream_t stream);

/*
 * Bytes of device workspace gdn_chunk_prefill_layer needs: gdn_chunk_prefill's
 * own workspace, then the convolved values (when has_conv) and the gate factors
 * sigmoid(z) (when has_gate), each [tokens][HV*dv] of 2 bytes (bf16 calls) or
 * 4 bytes (fp32 calls); on the tensor-core path the convolved values get room for
 * a bf16 pair (twice the bytes), which the call uses with GDN_CONV_SILU.
 */
GDN_API size_t gdn_chunk_prefill_layer_workspace_size(int N, int64_t T, int HK, int HV, int dk,
                                                      int dv, int chunk, gdn_dtype dtype,
                                                      int varlen, int has_conv, int has_gate);

/*
 * gdn_chunk_prefill_ex with the layer steps: the short convolution of v
 * (gdn_short_conv into the workspace, stored in the call's dtype -- the
 * tensor-core path takes bf16 operands, and with GDN_CONV_SILU it takes the
 * convolved values as a bf16 pair value + remainder, ~2^-17 relative, since
 * SiLU-convolved values give the state a large common component beside which
 * their rounding would weigh on o; conv_state [N][conv_width-1][HV*dv] updated
 * as there), the gate factors sigmoid(z) into the workspace (fp16, relative
 * error <= 2^-12, for bf16 calls; fp32 for fp32 calls; formed in the
 * convolution's pass when there is one), then the prefill on the convolved
 * values, which multiplies o by the factors where it writes o (z like v; o is
 * rounded once).
 * conv_weight NULL: no convolution; z NULL: no gate.  flags: GDN_PROLOGUE_*,
 * GDN_ROW_DECAY and GDN_CONV_SILU.  Launches on `stream`: the convolution's two
 * (the factors with it) or, without a convolution, the factors' one, then the
 * prefill's one; arguments as in gdn_chunk_prefill_ex and gdn_short_conv.  z
 * 16-byte aligned.
 */
GDN_API gdn_status gdn_chunk_prefill_layer(const void *q, const void *k, const void *v,
                                           const float *g, const float *beta, const float *h0,
                                           const int32_t *cu_seqlens, int N, int64_t T, int HK,
                                           int HV, int dk, int dv, int chunk, float scale,
                                           gdn_dtype dtype, void *o, float *hT,
                                           const float *conv_weight, const float *conv_bias,
                                           void *conv_state, int conv_width, const void *z,
                                           unsigned flags, void *workspace,
                                           size_t workspace_bytes, gdn_stream_t stream);

/*
 * Reads the device status word a prefill call left in its workspace (HOST
 * call; synchronises `stream`).  Returns GDN_OK when every on-device wait of
 * the last call on this workspace completed, GDN_ERR_TIMEOUT when one gave up
 * (the outputs of that call are then undefined), or GDN_ERR_CUDA.
 * workspace NULL: reads the status word in the library array that
 * gdn_chunk_prefill_noalloc uses on the current device (the last such call's
 * waits); GDN_ERR_CUDA when no device is usable.
 */
GDN_API gdn_status gdn_read_status(const void *workspace, size_t workspace_bytes, gdn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GDN_B200_H */
