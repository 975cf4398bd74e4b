// C ABI entry points (declared in include/gdn.h): argument validation, workspace
// sizing and dispatch to the kernels.  No allocation, no synchronisation, no
// global state; every launch goes to the caller's stream.
#include <cuda_runtime.h>


#include "gdn.h"
#include "gdn_internal.h"

static_assert(gdn::kVerifyMaxDrafts == GDN_VERIFY_MAX_DRAFTS,
              "the verify kernels size their shared memory for the declared draft limit");

namespace {

bool aligned16(const void *p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

bool tc_path(int dk, int dv, int chunk, gdn_dtype dt) {
    return gdn::prefill_ring_supported(dk, dv, chunk, dt);
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

namespace gdn {

size_t prefill_workspace_bytes(const PrefillArgs &a) {
    if (!tc_path(a.dk, a.dv, a.chunk, a.dtype) || (a.prologue & GDN_ROW_DECAY)) return 0;
    return a.status_only ? prefill_cluster_workspace(a.N, a.T, a.HV, a.chunk, a.cu_seqlens != nullptr)
                         : prefill_ring_workspace(a.N, a.T, a.HV, a.chunk, a.cu_seqlens != nullptr);
}

// Validation, workspace check and dispatch of one prefill call (tensor-core path
// for bf16 / d = 128 / chunk 64, CUDA-core path otherwise).
gdn_status enqueue_prefill(const PrefillArgs &a, cudaStream_t stream) {
    gdn_status st = check_prefill(a);
    if (st != GDN_OK) return st;
    if (a.N == 0) return GDN_OK;
    cudaError_t err;
    // one decay per value row: the row-recurrent CUDA-core kernel (the rows of the
    // state never mix under that rule)
    if (a.prologue & GDN_ROW_DECAY) {
        err = launch_prefill_rows(a, stream);
    } else if (tc_path(a.dk, a.dv, a.chunk, a.dtype)) {
        const size_t need = prefill_workspace_bytes(a);
        if (need > 0 && (a.workspace == nullptr || a.workspace_bytes < need)) return GDN_ERR_WORKSPACE;
        if (!aligned16(a.workspace)) return GDN_ERR_ALIGNMENT;
        err = a.status_only ? launch_prefill_cluster(a, stream) : launch_prefill_ring(a, stream);
    } else {
        err = launch_prefill_simt(a, stream);
    }
    return err == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace gdn

namespace {

using gdn::enqueue_prefill;

// Device workspace of gdn_chunk_prefill_host: the status word, two input and two
// output segment buffers (inputs packed q | k | v | g | beta) and two states.
struct HostPlan {
    int64_t seg;
    size_t elt, q_bytes, v_bytes, g_bytes;
    size_t status, pre, in[2], out[2], st[2], total;
    static size_t up(size_t x) { return (x + 255) & ~size_t(255); }
    HostPlan(int N, int64_t T, int HK, int HV, int dk, int dv, int chunk, gdn_dtype dtype,
             int64_t segment) {
        seg = segment > 0 ? segment : 4096;
        if (T > 0 && seg > T) seg = T;
        if (seg <= 0) seg = 1;
        elt = dtype == GDN_BF16 ? 2 : 4;
        const size_t rows = (size_t)N * (size_t)seg;
        q_bytes = up(rows * HK * dk * elt);
        v_bytes = up(rows * HV * dv * elt);
        g_bytes = up(rows * HV * 4);
        const size_t in_b = 2 * q_bytes + v_bytes + 2 * g_bytes;
        const size_t out_b = v_bytes;
        const size_t st_b = up((size_t)N * HV * dv * dk * 4);
        // the segment prefill's own workspace (status word first) at the start
        gdn::PrefillArgs a{};
        a.N = N;
        a.T = seg;
        a.HV = HV;
        a.dk = dk;
        a.dv = dv;
        a.chunk = chunk;
        a.dtype = dtype;
        status = 0;
        pre = up(gdn::prefill_workspace_bytes(a) > 256 ? gdn::prefill_workspace_bytes(a) : 256);
        size_t off = pre;
        for (int b = 0; b < 2; ++b) { in[b] = off; off += in_b; }
        for (int b = 0; b < 2; ++b) { out[b] = off; off += out_b; }
        for (int b = 0; b < 2; ++b) { st[b] = off; off += st_b; }
        total = off;
    }
};

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
    if (tc_path(dk, dv, chunk, dtype)) return gdn::prefill_ring_workspace(N, T, HV, chunk, varlen != 0);
    return 0;
}

gdn_status gdn_chunk_prefill(const void *q, const void *k, const void *v, const float *g,
                             const float *beta, const float *h0, const int32_t *cu_seqlens,
                             int N, int64_t T, int HK, int HV, int dk, int dv, int chunk,
                             float scale, gdn_dtype dtype, void *o, float *hT, void *workspace,
                             size_t workspace_bytes, gdn_stream_t stream) {
    gdn::PrefillArgs a{q, k, v, g, beta, h0, cu_seqlens, N, T, HK, HV, dk, dv, chunk,
                       scale, dtype, o, hT, workspace, workspace_bytes};
    return enqueue_prefill(a, reinterpret_cast<cudaStream_t>(stream));
}

gdn_status gdn_chunk_prefill_ex(const void *q, const void *k, const void *v, const float *g,
                                const float *beta, const float *h0, const int32_t *cu_seqlens,
                                int N, int64_t T, int HK, int HV, int dk, int dv, int chunk,
                                float scale, gdn_dtype dtype, void *o, float *hT, void *workspace,
                                size_t workspace_bytes, unsigned prologue, gdn_stream_t stream) {
    if (prologue & ~GDN_FLAGS_VALID) return GDN_ERR_INVALID_ARG;
    if ((prologue & GDN_ROW_DECAY) && !gdn::prefill_simt_supported(dk, dv, chunk))
        return GDN_ERR_UNSUPPORTED;
    gdn::PrefillArgs a{q, k, v, g, beta, h0, cu_seqlens, N, T, HK, HV, dk, dv, chunk,
                       scale, dtype, o, hT, workspace, workspace_bytes};
    a.prologue = prologue;
    return enqueue_prefill(a, reinterpret_cast<cudaStream_t>(stream));
}

size_t gdn_chunk_prefill_host_workspace_size(int N, int64_t T, int HK, int HV, int dk, int dv,
                                             int chunk, gdn_dtype dtype, int64_t segment) {
    if (N <= 0 || T < 0 || HK <= 0 || HV <= 0 || HV % HK || chunk <= 0 || segment < 0) return 0;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return 0;
    if (gdn_chunk_prefill_path(dk, dv, chunk, dtype) < 0) return 0;
    return HostPlan(N, T, HK, HV, dk, dv, chunk, dtype, segment).total;
}

gdn_status gdn_chunk_prefill_host(const void *q, const void *k, const void *v, const float *g,
                                  const float *beta, const float *h0, int N, int64_t T, int HK,
                                  int HV, int dk, int dv, int chunk, float scale, gdn_dtype dtype,
                                  void *o, float *hT, void *workspace, size_t workspace_bytes,
                                  int64_t segment, gdn_stream_t stream, gdn_stream_t copy_in,
                                  gdn_stream_t copy_out) {
    // validate the per-segment call once, with device-side stand-ins for the host buffers
    if (!q || !k || !v || !g || !beta || !o) return GDN_ERR_INVALID_ARG;
    if (N <= 0 || T < 0 || segment < 0) return GDN_ERR_INVALID_ARG;
    {
        gdn::PrefillArgs a{q, k, v, g, beta, h0, nullptr, N, T, HK, HV, dk, dv, chunk,
                           scale, dtype, o, hT, nullptr, 0};
        const gdn_status st = check_prefill(a);
        if (st != GDN_OK) return st;
    }
    const HostPlan plan(N, T, HK, HV, dk, dv, chunk, dtype, segment);
    if (workspace == nullptr || workspace_bytes < plan.total) return GDN_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return GDN_ERR_ALIGNMENT;
    if (T == 0) return GDN_OK;
    cudaStream_t sc = reinterpret_cast<cudaStream_t>(stream);
    cudaStream_t si = reinterpret_cast<cudaStream_t>(copy_in);
    cudaStream_t so = reinterpret_cast<cudaStream_t>(copy_out);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const int64_t S = plan.seg, nseg = (T + S - 1) / S;
    // the events that order the three streams, two of each kind (by segment parity):
    // a stream wait takes the event's latest record when it is enqueued, and the record
    // of segment s is the latest one of its pair until segment s + 2 records it again,
    // after that segment's waits on it are enqueued.  Destroyed below once enqueued
    // (the runtime keeps each alive until it has completed).
    constexpr int nev = 7;
    cudaEvent_t evs[nev];
    int made = 0;
    gdn_status result = GDN_OK;
    for (; made < nev; ++made)
        if (cudaEventCreateWithFlags(&evs[made], cudaEventDisableTiming) != cudaSuccess) {
            result = GDN_ERR_CUDA;
            break;
        }
    auto ev_in = [&](int64_t s) { return evs[1 + 3 * (s & 1)]; };
    auto ev_done = [&](int64_t s) { return evs[2 + 3 * (s & 1)]; };
    auto ev_out = [&](int64_t s) { return evs[3 + 3 * (s & 1)]; };
    auto ok = [&](cudaError_t e) {
        if (e != cudaSuccess && result == GDN_OK) result = GDN_ERR_CUDA;
        return result == GDN_OK;
    };
    const size_t eq = plan.elt * (size_t)HK * dk, ev = plan.elt * (size_t)HV * dv, eg = 4u * HV;
    // the copy streams start after everything already queued on the compute stream
    if (result == GDN_OK && ok(cudaEventRecord(evs[0], sc)) && ok(cudaStreamWaitEvent(si, evs[0], 0)))
        ok(cudaStreamWaitEvent(so, evs[0], 0));
    if (result == GDN_OK) ok(cudaMemsetAsync(ws + plan.status, 0, sizeof(unsigned int), sc));
    for (int64_t s = 0; s < nseg && result == GDN_OK; ++s) {
        const int64_t t0 = s * S, Ls = T - t0 < S ? T - t0 : S;
        const int b = (int)(s & 1);
        uint8_t *in = ws + plan.in[b];
        uint8_t *dq = in, *dk_ = in + plan.q_bytes, *dv_ = dk_ + plan.q_bytes,
                *dg = dv_ + plan.v_bytes, *db = dg + plan.g_bytes;
        // inputs of segment s into buffer b (free once segment s - 2 is computed)
        if (s >= 2 && !ok(cudaStreamWaitEvent(si, ev_done(s - 2), 0))) break;
        const struct { const void *src; void *dst; size_t row; } cp[5] = {
            {q, dq, eq}, {k, dk_, eq}, {v, dv_, ev}, {g, dg, eg}, {beta, db, eg}};
        for (const auto &c : cp)
            if (!ok(cudaMemcpy2DAsync(c.dst, (size_t)Ls * c.row,
                                      static_cast<const uint8_t *>(c.src) + (size_t)t0 * c.row,
                                      (size_t)T * c.row, (size_t)Ls * c.row, (size_t)N,
                                      cudaMemcpyHostToDevice, si)))
                break;
        if (result != GDN_OK || !ok(cudaEventRecord(ev_in(s), si))) break;
        // segment s: state from the previous segment (or h0), outputs into buffer b
        // (free once segment s - 2's outputs have been copied out)
        if (!ok(cudaStreamWaitEvent(sc, ev_in(s), 0))) break;
        if (s >= 2 && !ok(cudaStreamWaitEvent(sc, ev_out(s - 2), 0))) break;
        const float *hin = s == 0 ? h0 : reinterpret_cast<const float *>(ws + plan.st[(s - 1) & 1]);
        float *hout = (s == nseg - 1 && hT) ? hT : reinterpret_cast<float *>(ws + plan.st[b]);
        uint8_t *out = ws + plan.out[b];
        gdn::PrefillArgs a{dq, dk_, dv_, reinterpret_cast<const float *>(dg),
                           reinterpret_cast<const float *>(db), hin, nullptr, N, Ls, HK, HV, dk,
                           dv, chunk, scale, dtype, out, hout, ws + plan.status, plan.pre};
        a.keep_status = true;
        const gdn_status st = enqueue_prefill(a, sc);
        if (st != GDN_OK) {
            result = st;
            break;
        }
        if (!ok(cudaEventRecord(ev_done(s), sc))) break;
        // outputs of segment s back to the host
        if (!ok(cudaStreamWaitEvent(so, ev_done(s), 0))) break;
        if (!ok(cudaMemcpy2DAsync(static_cast<uint8_t *>(o) + (size_t)t0 * ev, (size_t)T * ev, out,
                                  (size_t)Ls * ev, (size_t)Ls * ev, (size_t)N,
                                  cudaMemcpyDeviceToHost, so)))
            break;
        ok(cudaEventRecord(ev_out(s), so));
    }
    // everything the call enqueued is ordered before later work on the compute stream
    if (result == GDN_OK) ok(cudaStreamWaitEvent(sc, ev_out(nseg - 1), 0));
    for (int i = 0; i < made; ++i) cudaEventDestroy(evs[i]);
    return result;
}

gdn_status gdn_recurrent_step(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, float *state, int N, int HK, int HV, int dk,
                              int dv, float scale, gdn_dtype dtype, void *o,
                              gdn_stream_t stream) {
    return gdn_recurrent_step_ex(q, k, v, g, beta, state, N, HK, HV, dk, dv, scale, dtype, o, 0u,
                                 stream);
}

gdn_status gdn_recurrent_step_ex(const void *q, const void *k, const void *v, const float *g,
                                 const float *beta, float *state, int N, int HK, int HV, int dk,
                                 int dv, float scale, gdn_dtype dtype, void *o, unsigned prologue,
                                 gdn_stream_t stream) {
    if (prologue & ~GDN_FLAGS_VALID) return GDN_ERR_INVALID_ARG;
    if (!q || !k || !v || !g || !beta || !state || !o) return GDN_ERR_INVALID_ARG;
    if (N < 0 || HK <= 0 || HV <= 0 || dk <= 0 || dv <= 0 || HV % HK) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if ((int64_t)N * HV > 0x7fffffff) return GDN_ERR_UNSUPPORTED;
    if (!gdn::decode_supported(dk, dv)) return GDN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(state))
        return GDN_ERR_ALIGNMENT;
    if (N == 0) return GDN_OK;
    gdn::StepArgs a{q, k, v, g, beta, state, N, HK, HV, dk, dv, scale, dtype, o, prologue};
    const cudaError_t err = gdn::launch_decode(a, reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status gdn_recurrent_verify(const void *q, const void *k, const void *v, const float *g,
                                const float *beta, const float *state, int N, int K, int HK, int HV,
                                int dk, int dv, float scale, gdn_dtype dtype, void *o,
                                float *states_out, float *u_out, unsigned prologue,
                                void *workspace, size_t workspace_bytes, gdn_stream_t stream) {
    if (prologue & ~GDN_FLAGS_VALID) return GDN_ERR_INVALID_ARG;
    if (N < 0 || K <= 0 || HK <= 0 || HV <= 0 || dk <= 0 || dv <= 0 || HV % HK)
        return GDN_ERR_INVALID_ARG;
    if (N == 0) return GDN_OK;   // empty batch: buffers may be NULL
    if (!q || !k || !v || !g || !beta || !state || !o) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (K > GDN_VERIFY_MAX_DRAFTS || (int64_t)N * HV > 0x7fffffff) return GDN_ERR_UNSUPPORTED;
    if (!gdn::decode_supported(dk, dv)) return GDN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(state) ||
        !aligned16(states_out) || !aligned4(u_out))
        return GDN_ERR_ALIGNMENT;
    if (!states_out) {   // update-vector form: tables in the workspace (unused with row decays)
        if (!workspace ||
            workspace_bytes < gdn::verify_workspace_floats(N, K, HV, dk) * sizeof(float))
            return GDN_ERR_WORKSPACE;
        if (!aligned16(workspace)) return GDN_ERR_ALIGNMENT;
    }
    gdn::VerifyArgs a{q, k, v, g, beta, state, states_out, u_out, N, K, HK, HV, dk, dv, scale,
                      dtype, o, prologue, workspace, workspace_bytes};
    const cudaError_t err = gdn::launch_verify(a, reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status gdn_recurrent_commit_verify(const void *prev_k, const float *prev_g, const float *prev_u,
                                       const int32_t *accepted, int prev_K, const void *q,
                                       const void *k, const void *v, const float *g,
                                       const float *beta, float *state, int N, int K, int HK,
                                       int HV, int dk, int dv, float scale, gdn_dtype dtype,
                                       void *o, float *u_out, unsigned prologue, void *workspace,
                                       size_t workspace_bytes, gdn_stream_t stream) {
    if (prologue & ~GDN_FLAGS_VALID) return GDN_ERR_INVALID_ARG;
    if (N < 0 || K <= 0 || prev_K <= 0 || HK <= 0 || HV <= 0 || dk <= 0 || dv <= 0 || HV % HK)
        return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (N == 0) return GDN_OK;   // empty batch: buffers may be NULL
    if (!q || !k || !v || !g || !beta || !state || !o || !prev_k || !prev_g || !prev_u || !accepted)
        return GDN_ERR_INVALID_ARG;
    if (K > GDN_VERIFY_MAX_DRAFTS || prev_K > GDN_VERIFY_MAX_DRAFTS || (int64_t)N * HV > 0x7fffffff)
        return GDN_ERR_UNSUPPORTED;
    if (!gdn::decode_supported(dk, dv)) return GDN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(state) ||
        !aligned16(prev_k) || !aligned4(prev_u) || !aligned4(accepted) || !aligned4(u_out))
        return GDN_ERR_ALIGNMENT;
    if (!workspace ||
        workspace_bytes < gdn::verify_workspace_floats(N, K, HV, dk, prev_K) * sizeof(float))
        return GDN_ERR_WORKSPACE;
    if (!aligned16(workspace)) return GDN_ERR_ALIGNMENT;
    gdn::VerifyArgs a{q, k, v, g, beta, state, nullptr, u_out, N, K, HK, HV, dk, dv, scale,
                      dtype, o, prologue, workspace, workspace_bytes};
    if (prologue & GDN_ROW_DECAY) {
        // one decay per value row: the previous round's commit from its update vectors,
        // then this round's verify writing update vectors (two passes over the states;
        // the one-pass form mixes the drafts per head)
        gdn::CommitDeltasArgs c{prev_k, prev_g, prev_u, accepted, state, N, prev_K, HK, HV, dk, dv,
                                dtype, prologue};
        cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
        if (gdn::launch_commit_deltas(c, s) != cudaSuccess) return GDN_ERR_CUDA;
        return gdn::launch_verify(a, s) == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
    }
    a.prev_k = prev_k;
    a.prev_g = prev_g;
    a.prev_u = prev_u;
    a.accepted = accepted;
    a.prev_K = prev_K;
    const cudaError_t err = gdn::launch_verify(a, reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

size_t gdn_recurrent_commit_verify_workspace_size(int N, int prev_K, int K, int HV, int dk) {
    if (N < 0 || K <= 0 || K > GDN_VERIFY_MAX_DRAFTS || prev_K <= 0 ||
        prev_K > GDN_VERIFY_MAX_DRAFTS || HV <= 0 || dk <= 0)
        return 0;
    return gdn::verify_workspace_floats(N, K, HV, dk, prev_K) * sizeof(float);
}

size_t gdn_recurrent_verify_workspace_size(int N, int K, int HV, int dk) {
    if (N < 0 || K <= 0 || K > GDN_VERIFY_MAX_DRAFTS || HV <= 0 || dk <= 0) return 0;
    return gdn::verify_workspace_floats(N, K, HV, dk) * sizeof(float);
}

gdn_status gdn_state_commit(const float *states, const int32_t *accepted, float *state, int N, int K,
                            int HV, int dk, int dv, gdn_stream_t stream) {
    if (N < 0 || K <= 0 || HV <= 0 || dk <= 0 || dv <= 0) return GDN_ERR_INVALID_ARG;
    if (N == 0) return GDN_OK;   // empty batch: buffers may be NULL
    if (!states || !accepted || !state) return GDN_ERR_INVALID_ARG;
    if ((int64_t)N * HV > 0x7fffffff || ((int64_t)dk * dv) % 4) return GDN_ERR_UNSUPPORTED;
    if (!aligned16(states) || !aligned16(state) || !aligned4(accepted)) return GDN_ERR_ALIGNMENT;
    if (N == 0) return GDN_OK;
    const cudaError_t err = gdn::launch_commit(states, accepted, state, N, K, HV, dv, dk,
                                               reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status gdn_state_commit_deltas(const void *k, const float *g, const float *u,
                                   const int32_t *accepted, float *state, int N, int K, int HK,
                                   int HV, int dk, int dv, gdn_dtype dtype, unsigned prologue,
                                   gdn_stream_t stream) {
    if (prologue & ~GDN_FLAGS_VALID) return GDN_ERR_INVALID_ARG;
    if (N < 0 || K <= 0 || HK <= 0 || HV <= 0 || dk <= 0 || dv <= 0 || HV % HK)
        return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (N == 0) return GDN_OK;   // empty batch: buffers may be NULL
    if (!k || !g || !u || !accepted || !state) return GDN_ERR_INVALID_ARG;
    if (K > GDN_VERIFY_MAX_DRAFTS || (int64_t)N * HV > 0x7fffffff) return GDN_ERR_UNSUPPORTED;
    if (!gdn::decode_supported(dk, dv)) return GDN_ERR_UNSUPPORTED;
    if (!aligned16(k) || !aligned16(state) || !aligned4(u) || !aligned4(accepted))
        return GDN_ERR_ALIGNMENT;
    gdn::CommitDeltasArgs a{k, g, u, accepted, state, N, K, HK, HV, dk, dv, dtype, prologue};
    const cudaError_t err = gdn::launch_commit_deltas(a, reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// ---- layer steps: short convolution on the values, output gate ----

}  // extern "C"

namespace {

bool aligned_elt(const void *p, gdn_dtype dt) {
    return dt == GDN_BF16 ? (reinterpret_cast<uintptr_t>(p) & 1u) == 0 : aligned4(p);
}

// host checks of one short-convolution call (nothing enqueued)
gdn_status check_conv(const gdn::ConvArgs &a) {
    if (!a.x || !a.weight || !a.y) return GDN_ERR_INVALID_ARG;
    if (a.N < 0 || a.T < 0 || a.C <= 0) return GDN_ERR_INVALID_ARG;
    if (a.dtype != GDN_F32 && a.dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (a.width < 2 || a.width > gdn::kConvMaxWidth) return GDN_ERR_UNSUPPORTED;
    if (a.C % gdn::conv_vector_channels(a.dtype)) return GDN_ERR_UNSUPPORTED;
    if (a.C / gdn::conv_vector_channels(a.dtype) > 65535 * 128) return GDN_ERR_UNSUPPORTED;
    const int64_t tokens = a.cu_seqlens ? a.T : (int64_t)a.N * a.T;
    if (a.cu_seqlens == nullptr && a.N > 0 && a.T > 0 && tokens / a.N != a.T) return GDN_ERR_INVALID_ARG;
    if ((tokens + 7) / 8 * ((a.C / gdn::conv_vector_channels(a.dtype) + 127) / 128) > 0x7fffffffLL)
        return GDN_ERR_UNSUPPORTED;
    if (!aligned16(a.x) || !aligned16(a.y) || !aligned16(a.conv_state) || !aligned16(a.weight) ||
        !aligned4(a.bias))
        return GDN_ERR_ALIGNMENT;
    return GDN_OK;
}

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

size_t layer_vconv_bytes(int N, int64_t T, int HV, int dv, gdn_dtype dt, bool varlen) {
    const int64_t tokens = varlen ? T : (int64_t)N * T;
    return up256((size_t)tokens * (size_t)HV * (size_t)dv * (dt == GDN_BF16 ? 2 : 4));
}

}  // namespace

extern "C" {

gdn_status gdn_short_conv(const void *x, const float *weight, const float *bias, void *conv_state,
                          const int32_t *cu_seqlens, int N, int64_t T, int C, int width,
                          unsigned flags, gdn_dtype dtype, void *y, gdn_stream_t stream) {
    if (flags & ~GDN_CONV_SILU) return GDN_ERR_INVALID_ARG;
    gdn::ConvArgs a{x, weight, bias, conv_state, cu_seqlens, N, T, C, width,
                    (flags & GDN_CONV_SILU) != 0, dtype, y};
    const gdn_status st = check_conv(a);
    if (st != GDN_OK) return st;
    if (N == 0) return GDN_OK;
    const cudaError_t err = gdn::launch_short_conv(a, reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status gdn_output_gate(void *o, const void *z, int64_t rows, int C, gdn_dtype dtype,
                           gdn_stream_t stream) {
    if (!o || !z || rows < 0 || C <= 0) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (rows > ((int64_t)1 << 40) / C) return GDN_ERR_INVALID_ARG;
    const int64_t elems = rows * (int64_t)C;
    if (elems % gdn::conv_vector_channels(dtype)) return GDN_ERR_UNSUPPORTED;
    if (!aligned16(o) || !aligned16(z)) return GDN_ERR_ALIGNMENT;
    if (elems == 0) return GDN_OK;
    const cudaError_t err =
        gdn::launch_output_gate(o, z, elems, dtype, reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status gdn_recurrent_step_layer(const void *q, const void *k, const void *v, const float *g,
                                    const float *beta, float *state, const float *conv_weight,
                                    const float *conv_bias, void *conv_state, int conv_width,
                                    const void *z, int N, int HK, int HV, int dk, int dv,
                                    float scale, gdn_dtype dtype, void *o, unsigned flags,
                                    gdn_stream_t stream) {
    if (flags & ~(GDN_FLAGS_VALID | GDN_CONV_SILU)) return GDN_ERR_INVALID_ARG;
    if (!q || !k || !v || !g || !beta || !state || !o) return GDN_ERR_INVALID_ARG;
    if (N < 0 || HK <= 0 || HV <= 0 || dk <= 0 || dv <= 0 || HV % HK) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (conv_weight && !conv_state) return GDN_ERR_INVALID_ARG;
    if (conv_weight && (conv_width < 2 || conv_width > GDN_CONV_MAX_WIDTH)) return GDN_ERR_UNSUPPORTED;
    if ((int64_t)N * HV > 0x7fffffff) return GDN_ERR_UNSUPPORTED;
    if (!gdn::decode_supported(dk, dv)) return GDN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(state))
        return GDN_ERR_ALIGNMENT;
    if (!aligned4(conv_weight) || !aligned4(conv_bias) ||
        (conv_weight && !aligned_elt(conv_state, dtype)) || (z && !aligned_elt(z, dtype)))
        return GDN_ERR_ALIGNMENT;
    if (N == 0) return GDN_OK;
    gdn::StepArgs a{q, k, v, g, beta, state, N, HK, HV, dk, dv, scale, dtype, o,
                    flags & GDN_FLAGS_VALID};
    if (conv_weight) {
        a.conv_w = conv_weight;
        a.conv_b = conv_bias;
        a.conv_state = conv_state;
        a.conv_width = conv_width;
        a.conv_silu = (flags & GDN_CONV_SILU) != 0;
    }
    a.z = z;
    const cudaError_t err = gdn::launch_decode(a, reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

size_t gdn_chunk_prefill_layer_workspace_size(int N, int64_t T, int HK, int HV, int dk, int dv,
                                              int chunk, gdn_dtype dtype, int varlen,
                                              int has_conv, int has_gate) {
    if (N < 0 || T < 0 || HK <= 0 || HV <= 0 || HV % HK || dv <= 0 || chunk <= 0) return 0;
    const size_t pre = up256(gdn_chunk_prefill_workspace_size(N, T, HK, HV, dk, dv, chunk, dtype, varlen));
    const bool vpair = has_conv && tc_path(dk, dv, chunk, dtype);
    return pre + (has_conv ? layer_vconv_bytes(N, T, HV, dv, dtype, varlen != 0) * (vpair ? 2 : 1) : 0) +
           (has_gate ? layer_vconv_bytes(N, T, HV, dv, dtype, varlen != 0) : 0);
}

gdn_status gdn_chunk_prefill_layer(const void *q, const void *k, const void *v, const float *g,
                                   const float *beta, const float *h0, const int32_t *cu_seqlens,
                                   int N, int64_t T, int HK, int HV, int dk, int dv, int chunk,
                                   float scale, gdn_dtype dtype, void *o, float *hT,
                                   const float *conv_weight, const float *conv_bias,
                                   void *conv_state, int conv_width, const void *z, unsigned flags,
                                   void *workspace, size_t workspace_bytes, gdn_stream_t stream) {
    if (flags & ~(GDN_FLAGS_VALID | GDN_CONV_SILU)) return GDN_ERR_INVALID_ARG;
    const unsigned prologue = flags & GDN_FLAGS_VALID;
    if ((prologue & GDN_ROW_DECAY) && !gdn::prefill_simt_supported(dk, dv, chunk))
        return GDN_ERR_UNSUPPORTED;
    gdn::PrefillArgs a{q, k, v, g, beta, h0, cu_seqlens, N, T, HK, HV, dk, dv, chunk,
                       scale, dtype, o, hT, workspace, workspace_bytes};
    a.prologue = prologue;
    gdn_status st = check_prefill(a);
    if (st != GDN_OK) return st;
    const bool varlen = cu_seqlens != nullptr;
    if ((size_t)HV * dv > 0x7fffffffu) return GDN_ERR_UNSUPPORTED;
    const int C = HV * dv;
    gdn::ConvArgs ca{v, conv_weight, conv_bias, conv_state, cu_seqlens, N, T, C, conv_width,
                     (flags & GDN_CONV_SILU) != 0, dtype, nullptr};
    if (conv_weight) {
        ca.y = o;   // placeholder for the host checks; the real target is the workspace
        st = check_conv(ca);
        if (st != GDN_OK) return st;
    }
    if (z && !aligned16(z)) return GDN_ERR_ALIGNMENT;
    if (N == 0) return GDN_OK;
    // workspace: [prefill's own | convolved values | gate factors (fp16)]
    const size_t pre = up256(gdn::prefill_workspace_bytes(a));
    // on the tensor-core path SiLU-convolved values go to the rule as a bf16 pair
    // (values + remainders): their positive mean gives the state a large common
    // component, beside which the bf16 rounding of the values alone would weigh on
    // o; without the activation the values are as centred as v and stay single bf16
    const bool vpair = conv_weight && (flags & GDN_CONV_SILU) && tc_path(dk, dv, chunk, dtype) &&
                       !(prologue & GDN_ROW_DECAY);
    const size_t vbytes = conv_weight ? layer_vconv_bytes(N, T, HV, dv, dtype, varlen) * (vpair ? 2 : 1) : 0;
    const size_t need = pre + vbytes + (z ? layer_vconv_bytes(N, T, HV, dv, dtype, varlen) : 0);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return GDN_ERR_WORKSPACE;
    if (!aligned16(workspace)) return GDN_ERR_ALIGNMENT;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // sigmoid(z) factors (fp16 for bf16, fp32 for fp32), applied in the prefill's
    // read-out before o is rounded: formed by the convolution's launch when there is
    // one (z has v's layout), else by a pass of their own
    void *f = z ? static_cast<char *>(workspace) + pre + vbytes : nullptr;
    if (conv_weight) {
        ca.y = static_cast<char *>(workspace) + pre;
        if (vpair) ca.y_lo = static_cast<char *>(workspace) + pre + vbytes / 2;
        ca.z = z;
        ca.f = f;
        if (gdn::launch_short_conv(ca, s) != cudaSuccess) return GDN_ERR_CUDA;
        a.v = ca.y;
        a.v_lo = ca.y_lo;
    } else if (z) {
        const int64_t tokens = varlen ? T : (int64_t)N * T;
        if (gdn::launch_gate_factor(z, f, tokens * (int64_t)C, dtype, s) != cudaSuccess)
            return GDN_ERR_CUDA;
    }
    if (z) a.gate = f;
    a.workspace_bytes = pre;
    if (pre == 0) a.workspace = nullptr;
    return enqueue_prefill(a, s);
}

gdn_status gdn_read_status(const void *workspace, size_t workspace_bytes, gdn_stream_t stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // NULL: the library array of the workspace-free prefill on the current device
    if (workspace == nullptr) return gdn::noalloc_read_status(s);
    if (workspace_bytes < sizeof(unsigned int)) return GDN_OK;
    unsigned int word = 0;
    if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return GDN_ERR_CUDA;
    return word == 0 ? GDN_OK : GDN_ERR_TIMEOUT;
}

}  // extern "C"
