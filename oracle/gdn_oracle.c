/*
 * Float64 CPU oracle for the gated delta rule.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may load, call or
 * link this file: only the tests, the smoke check and the benchmark's CPU
 * baseline use it.  It shares no code, header or constant with the CUDA
 * library; the two meet only through the seeded synthetic inputs.
 *
 * What it computes (sources are the pages of "Qwen3-Next" by sghael.github.io,
 * section "Correcting a memory instead of adding to it", and the model card
 * "Qwen3-Next-80B-A3B-Instruct", section "Model Overview"):
 *
 *   The state S of one value head is a dv x dk matrix of key -> value
 *   associations (rows index the value dimension, columns the key dimension,
 *   the orientation of the teaching scan "W @ k" in "The Evolving Transformer
 *   / Qwen3-Next", section 01 GatedDeltaNet).  For every token t, in order:
 *
 *       alpha = exp(g_t)                          decay of the old memory
 *       S     = alpha * S                         shrink first ...
 *       S     = S + beta_t (v_t - S k_t) k_t^T    ... then correct along k_t
 *       o_t   = scale * S q_t                     read-out after the update
 *
 *   which equals S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T.
 *   The scalar worked example on the first page (6 -> 3 -> 6.5 with decay 0.5
 *   and write strength 0.5) fixes that the error term is taken on the
 *   decayed state.
 *
 *   Value head h reads query/key head floor(h / (HV / HK)).
 *
 * Two independent forms are provided:
 *   gdn_oracle_prefill          token-by-token recurrence (the definition)
 *   gdn_oracle_prefill_chunked  the chunkwise WY form derived from it
 *                               (used only to cross-check the definition)
 *   gdn_oracle_step             one decode token per sequence, state in place
 *
 * Array layouts (all float64, row-major, contiguous):
 *   q, k  [Ttot][HK][dk]     v, o  [Ttot][HV][dv]     g, beta [Ttot][HV]
 *   h0, hT [N][HV][dv][dk]   cu_seqlens: N+1 int64 offsets into Ttot, cu[0]=0
 * h0 may be NULL (zero start state); hT may be NULL (not returned).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

typedef struct {
    const double *q, *k, *v, *g, *beta, *h0;
    const int64_t *cu;
    int64_t N;
    int HK, HV, dk, dv, chunk;
    double scale;
    double *o, *hT;
} problem_t;

/* ------------------------------------------------------------------ */
/* Sequential definition, one (sequence, value head) unit.            */
/* ------------------------------------------------------------------ */
static void token_update(double *S, int dk, int dv, double alpha, double b,
                         const double *kt, const double *vt) {
    /* S <- alpha*S ; S <- S + b (v - S k) k^T  (error on the decayed state) */
    for (int i = 0; i < dv; ++i) {
        double *row = S + (size_t)i * dk;
        double sk = 0.0;
        for (int a = 0; a < dk; ++a) {
            row[a] *= alpha;
            sk += row[a] * kt[a];
        }
        double u = b * (vt[i] - sk);
        for (int a = 0; a < dk; ++a) row[a] += u * kt[a];
    }
}

static void token_readout(const double *S, int dk, int dv, double scale,
                          const double *qt, double *ot) {
    for (int i = 0; i < dv; ++i) {
        const double *row = S + (size_t)i * dk;
        double acc = 0.0;
        for (int a = 0; a < dk; ++a) acc += row[a] * qt[a];
        ot[i] = scale * acc;
    }
}

static void run_unit_sequential(const problem_t *P, int64_t n, int h, double *S) {
    const int dk = P->dk, dv = P->dv, HK = P->HK, HV = P->HV;
    const int c = h / (HV / HK);
    const size_t sdim = (size_t)dv * dk;
    if (P->h0) memcpy(S, P->h0 + ((size_t)n * HV + h) * sdim, sdim * sizeof(double));
    else memset(S, 0, sdim * sizeof(double));
    for (int64_t t = P->cu[n]; t < P->cu[n + 1]; ++t) {
        const double alpha = exp(P->g[t * HV + h]);
        const double b = P->beta[t * HV + h];
        const double *kt = P->k + ((size_t)t * HK + c) * dk;
        const double *qt = P->q + ((size_t)t * HK + c) * dk;
        const double *vt = P->v + ((size_t)t * HV + h) * dv;
        token_update(S, dk, dv, alpha, b, kt, vt);
        token_readout(S, dk, dv, P->scale, qt, P->o + ((size_t)t * HV + h) * dv);
    }
    if (P->hT) memcpy(P->hT + ((size_t)n * HV + h) * sdim, S, sdim * sizeof(double));
}

/* ------------------------------------------------------------------ */
/* Chunkwise WY form, one (sequence, value head) unit.                */
/*                                                                    */
/* Within a chunk that starts from state S0, with G_i the chunk-local */
/* running sum of g and gamma_i = exp(G_i), write                     */
/*   u_t = beta_t (v_t - alpha_t S_{t-1} k_t),  S_t = alpha_t S_{t-1} + u_t k_t^T. */
/* Unrolling gives S_i = gamma_i S0 + sum_{j<=i} (gamma_i/gamma_j) u_j k_j^T, */
/* and substituting into u gives (I + A) U = diag(beta) V - diag(beta gamma) K S0^T */
/* with A_ij = beta_i (gamma_i/gamma_j) k_i.k_j for j < i.  Hence      */
/*   T  = (I + A)^-1                                                  */
/*   U  = T diag(beta) V - T diag(beta gamma) K S0^T                  */
/*   O  = diag(gamma) Q S0^T + (M o Q K^T) U,  M_ij = gamma_i/gamma_j (j<=i) */
/*   S  = gamma_L S0 + U^T diag(gamma_L/gamma) K                      */
/* Ratios gamma_i/gamma_j are formed as exp(G_i - G_j), never as a    */
/* quotient, so strong decay cannot overflow.                         */
/* ------------------------------------------------------------------ */
static void run_unit_chunked(const problem_t *P, int64_t n, int h, double *S, double *work) {
    const int dk = P->dk, dv = P->dv, HK = P->HK, HV = P->HV, C = P->chunk;
    const int c = h / (HV / HK);
    const size_t sdim = (size_t)dv * dk;
    double *G = work;                         /* C        */
    double *A = G + C;                        /* C x C    */
    double *T = A + (size_t)C * C;            /* C x C    */
    double *U = T + (size_t)C * C;            /* C x dv   */
    double *W = U + (size_t)C * dv;           /* C x dk   */
    double *Sn = W + (size_t)C * dk;          /* dv x dk  */
    if (P->h0) memcpy(S, P->h0 + ((size_t)n * HV + h) * sdim, sdim * sizeof(double));
    else memset(S, 0, sdim * sizeof(double));

    for (int64_t s0 = P->cu[n]; s0 < P->cu[n + 1]; s0 += C) {
        int L = (int)((P->cu[n + 1] - s0) < C ? (P->cu[n + 1] - s0) : C);
#define KR(i) (P->k + ((size_t)(s0 + (i)) * HK + c) * dk)
#define QR(i) (P->q + ((size_t)(s0 + (i)) * HK + c) * dk)
#define VR(i) (P->v + ((size_t)(s0 + (i)) * HV + h) * dv)
#define BETA(i) (P->beta[(s0 + (i)) * HV + h])
        /* chunk-local log-decay running sum */
        double run = 0.0;
        for (int i = 0; i < L; ++i) { run += P->g[(s0 + i) * HV + h]; G[i] = run; }
        /* strictly lower A */
        for (int i = 0; i < L; ++i)
            for (int j = 0; j < L; ++j) {
                double val = 0.0;
                if (j < i) {
                    double kk = 0.0;
                    for (int a = 0; a < dk; ++a) kk += KR(i)[a] * KR(j)[a];
                    val = BETA(i) * exp(G[i] - G[j]) * kk;
                }
                A[(size_t)i * C + j] = val;
            }
        /* T = (I + A)^-1 by forward substitution, row by row */
        for (int i = 0; i < L; ++i)
            for (int j = 0; j < L; ++j) {
                double val = (i == j) ? 1.0 : 0.0;
                if (j < i)
                    for (int m = j; m < i; ++m) val -= A[(size_t)i * C + m] * T[(size_t)m * C + j];
                T[(size_t)i * C + j] = val;
            }
        /* U = T diag(beta) V - T diag(beta gamma) K S0^T ; W = T diag(beta gamma) K */
        for (int i = 0; i < L; ++i) {
            for (int a = 0; a < dk; ++a) {
                double acc = 0.0;
                for (int j = 0; j <= i; ++j) acc += T[(size_t)i * C + j] * BETA(j) * exp(G[j]) * KR(j)[a];
                W[(size_t)i * dk + a] = acc;
            }
            for (int e = 0; e < dv; ++e) {
                double acc = 0.0;
                for (int j = 0; j <= i; ++j) acc += T[(size_t)i * C + j] * BETA(j) * VR(j)[e];
                double ws = 0.0;
                for (int a = 0; a < dk; ++a) ws += W[(size_t)i * dk + a] * S[(size_t)e * dk + a];
                U[(size_t)i * dv + e] = acc - ws;
            }
        }
        /* O = diag(gamma) Q S0^T + (M o Q K^T) U */
        for (int i = 0; i < L; ++i) {
            double *oi = P->o + ((size_t)(s0 + i) * HV + h) * dv;
            double mq[256];
            for (int j = 0; j <= i; ++j) {
                double qk = 0.0;
                for (int a = 0; a < dk; ++a) qk += QR(i)[a] * KR(j)[a];
                mq[j] = exp(G[i] - G[j]) * qk;
            }
            for (int e = 0; e < dv; ++e) {
                double inter = 0.0;
                for (int a = 0; a < dk; ++a) inter += QR(i)[a] * S[(size_t)e * dk + a];
                double intra = 0.0;
                for (int j = 0; j <= i; ++j) intra += mq[j] * U[(size_t)j * dv + e];
                oi[e] = P->scale * (exp(G[i]) * inter + intra);
            }
        }
        /* S = gamma_L S0 + U^T diag(gamma_L / gamma) K */
        for (int e = 0; e < dv; ++e)
            for (int a = 0; a < dk; ++a) {
                double acc = exp(G[L - 1]) * S[(size_t)e * dk + a];
                for (int j = 0; j < L; ++j) acc += U[(size_t)j * dv + e] * exp(G[L - 1] - G[j]) * KR(j)[a];
                Sn[(size_t)e * dk + a] = acc;
            }
        memcpy(S, Sn, sdim * sizeof(double));
#undef KR
#undef QR
#undef VR
#undef BETA
    }
    if (P->hT) memcpy(P->hT + ((size_t)n * HV + h) * sdim, S, sdim * sizeof(double));
}

/* ------------------------------------------------------------------ */
/* Thread pool over (sequence, value head) units.                     */
/* ------------------------------------------------------------------ */
typedef struct {
    const problem_t *P;
    int chunked;
    int64_t next;     /* guarded by mu */
    pthread_mutex_t mu;
    int err;
} pool_t;

static void *worker(void *arg) {
    pool_t *pool = (pool_t *)arg;
    const problem_t *P = pool->P;
    const int64_t units = P->N * P->HV;
    size_t sdim = (size_t)P->dv * P->dk;
    size_t wsz = pool->chunked
        ? (size_t)P->chunk + 2 * (size_t)P->chunk * P->chunk + (size_t)P->chunk * (P->dv + P->dk) + sdim
        : 0;
    double *S = (double *)malloc(sdim * sizeof(double));
    double *work = wsz ? (double *)malloc(wsz * sizeof(double)) : NULL;
    if (!S || (wsz && !work)) {
        pthread_mutex_lock(&pool->mu); pool->err = 1; pthread_mutex_unlock(&pool->mu);
        free(S); free(work);
        return NULL;
    }
    for (;;) {
        pthread_mutex_lock(&pool->mu);
        int64_t u = pool->next++;
        pthread_mutex_unlock(&pool->mu);
        if (u >= units) break;
        int64_t n = u / P->HV;
        int h = (int)(u % P->HV);
        if (pool->chunked) run_unit_chunked(P, n, h, S, work);
        else run_unit_sequential(P, n, h, S);
    }
    free(S); free(work);
    return NULL;
}

static int run_pool(const problem_t *P, int chunked, int nthreads) {
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 512) nthreads = 512;
    pool_t pool;
    pool.P = P; pool.chunked = chunked; pool.next = 0; pool.err = 0;
    pthread_mutex_init(&pool.mu, NULL);
    pthread_t tid[512];
    int started = 0;
    for (int i = 0; i < nthreads; ++i) {
        if (pthread_create(&tid[i], NULL, worker, &pool) != 0) break;
        ++started;
    }
    if (started == 0) worker(&pool);
    for (int i = 0; i < started; ++i) pthread_join(tid[i], NULL);
    pthread_mutex_destroy(&pool.mu);
    return pool.err ? -2 : 0;
}

static int check_args(int64_t N, int HK, int HV, int dk, int dv, const int64_t *cu) {
    if (N < 0 || HK <= 0 || HV <= 0 || dk <= 0 || dv <= 0) return -1;
    if (HV % HK != 0) return -1;
    if (!cu || cu[0] != 0) return -1;
    for (int64_t n = 0; n < N; ++n) if (cu[n + 1] < cu[n]) return -1;
    return 0;
}

int gdn_oracle_prefill(const double *q, const double *k, const double *v,
                       const double *g, const double *beta, const double *h0,
                       const int64_t *cu_seqlens, int64_t N, int HK, int HV,
                       int dk, int dv, double scale, double *o, double *hT,
                       int nthreads) {
    if (check_args(N, HK, HV, dk, dv, cu_seqlens)) return -1;
    problem_t P = {q, k, v, g, beta, h0, cu_seqlens, N, HK, HV, dk, dv, 0, scale, o, hT};
    return run_pool(&P, 0, nthreads);
}

int gdn_oracle_prefill_chunked(const double *q, const double *k, const double *v,
                               const double *g, const double *beta, const double *h0,
                               const int64_t *cu_seqlens, int64_t N, int HK, int HV,
                               int dk, int dv, int chunk, double scale, double *o,
                               double *hT, int nthreads) {
    if (check_args(N, HK, HV, dk, dv, cu_seqlens)) return -1;
    if (chunk <= 0 || chunk > 256) return -1;
    problem_t P = {q, k, v, g, beta, h0, cu_seqlens, N, HK, HV, dk, dv, chunk, scale, o, hT};
    return run_pool(&P, 1, nthreads);
}

/* One decode token per sequence: q,k [N][HK][dk], v,o [N][HV][dv],
 * g,beta [N][HV], state [N][HV][dv][dk] updated in place. */
int gdn_oracle_step(const double *q, const double *k, const double *v,
                    const double *g, const double *beta, double *state,
                    int64_t N, int HK, int HV, int dk, int dv, double scale,
                    double *o) {
    if (N < 0 || HK <= 0 || HV <= 0 || dk <= 0 || dv <= 0 || HV % HK) return -1;
    const size_t sdim = (size_t)dv * dk;
    for (int64_t n = 0; n < N; ++n)
        for (int h = 0; h < HV; ++h) {
            int c = h / (HV / HK);
            double *S = state + ((size_t)n * HV + h) * sdim;
            const double *kt = k + ((size_t)n * HK + c) * dk;
            const double *qt = q + ((size_t)n * HK + c) * dk;
            const double *vt = v + ((size_t)n * HV + h) * dv;
            token_update(S, dk, dv, exp(g[n * HV + h]), beta[n * HV + h], kt, vt);
            token_readout(S, dk, dv, scale, qt, o + ((size_t)n * HV + h) * dv);
        }
    return 0;
}
