/* CPU oracle for the gated delta rule (Gated DeltaNet token mixing).
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the CPU
 * baseline leg of bench.py load this library.  It shares no code, header,
 * table or helper with the CUDA library; the two meet only on the seeded
 * inputs drawn by linear_attention_token_b200/inputs.py.
 *
 * Source: "論文解説: Qwen3.8-Next の設計" (ta-paperlens), section "GDNの中身":
 *   Eq. (1)   S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T
 *   text under Eq. (1): alpha_t in (0,1) is the decay gate, beta_t in (0,1) the
 *             write strength;
 *   concept code: the output is read after the update, y = S^T q.
 * Readings where the pages are silent:
 *   alpha_t = exp(g_t); S is dk x dv with dv contiguous; value head h reads
 *   q/k head h / (H_v / H_qk); the output is multiplied by `scale`; the optional
 *   q/k L2 normalisation divides by sqrt(sum x^2 + 1e-6).
 *
 * Entry points (all layouts row-major, sequences delimited by cu_seqlens):
 *   q, k [T_total, H_qk, dk]; v, out [T_total, H_v, dv]; g, beta [T_total, H_v];
 *   S0, S_final [num_seqs, H_v, dk, dv] (S0 may be NULL -> zero state;
 *   S_final may be NULL).
 *   gdn_oracle_recurrent_f64  sequential Eq. (1) in double   (the parity oracle)
 *   gdn_oracle_recurrent_f32  the same in float              (timed CPU baseline)
 *   gdn_oracle_chunked_f64    the chunked (WY / UT) re-association in double,
 *                             chunk size C, used only to pin the chunk algebra
 *                             against the sequential form.
 * Threads: jobs are (sequence, value head) pairs spread over `threads` POSIX
 * threads (threads <= 0 -> all online cores).  Returns 0, or -1 on bad sizes.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

typedef struct {
    const void *q, *k, *v, *g, *beta, *S0;
    void *out, *S_final;
    const int64_t *cu_seqlens;
    int num_seqs, H_qk, H_v, dk, dv, l2norm, chunk;
    double scale;
} oracle_args;

/* ---- sequential recurrence, double and float ---------------------------- */
#define REAL double
#define SFX(name) name##_f64
#define EXP exp
#define SQRT sqrt
#include "recurrence.inc"
#undef REAL
#undef SFX
#undef EXP
#undef SQRT

#define REAL float
#define SFX(name) name##_f32
#define EXP expf
#define SQRT sqrtf
#include "recurrence.inc"
#undef REAL
#undef SFX
#undef EXP
#undef SQRT

/* ---- chunked form (double) ------------------------------------------------
 * Within a chunk of L tokens starting from state S (notation: G_i = sum_{s<=i}
 * g_s, gamma_i = exp(G_i)), unrolling Eq. (1) as S_i = alpha_i S_{i-1} + k_i u_i^T
 * with u_i = beta_i (v_i - alpha_i S_{i-1}^T k_i) gives
 *   (I + A) U = diag(beta) V - diag(beta gamma) K S,
 *   A_ij = beta_i exp(G_i - G_j) k_i.k_j  (j < i), 0 otherwise,
 * so with T = (I + A)^-1, W = T diag(beta gamma) K, Ut = T diag(beta) V:
 *   U = Ut - W S
 *   O = diag(gamma) Q S + P U,   P_ij = exp(G_i - G_j) q_i.k_j  (j <= i)
 *   S <- gamma_{L-1} S + sum_j exp(G_{L-1} - G_j) k_j u_j^T
 */
static void chunked_one(const oracle_args *A, int n, int h)
{
    const int dk = A->dk, dv = A->dv, C = A->chunk;
    const int hq = h / (A->H_v / A->H_qk);
    const int64_t t_begin = A->cu_seqlens[n], t_end = A->cu_seqlens[n + 1];
    const double *q = A->q, *k = A->k, *v = A->v, *g = A->g, *beta = A->beta;
    double *out = A->out;

    double *S = calloc((size_t)dk * dv, sizeof(double));
    double *K = malloc(sizeof(double) * C * dk), *Q = malloc(sizeof(double) * C * dk);
    double *V = malloc(sizeof(double) * C * dv);
    double *G = malloc(sizeof(double) * C), *b = malloc(sizeof(double) * C);
    double *Am = malloc(sizeof(double) * C * C), *T = malloc(sizeof(double) * C * C);
    double *P = malloc(sizeof(double) * C * C);
    double *W = malloc(sizeof(double) * C * dk), *U = malloc(sizeof(double) * C * dv);
    double *O = malloc(sizeof(double) * C * dv), *Snew = malloc(sizeof(double) * dk * dv);

    if (A->S0)
        memcpy(S, (const double *)A->S0 + ((size_t)n * A->H_v + h) * dk * dv,
               sizeof(double) * dk * dv);

    for (int64_t c0 = t_begin; c0 < t_end; c0 += C) {
        const int L = (int)((t_end - c0) < C ? (t_end - c0) : C);
        for (int i = 0; i < L; ++i) {
            const int64_t t = c0 + i;
            const double *kin = k + ((size_t)t * A->H_qk + hq) * dk;
            const double *qin = q + ((size_t)t * A->H_qk + hq) * dk;
            double sk = 0, sq = 0;
            for (int d = 0; d < dk; ++d) { sk += kin[d] * kin[d]; sq += qin[d] * qin[d]; }
            const double rk = A->l2norm ? 1.0 / sqrt(sk + 1e-6) : 1.0;
            const double rq = A->l2norm ? 1.0 / sqrt(sq + 1e-6) : 1.0;
            for (int d = 0; d < dk; ++d) { K[i * dk + d] = kin[d] * rk; Q[i * dk + d] = qin[d] * rq; }
            for (int e = 0; e < dv; ++e) V[i * dv + e] = v[((size_t)t * A->H_v + h) * dv + e];
            G[i] = (i ? G[i - 1] : 0.0) + g[(size_t)t * A->H_v + h];
            b[i] = beta[(size_t)t * A->H_v + h];
        }
        /* A (strictly lower) and P (lower incl. diagonal) */
        for (int i = 0; i < L; ++i)
            for (int j = 0; j < L; ++j) {
                double kk = 0, qk = 0;
                for (int d = 0; d < dk; ++d) { kk += K[i * dk + d] * K[j * dk + d]; qk += Q[i * dk + d] * K[j * dk + d]; }
                Am[i * C + j] = (j < i) ? b[i] * exp(G[i] - G[j]) * kk : 0.0;
                P[i * C + j] = (j <= i) ? exp(G[i] - G[j]) * qk : 0.0;
            }
        /* T = (I + A)^-1 by forward substitution (unit lower triangular) */
        for (int i = 0; i < L; ++i)
            for (int j = 0; j < L; ++j) {
                if (j > i) { T[i * C + j] = 0.0; continue; }
                double acc = (i == j) ? 1.0 : 0.0;
                for (int m = j; m < i; ++m) acc -= Am[i * C + m] * T[m * C + j];
                T[i * C + j] = acc;
            }
        /* W = T diag(beta gamma) K ; U = T diag(beta) V - W S */
        for (int i = 0; i < L; ++i) {
            for (int d = 0; d < dk; ++d) {
                double acc = 0;
                for (int j = 0; j <= i; ++j) acc += T[i * C + j] * b[j] * exp(G[j]) * K[j * dk + d];
                W[i * dk + d] = acc;
            }
            for (int e = 0; e < dv; ++e) {
                double acc = 0;
                for (int j = 0; j <= i; ++j) acc += T[i * C + j] * b[j] * V[j * dv + e];
                for (int d = 0; d < dk; ++d) acc -= W[i * dk + d] * S[d * dv + e];
                U[i * dv + e] = acc;
            }
        }
        /* O = diag(gamma) Q S + P U */
        for (int i = 0; i < L; ++i)
            for (int e = 0; e < dv; ++e) {
                double qs = 0, pu = 0;
                for (int d = 0; d < dk; ++d) qs += Q[i * dk + d] * S[d * dv + e];
                for (int j = 0; j <= i; ++j) pu += P[i * C + j] * U[j * dv + e];
                O[i * dv + e] = exp(G[i]) * qs + pu;
                out[((size_t)(c0 + i) * A->H_v + h) * dv + e] = A->scale * O[i * dv + e];
            }
        /* S <- gamma_{L-1} S + sum_j exp(G_{L-1} - G_j) k_j u_j^T */
        for (int d = 0; d < dk; ++d)
            for (int e = 0; e < dv; ++e) {
                double acc = exp(G[L - 1]) * S[d * dv + e];
                for (int j = 0; j < L; ++j) acc += exp(G[L - 1] - G[j]) * K[j * dk + d] * U[j * dv + e];
                Snew[d * dv + e] = acc;
            }
        memcpy(S, Snew, sizeof(double) * dk * dv);
    }
    if (A->S_final)
        memcpy((double *)A->S_final + ((size_t)n * A->H_v + h) * dk * dv, S, sizeof(double) * dk * dv);
    free(S); free(K); free(Q); free(V); free(G); free(b); free(Am); free(T); free(P);
    free(W); free(U); free(O); free(Snew);
}

/* ---- thread pool over (sequence, value head) jobs ----------------------- */
typedef struct {
    const oracle_args *A;
    void (*fn)(const oracle_args *, int, int);
    int64_t next;        /* shared job counter */
} pool_t;

static void *worker(void *p)
{
    pool_t *P = (pool_t *)p;
    const int64_t jobs = (int64_t)P->A->num_seqs * P->A->H_v;
    for (;;) {
        const int64_t j = __atomic_fetch_add(&P->next, 1, __ATOMIC_RELAXED);
        if (j >= jobs) break;
        P->fn(P->A, (int)(j / P->A->H_v), (int)(j % P->A->H_v));
    }
    return NULL;
}

static int run_pool(const oracle_args *A, void (*fn)(const oracle_args *, int, int), int threads)
{
    if (A->num_seqs < 0 || A->H_qk <= 0 || A->H_v <= 0 || A->dk <= 0 || A->dv <= 0 ||
        A->H_v % A->H_qk != 0)
        return -1;
    for (int n = 0; n < A->num_seqs; ++n)
        if (A->cu_seqlens[n + 1] < A->cu_seqlens[n]) return -1;
    if (threads <= 0) threads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (threads < 1) threads = 1;
    pool_t P = {A, fn, 0};
    pthread_t *tid = malloc(sizeof(pthread_t) * threads);
    int started = 0;
    for (int i = 0; i < threads; ++i)
        if (pthread_create(&tid[i], NULL, worker, &P) == 0) ++started;
    if (started == 0) worker(&P);
    for (int i = 0; i < started; ++i) pthread_join(tid[i], NULL);
    free(tid);
    return 0;
}

#define ORACLE_ARGS_FROM_PARAMS                                                         \
    oracle_args A = {q, k, v, g, beta, S0, out, S_final, cu_seqlens, num_seqs, H_qk, H_v, \
                     dk, dv, l2norm, 0, scale}

int gdn_oracle_recurrent_f64(const double *q, const double *k, const double *v,
                             const double *g, const double *beta, const double *S0,
                             double *out, double *S_final, const int64_t *cu_seqlens,
                             int num_seqs, int H_qk, int H_v, int dk, int dv,
                             double scale, int l2norm, int threads)
{
    ORACLE_ARGS_FROM_PARAMS;
    return run_pool(&A, recurrent_one_f64, threads);
}

int gdn_oracle_recurrent_f32(const float *q, const float *k, const float *v,
                             const float *g, const float *beta, const float *S0,
                             float *out, float *S_final, const int64_t *cu_seqlens,
                             int num_seqs, int H_qk, int H_v, int dk, int dv,
                             double scale, int l2norm, int threads)
{
    ORACLE_ARGS_FROM_PARAMS;
    return run_pool(&A, recurrent_one_f32, threads);
}

int gdn_oracle_chunked_f64(const double *q, const double *k, const double *v,
                           const double *g, const double *beta, const double *S0,
                           double *out, double *S_final, const int64_t *cu_seqlens,
                           int num_seqs, int H_qk, int H_v, int dk, int dv,
                           double scale, int l2norm, int chunk, int threads)
{
    ORACLE_ARGS_FROM_PARAMS;
    if (chunk <= 0) return -1;
    A.chunk = chunk;
    return run_pool(&A, chunked_one, threads);
}

/* Number of threads a call with `threads` <= 0 would use. */
int gdn_oracle_default_threads(void) { return (int)sysconf(_SC_NPROCESSORS_ONLN); }
