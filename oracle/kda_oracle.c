/*
 * kda_oracle.c -- fp64 CPU oracle for the chunk-KDA forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py load this library.  The product
 * path (libkda, the CUDA kernels) shares no code with it and never calls it.
 *
 * What it computes: Kimi Delta Attention (KDA), the gated delta rule with a
 * per-key-channel decay, run token by token with no chunking at all.  For each
 * packed document (the state resets at every document boundary, as the
 * fused-kernel contract on the kda_fused page of
 * nemo_automodel.components.models.kimi_k3 states for the packed layout) and
 * each head, starting from the zero state S (K x V, rows = key channels,
 * columns = value channels):
 *
 *   q^ = q / sqrt(|q|^2 + eps),  k^ = k / sqrt(|k|^2 + eps)
 *        (q/k l2-normalised inside the op, kda_fused page, module description)
 *   S' = Diag(exp(g_t)) S                      decay first, per key channel
 *   S  = S' + beta_t k^ (v_t - S'^T k^)^T      = (I - beta k^ k^T) S' + beta k^ v^T
 *   o_t = scale * S^T q^                       uses the state after token t
 *
 * Everything is computed in double precision from the exact input values
 * (bf16 q/k/v widened to fp32 by the caller, fp32 g and beta).  No chunking,
 * blocking or reordering: a reader can check each line against the formulas
 * above.  Chains (document, head) are independent and are spread over
 * threads; inside a chain the loop over tokens is strictly sequential, so the
 * result does not depend on the thread count.
 *
 * The state may start from a given S_0 (initial_state, one K x V matrix per
 * (document, head) chain) instead of zero, and the state after a document's
 * last token can be returned (final_state): FLA's initial/final state
 * convention, which the fused contract leaves out and the library offers as
 * an extension.
 *
 * erase = 0 drops the "- S'^T k^" term (test-only switch): the recurrence then
 * becomes gated linear attention, which has an independent closed form that
 * the tests use to pin the decay bookkeeping.
 *
 * Parity pins for this file live in tests/test_oracle.py.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    const float *q, *k, *v, *g, *beta;
    const int32_t *cu;
    int n_docs;
    int64_t T;
    int H, K, V;
    double scale, eps;
    int erase;
    const int32_t *chains;   /* chain id = doc * H + head */
    int n_chains;
    double *out;             /* [T, H, V] */
    double *final_state;     /* [n_chains, K, V] or NULL */
    const float *initial_state;  /* [n_docs * H, K, V] by chain id, or NULL (zero) */
    int next;                /* work counter */
    pthread_mutex_t mu;
} job_t;

static void run_chain(job_t *j, int idx) {
    const int chain = j->chains ? j->chains[idx] : idx;
    const int doc = chain / j->H, h = chain % j->H;
    const int K = j->K, V = j->V, H = j->H;
    const int64_t t0 = j->cu[doc], t1 = j->cu[doc + 1];
    double *S = calloc((size_t)K * V, sizeof(double));
    if (j->initial_state)
        for (size_t e = 0; e < (size_t)K * V; ++e) S[e] = j->initial_state[(size_t)chain * K * V + e];
    double *qn = malloc(sizeof(double) * K), *kn = malloc(sizeof(double) * K);
    double *p = malloc(sizeof(double) * V);
    for (int64_t t = t0; t < t1; ++t) {
        const float *qt = j->q + (t * H + h) * K;
        const float *kt = j->k + (t * H + h) * K;
        const float *vt = j->v + (t * H + h) * V;
        const float *gt = j->g + (t * H + h) * K;
        const double b = j->beta[t * H + h];
        double sq = 0.0, sk = 0.0;
        for (int c = 0; c < K; ++c) {
            sq += (double)qt[c] * qt[c];
            sk += (double)kt[c] * kt[c];
        }
        const double rq = 1.0 / sqrt(sq + j->eps), rk = 1.0 / sqrt(sk + j->eps);
        for (int c = 0; c < K; ++c) {
            qn[c] = qt[c] * rq;
            kn[c] = kt[c] * rk;
        }
        /* S' = Diag(exp(g_t)) S */
        for (int c = 0; c < K; ++c) {
            const double a = exp((double)gt[c]);
            for (int x = 0; x < V; ++x) S[c * V + x] *= a;
        }
        /* p = S'^T k^ (the value S' currently stores under key k^) */
        for (int x = 0; x < V; ++x) p[x] = 0.0;
        if (j->erase)
            for (int c = 0; c < K; ++c)
                for (int x = 0; x < V; ++x) p[x] += S[c * V + x] * kn[c];
        /* S = S' + beta k^ (v - p)^T */
        for (int c = 0; c < K; ++c)
            for (int x = 0; x < V; ++x) S[c * V + x] += b * kn[c] * ((double)vt[x] - p[x]);
        /* o = scale S^T q^ */
        double *ot = j->out + (t * H + h) * V;
        for (int x = 0; x < V; ++x) {
            double acc = 0.0;
            for (int c = 0; c < K; ++c) acc += S[c * V + x] * qn[c];
            ot[x] = j->scale * acc;
        }
    }
    if (j->final_state) memcpy(j->final_state + (size_t)idx * K * V, S, sizeof(double) * K * V);
    free(S);
    free(qn);
    free(kn);
    free(p);
}

static void *worker(void *arg) {
    job_t *j = (job_t *)arg;
    for (;;) {
        pthread_mutex_lock(&j->mu);
        const int idx = j->next++;
        pthread_mutex_unlock(&j->mu);
        if (idx >= j->n_chains) break;
        run_chain(j, idx);
    }
    return NULL;
}

/* Returns 0 on success, -1 on a malformed cu_seqlens table or bad sizes.
 * chains == NULL means every (doc, head) chain, in the order doc * H + head.
 * Only output rows of the selected chains are written. */
int kda_oracle_fwd(const float *q, const float *k, const float *v, const float *g,
                   const float *beta, const int32_t *cu_seqlens, int n_docs, int64_t T,
                   int H, int K, int V, double scale, double eps, int erase,
                   const int32_t *chains, int n_chains, double *out, double *final_state,
                   const float *initial_state, int n_threads) {
    if (n_docs < 1 || H < 1 || K < 1 || V < 1 || T < 0) return -1;
    if (cu_seqlens[0] != 0 || cu_seqlens[n_docs] != T) return -1;
    for (int d = 0; d < n_docs; ++d)
        if (cu_seqlens[d + 1] < cu_seqlens[d]) return -1;
    job_t j = {q, k, v, g, beta, cu_seqlens, n_docs, T, H, K, V, scale, eps, erase,
               chains, chains ? n_chains : n_docs * H, out, final_state, initial_state, 0};
    for (int i = 0; chains && i < n_chains; ++i)
        if (chains[i] < 0 || chains[i] >= n_docs * H) return -1;
    pthread_mutex_init(&j.mu, NULL);
    if (n_threads < 1) n_threads = 1;
    if (n_threads > j.n_chains) n_threads = j.n_chains > 0 ? j.n_chains : 1;
    pthread_t *th = malloc(sizeof(pthread_t) * n_threads);
    for (int i = 0; i < n_threads; ++i) pthread_create(&th[i], NULL, worker, &j);
    for (int i = 0; i < n_threads; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&j.mu);
    return 0;
}
