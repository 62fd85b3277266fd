/*
 * kda_oracle_bwd.c -- fp64 CPU oracle for the chunk-KDA backward (and an
 * fp64-input forward used to check it by finite differences).
 *
 * TEST INFRASTRUCTURE ONLY, like kda_oracle.c: only tests/, the smoke check and
 * bench.py's baseline legs load it; the CUDA library shares no code with it.
 *
 * The forward is the same token recurrence as kda_oracle.c (KDA: the gated
 * delta rule with a per-key-channel decay; kda_fused page of
 * nemo_automodel.components.models.kimi_k3, module description and
 * fused_chunk_kda), here on fp64 inputs:
 *
 *   q^ = q r_q, r_q = (|q|^2 + eps)^-1/2   (same for k)
 *   S' = Diag(a) S_prev,  a_c = exp(g_c)
 *   p  = S'^T k^,  e = v - p
 *   S  = S' + beta k^ e^T
 *   o  = scale S^T q^
 *
 * The backward is reverse-mode differentiation of exactly these lines, token
 * by token from the last token of a document to the first (the pages' backward
 * is a recompute-from-inputs backward producing dq, dk, dv, dg and dbeta; the
 * steps below are the chain rule applied to the forward above, written out):
 *
 *   dS  += scale q^ do^T                 (dS is the gradient of the state after t)
 *   dq^  = scale S do
 *   u    = dS e;   dbeta = k^ . u;   dk^ = beta u
 *   de   = beta dS^T k^;   dv = de;   dp = -de
 *   dS'  = dS + k^ dp^T;   dk^ += S' dp
 *   dg_c = sum_v S'[c][v] dS'[c][v]      (d/dg_c of a_c S_prev = S')
 *   dS   = Diag(a) dS'                   (gradient of the state before t)
 *   dq   = r_q (dq^ - q^ (q^ . dq^))     (l2-norm chain rule; same for k)
 *
 * The states S_prev are recomputed: the forward stores the state at every
 * 64th token, and the reverse pass re-runs the same forward lines from each
 * stored state over its 64 tokens.  The recomputed states are bit-identical to
 * the first pass (same operations in the same order); the stride only bounds
 * memory.  Chains (document, head) are independent and spread over threads.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define CKPT 64

typedef struct {
    const double *q, *k, *v, *g, *beta, *dout;
    const int32_t *cu;
    int n_docs;
    int64_t T;
    int H, K, V;
    double scale, eps;
    const int32_t *chains;
    int n_chains;
    double *out;                          /* forward: [T, H, V] */
    double *dq, *dk, *dv, *dg, *dbeta;    /* backward */
    int next;
    pthread_mutex_t mu;
} bjob_t;

/* q^ = q r, r = (|q|^2 + eps)^-1/2 */
static double normalise(const double *x, double *xn, int n, double eps) {
    double s = 0.0;
    for (int c = 0; c < n; ++c) s += x[c] * x[c];
    const double r = 1.0 / sqrt(s + eps);
    for (int c = 0; c < n; ++c) xn[c] = x[c] * r;
    return r;
}

/* one forward token: S (in: S_prev, out: S_t); Sd (if not NULL) receives S' */
static void step(double *S, double *Sd, const double *kn, const double *vt, const double *gt, double b,
                 double *p, int K, int V) {
    for (int c = 0; c < K; ++c) {
        const double a = exp(gt[c]);
        for (int x = 0; x < V; ++x) S[c * V + x] *= a;
    }
    if (Sd) memcpy(Sd, S, sizeof(double) * K * V);
    for (int x = 0; x < V; ++x) p[x] = 0.0;
    for (int c = 0; c < K; ++c)
        for (int x = 0; x < V; ++x) p[x] += S[c * V + x] * kn[c];
    for (int c = 0; c < K; ++c)
        for (int x = 0; x < V; ++x) S[c * V + x] += b * kn[c] * (vt[x] - p[x]);
}

static void fwd_chain(bjob_t *j, int idx) {
    const int chain = j->chains ? j->chains[idx] : idx;
    const int doc = chain / j->H, h = chain % j->H;
    const int K = j->K, V = j->V, H = j->H;
    const int64_t t0 = j->cu[doc], t1 = j->cu[doc + 1];
    double *S = calloc((size_t)K * V, sizeof(double));
    double *qn = malloc(sizeof(double) * K), *kn = malloc(sizeof(double) * K), *p = malloc(sizeof(double) * V);
    for (int64_t t = t0; t < t1; ++t) {
        const int64_t row = t * H + h;
        normalise(j->q + row * K, qn, K, j->eps);
        normalise(j->k + row * K, kn, K, j->eps);
        step(S, NULL, kn, j->v + row * V, j->g + row * K, j->beta[row], p, K, V);
        for (int x = 0; x < V; ++x) {
            double acc = 0.0;
            for (int c = 0; c < K; ++c) acc += S[c * V + x] * qn[c];
            j->out[row * V + x] = j->scale * acc;
        }
    }
    free(S);
    free(qn);
    free(kn);
    free(p);
}

static void bwd_chain(bjob_t *j, int idx) {
    const int chain = j->chains ? j->chains[idx] : idx;
    const int doc = chain / j->H, h = chain % j->H;
    const int K = j->K, V = j->V, H = j->H;
    const size_t KV = (size_t)K * V;
    const int64_t t0 = j->cu[doc], t1 = j->cu[doc + 1];
    const int64_t L = t1 - t0;
    if (L <= 0) return;
    const int64_t nck = (L + CKPT - 1) / CKPT;
    double *ck = malloc(sizeof(double) * KV * (size_t)nck);     /* state before token t0 + CKPT*i */
    double *blk = malloc(sizeof(double) * KV * (CKPT + 1));     /* S_prev of each token of a block, then S_last */
    double *Sd = malloc(sizeof(double) * KV);                    /* S' of the current token */
    double *S = calloc(KV, sizeof(double));
    double *dS = calloc(KV, sizeof(double));
    double *qn = malloc(sizeof(double) * K), *kn = malloc(sizeof(double) * K);
    double *p = malloc(sizeof(double) * V), *e = malloc(sizeof(double) * V), *u = malloc(sizeof(double) * K);
    double *dqn = malloc(sizeof(double) * K), *dkn = malloc(sizeof(double) * K), *dp = malloc(sizeof(double) * V);

    /* first pass: states at the checkpoints */
    for (int64_t t = t0; t < t1; ++t) {
        const int64_t row = t * H + h;
        if ((t - t0) % CKPT == 0) memcpy(ck + KV * (size_t)((t - t0) / CKPT), S, sizeof(double) * KV);
        normalise(j->k + row * K, kn, K, j->eps);
        step(S, NULL, kn, j->v + row * V, j->g + row * K, j->beta[row], p, K, V);
    }

    for (int64_t bi = nck - 1; bi >= 0; --bi) {
        const int64_t b0 = t0 + bi * CKPT, b1 = (b0 + CKPT < t1) ? b0 + CKPT : t1;
        /* recompute the block: blk[i] = state before token b0 + i */
        memcpy(S, ck + KV * (size_t)bi, sizeof(double) * KV);
        for (int64_t t = b0; t < b1; ++t) {
            const int64_t row = t * H + h;
            memcpy(blk + KV * (size_t)(t - b0), S, sizeof(double) * KV);
            normalise(j->k + row * K, kn, K, j->eps);
            step(S, NULL, kn, j->v + row * V, j->g + row * K, j->beta[row], p, K, V);
        }
        for (int64_t t = b1 - 1; t >= b0; --t) {
            const int64_t row = t * H + h;
            const double *qt = j->q + row * K, *kt = j->k + row * K, *vt = j->v + row * V;
            const double *gt = j->g + row * K, *dot = j->dout + row * V;
            const double b = j->beta[row];
            const double rq = normalise(qt, qn, K, j->eps);
            const double rk = normalise(kt, kn, K, j->eps);
            /* forward lines of token t: S' (Sd), p, e, and S_t (S) */
            memcpy(S, blk + KV * (size_t)(t - b0), sizeof(double) * KV);
            step(S, Sd, kn, vt, gt, b, p, K, V);
            for (int x = 0; x < V; ++x) e[x] = vt[x] - p[x];

            /* o = scale S^T q^ */
            for (int c = 0; c < K; ++c)
                for (int x = 0; x < V; ++x) dS[c * V + x] += j->scale * qn[c] * dot[x];
            for (int c = 0; c < K; ++c) {
                double acc = 0.0;
                for (int x = 0; x < V; ++x) acc += S[c * V + x] * dot[x];
                dqn[c] = j->scale * acc;
            }
            /* S = S' + beta k^ e^T */
            double db = 0.0;
            for (int c = 0; c < K; ++c) {
                double acc = 0.0;
                for (int x = 0; x < V; ++x) acc += dS[c * V + x] * e[x];
                u[c] = acc;
                db += kn[c] * acc;
                dkn[c] = b * acc;
            }
            for (int x = 0; x < V; ++x) {
                double acc = 0.0;
                for (int c = 0; c < K; ++c) acc += dS[c * V + x] * kn[c];
                const double de = b * acc;
                j->dv[row * V + x] = de;
                dp[x] = -de;
            }
            /* p = S'^T k^ : dS' = dS + k^ dp^T, dk^ += S' dp */
            for (int c = 0; c < K; ++c) {
                double acc = 0.0;
                for (int x = 0; x < V; ++x) {
                    dS[c * V + x] += kn[c] * dp[x];
                    acc += Sd[c * V + x] * dp[x];
                }
                dkn[c] += acc;
            }
            /* S' = Diag(exp(g)) S_prev */
            for (int c = 0; c < K; ++c) {
                double acc = 0.0;
                for (int x = 0; x < V; ++x) acc += Sd[c * V + x] * dS[c * V + x];
                j->dg[row * K + c] = acc;
                const double a = exp(gt[c]);
                for (int x = 0; x < V; ++x) dS[c * V + x] *= a;
            }
            j->dbeta[row] = db;
            /* l2-norm chain rule */
            double sq = 0.0, sk = 0.0;
            for (int c = 0; c < K; ++c) {
                sq += qn[c] * dqn[c];
                sk += kn[c] * dkn[c];
            }
            for (int c = 0; c < K; ++c) {
                j->dq[row * K + c] = rq * (dqn[c] - qn[c] * sq);
                j->dk[row * K + c] = rk * (dkn[c] - kn[c] * sk);
            }
        }
    }
    free(ck); free(blk); free(Sd); free(S); free(dS); free(qn); free(kn); free(p); free(e); free(u);
    free(dqn); free(dkn); free(dp);
}

typedef struct { bjob_t *j; int bwd; } warg_t;

static void *bworker(void *arg) {
    warg_t *w = (warg_t *)arg;
    for (;;) {
        pthread_mutex_lock(&w->j->mu);
        const int idx = w->j->next++;
        pthread_mutex_unlock(&w->j->mu);
        if (idx >= w->j->n_chains) break;
        if (w->bwd) bwd_chain(w->j, idx);
        else fwd_chain(w->j, idx);
    }
    return NULL;
}

static int run(bjob_t *j, int bwd, int n_threads) {
    if (j->n_docs < 1 || j->H < 1 || j->K < 1 || j->V < 1 || j->T < 0) return -1;
    if (j->cu[0] != 0 || j->cu[j->n_docs] != j->T) return -1;
    for (int d = 0; d < j->n_docs; ++d)
        if (j->cu[d + 1] < j->cu[d]) return -1;
    for (int i = 0; j->chains && i < j->n_chains; ++i)
        if (j->chains[i] < 0 || j->chains[i] >= j->n_docs * j->H) return -1;
    pthread_mutex_init(&j->mu, NULL);
    if (n_threads < 1) n_threads = 1;
    if (n_threads > j->n_chains) n_threads = j->n_chains > 0 ? j->n_chains : 1;
    pthread_t *th = malloc(sizeof(pthread_t) * n_threads);
    warg_t w = {j, bwd};
    for (int i = 0; i < n_threads; ++i) pthread_create(&th[i], NULL, bworker, &w);
    for (int i = 0; i < n_threads; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&j->mu);
    return 0;
}

/* fp64-input forward; chains == NULL means all chains.  Returns 0, or -1 on bad arguments. */
int kda_oracle_fwd64(const double *q, const double *k, const double *v, const double *g, const double *beta,
                     const int32_t *cu_seqlens, int n_docs, int64_t T, int H, int K, int V, double scale,
                     double eps, const int32_t *chains, int n_chains, double *out, int n_threads) {
    bjob_t j;
    memset(&j, 0, sizeof(j));
    j.q = q; j.k = k; j.v = v; j.g = g; j.beta = beta; j.cu = cu_seqlens;
    j.n_docs = n_docs; j.T = T; j.H = H; j.K = K; j.V = V; j.scale = scale; j.eps = eps;
    j.chains = chains; j.n_chains = chains ? n_chains : n_docs * H; j.out = out;
    return run(&j, 0, n_threads);
}

/* fp64 backward of o = KDA(q, k, v, g, beta) against the upstream gradient dout.
 * Gradients are written for the rows of the selected chains only. */
int kda_oracle_bwd(const double *q, const double *k, const double *v, const double *g, const double *beta,
                   const double *dout, const int32_t *cu_seqlens, int n_docs, int64_t T, int H, int K,
                   int V, double scale, double eps, const int32_t *chains, int n_chains, double *dq,
                   double *dk, double *dv, double *dg, double *dbeta, int n_threads) {
    bjob_t j;
    memset(&j, 0, sizeof(j));
    j.q = q; j.k = k; j.v = v; j.g = g; j.beta = beta; j.dout = dout; j.cu = cu_seqlens;
    j.n_docs = n_docs; j.T = T; j.H = H; j.K = K; j.V = V; j.scale = scale; j.eps = eps;
    j.chains = chains; j.n_chains = chains ? n_chains : n_docs * H;
    j.dq = dq; j.dk = dk; j.dv = dv; j.dg = dg; j.dbeta = dbeta;
    return run(&j, 1, n_threads);
}
