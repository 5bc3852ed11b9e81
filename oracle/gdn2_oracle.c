/*
 * fp64 CPU oracle for the Gated Delta Rule-2 operator.  TEST INFRASTRUCTURE
 * ONLY: the tests, the smoke check and the bench's CPU-baseline leg load this
 * library; the product path never does.  It shares no code with the CUDA
 * library.
 *
 * Source: "Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention"
 * (anthology-of-the-sota LIT-802 review, "Key takeaways" 1, paper Sec. 3.1
 * Eqs. 8-10; wispaper.ai blog, "Methodology: Gated Delta Rule-2"):
 *
 *     S_t = (I - k_t (b_t . k_t)^T) D_t S_{t-1} + k_t (w_t . v_t)^T,
 *     D_t = diag(exp g_t),
 *
 * with b_t (erase gate) on the key axis and w_t (write gate) on the value
 * axis.  The pages never write the read; it is taken to be o_t = S_t^T q_t
 * after the update, with no scale.  The KDA and Gated DeltaNet recurrences
 * (the same review's App. A.5 ties; digg thread 10/) are written here in their
 * own literal matrix form, independently of the Gated Delta Rule-2 loop, so
 * that the tie identities can pin it.
 *
 * Layouts: q, k, g, b are [B, T, H, dk]; v, w, o are [B, T, H, dv]; the state
 * is [B, H, dk, dv] with dv fastest.  All arithmetic is double precision.
 * Every (b, h) pair is an independent problem; pairs are spread over
 * `nthreads` POSIX threads.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- helpers */

typedef struct {
    int B, T, H, dk, dv;
} dims_t;

static size_t tok_off(const dims_t *d, int bi, int t, int h, int width) {
    return (((size_t)bi * d->T + t) * d->H + h) * (size_t)width;
}

static size_t state_off(const dims_t *d, int bi, int h) {
    return ((size_t)bi * d->H + h) * (size_t)d->dk * d->dv;
}

typedef void (*pair_fn)(void *ctx, int bi, int h);

typedef struct {
    pair_fn fn;
    void *ctx;
    int B, H, nthreads, tid;
} worker_arg;

static void *worker(void *p) {
    worker_arg *a = (worker_arg *)p;
    int npairs = a->B * a->H;
    for (int i = a->tid; i < npairs; i += a->nthreads) a->fn(a->ctx, i / a->H, i % a->H);
    return NULL;
}

static void for_each_pair(pair_fn fn, void *ctx, int B, int H, int nthreads) {
    int npairs = B * H;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > npairs) nthreads = npairs;
    if (nthreads == 1) {
        for (int i = 0; i < npairs; ++i) fn(ctx, i / H, i % H);
        return;
    }
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
    worker_arg *args = (worker_arg *)malloc(sizeof(worker_arg) * nthreads);
    for (int t = 0; t < nthreads; ++t) {
        args[t].fn = fn; args[t].ctx = ctx; args[t].B = B; args[t].H = H;
        args[t].nthreads = nthreads; args[t].tid = t;
        pthread_create(&th[t], NULL, worker, &args[t]);
    }
    for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    free(th); free(args);
}

/* ------------------------------------------- Gated Delta Rule-2: forward */

/* One token of the recurrence, in place on S (dk x dv).  Decomposed as
 *   S' = D_t S;   delta = w.v - S'^T (b.k);   S = S' + k delta^T;
 * which expands to (I - k (b.k)^T) D_t S + k (w.v)^T.  `delta` (dv) is
 * scratch; if `Sprime` is non-NULL it receives S'. */
static void gdr2_token(double *S, const double *k, const double *v, const double *g,
                       const double *b, const double *w, double *delta, double *Sprime,
                       int dk, int dv) {
    for (int i = 0; i < dk; ++i) {
        double a = exp(g[i]);
        for (int j = 0; j < dv; ++j) S[i * dv + j] *= a;
    }
    if (Sprime) memcpy(Sprime, S, sizeof(double) * (size_t)dk * dv);
    for (int j = 0; j < dv; ++j) delta[j] = w[j] * v[j];
    for (int i = 0; i < dk; ++i) {
        double bk = b[i] * k[i];
        for (int j = 0; j < dv; ++j) delta[j] -= S[i * dv + j] * bk;
    }
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) S[i * dv + j] += k[i] * delta[j];
}

/* o = S^T q */
static void read_out(const double *S, const double *q, double *o, int dk, int dv) {
    for (int j = 0; j < dv; ++j) o[j] = 0.0;
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) o[j] += S[i * dv + j] * q[i];
}

typedef struct {
    dims_t d;
    const double *q, *k, *v, *g, *b, *w, *S0;
    double *o, *ST;
} fwd_ctx;

static void fwd_pair(void *p, int bi, int h) {
    fwd_ctx *c = (fwd_ctx *)p;
    const dims_t *d = &c->d;
    int dk = d->dk, dv = d->dv;
    double *S = (double *)calloc((size_t)dk * dv, sizeof(double));
    double *delta = (double *)malloc(sizeof(double) * dv);
    if (c->S0) memcpy(S, c->S0 + state_off(d, bi, h), sizeof(double) * (size_t)dk * dv);
    for (int t = 0; t < d->T; ++t) {
        size_t ok = tok_off(d, bi, t, h, dk), ov = tok_off(d, bi, t, h, dv);
        gdr2_token(S, c->k + ok, c->v + ov, c->g + ok, c->b + ok, c->w + ov, delta, NULL, dk, dv);
        if (c->o) read_out(S, c->q + ok, c->o + ov, dk, dv);
    }
    if (c->ST) memcpy(c->ST + state_off(d, bi, h), S, sizeof(double) * (size_t)dk * dv);
    free(S); free(delta);
}

/* Token-wise forward.  S0 may be NULL (zero state); o and ST may be NULL. */
int gdn2_oracle_forward(const double *q, const double *k, const double *v, const double *g,
                        const double *b, const double *w, const double *S0, double *o,
                        double *ST, int B, int T, int H, int dk, int dv, int nthreads) {
    if (B < 1 || T < 0 || H < 1 || dk < 1 || dv < 1) return 1;
    fwd_ctx c = {{B, T, H, dk, dv}, q, k, v, g, b, w, S0, o, ST};
    for_each_pair(fwd_pair, &c, B, H, nthreads);
    return 0;
}

/* ------------------------------------------ Gated Delta Rule-2: backward */

/* Reverse mode of the token loop for the loss L = <o, dO> + <S_T, dS_T>.
 * States are rebuilt by replaying the forward from fp64 checkpoints taken
 * every `ckpt` tokens.  For token t, with dS = dL/dS_t carried from t+1:
 *   o = S_t^T q         : dS += q dO^T,  dq = S_t dO
 *   S_t = S' + k delta^T : dk = dS delta, ddelta = dS^T k, dS' = dS
 *   delta = w.v - r      : dw = ddelta.v, dv = ddelta.w, dr = -ddelta
 *   r = S'^T (b.k)       : dS' += (b.k) dr^T, d(b.k) = S' dr
 *   (b.k)                : db = d(b.k).k, dk += d(b.k).b
 *   S' = D_t S_{t-1}     : dg = rowsum(dS' . S'), dS_{t-1} = D_t dS'
 */
typedef struct {
    dims_t d;
    const double *q, *k, *v, *g, *b, *w, *S0, *dO, *dST;
    double *dq, *dk, *dv, *dg, *db, *dw, *dS0;
    int ckpt;
} bwd_ctx;

static void bwd_pair(void *p, int bi, int h) {
    bwd_ctx *c = (bwd_ctx *)p;
    const dims_t *d = &c->d;
    const int dk = d->dk, dv = d->dv, T = d->T, C = c->ckpt;
    const size_t KV = (size_t)dk * dv;
    const int nseg = (T + C - 1) / C;
    double *ck = (double *)malloc(sizeof(double) * KV * (size_t)(nseg > 0 ? nseg : 1));
    double *seg = (double *)malloc(sizeof(double) * KV * (size_t)(C + 1)); /* S_{t0-1}..S_{t0+C-1} */
    double *segp = (double *)malloc(sizeof(double) * KV * (size_t)C);      /* S' per token */
    double *segd = (double *)malloc(sizeof(double) * (size_t)dv * C);      /* delta per token */
    double *S = (double *)calloc(KV, sizeof(double));
    double *dS = (double *)calloc(KV, sizeof(double));
    double *ddelta = (double *)malloc(sizeof(double) * dv);
    double *dr = (double *)malloc(sizeof(double) * dv);
    double *dbk = (double *)malloc(sizeof(double) * dk);
    if (c->S0) memcpy(S, c->S0 + state_off(d, bi, h), sizeof(double) * KV);
    /* forward pass: checkpoint S_{sC-1} (the state entering segment s) */
    for (int s = 0; s < nseg; ++s) {
        memcpy(ck + KV * s, S, sizeof(double) * KV);
        for (int t = s * C; t < T && t < (s + 1) * C; ++t) {
            size_t ok = tok_off(d, bi, t, h, dk), ov = tok_off(d, bi, t, h, dv);
            gdr2_token(S, c->k + ok, c->v + ov, c->g + ok, c->b + ok, c->w + ov, ddelta, NULL, dk, dv);
        }
    }
    if (c->dST) memcpy(dS, c->dST + state_off(d, bi, h), sizeof(double) * KV);
    for (int s = nseg - 1; s >= 0; --s) {
        int t0 = s * C, t1 = (s + 1) * C < T ? (s + 1) * C : T;
        memcpy(seg, ck + KV * s, sizeof(double) * KV);
        for (int t = t0; t < t1; ++t) {
            size_t ok = tok_off(d, bi, t, h, dk), ov = tok_off(d, bi, t, h, dv);
            double *cur = seg + KV * (t - t0 + 1);
            memcpy(cur, seg + KV * (t - t0), sizeof(double) * KV);
            gdr2_token(cur, c->k + ok, c->v + ov, c->g + ok, c->b + ok, c->w + ov,
                       segd + (size_t)dv * (t - t0), segp + KV * (t - t0), dk, dv);
        }
        for (int t = t1 - 1; t >= t0; --t) {
            size_t ok = tok_off(d, bi, t, h, dk), ov = tok_off(d, bi, t, h, dv);
            const double *St = seg + KV * (t - t0 + 1);
            const double *Sp = segp + KV * (t - t0);
            const double *delta = segd + (size_t)dv * (t - t0);
            const double *qt = c->q + ok, *kt = c->k + ok, *gt = c->g + ok, *bt = c->b + ok;
            const double *vt = c->v + ov, *wt = c->w + ov, *dOt = c->dO + ov;
            double *dqt = c->dq + ok, *dkt = c->dk + ok, *dgt = c->dg + ok, *dbt = c->db + ok;
            double *dvt = c->dv + ov, *dwt = c->dw + ov;
            /* read */
            for (int i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dv; ++j) {
                    dS[i * dv + j] += qt[i] * dOt[j];
                    acc += St[i * dv + j] * dOt[j];
                }
                dqt[i] = acc;
            }
            /* write */
            for (int j = 0; j < dv; ++j) ddelta[j] = 0.0;
            for (int i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dv; ++j) {
                    acc += dS[i * dv + j] * delta[j];
                    ddelta[j] += dS[i * dv + j] * kt[i];
                }
                dkt[i] = acc;
            }
            for (int j = 0; j < dv; ++j) {
                dwt[j] = ddelta[j] * vt[j];
                dvt[j] = ddelta[j] * wt[j];
                dr[j] = -ddelta[j];
            }
            /* erase read r = S'^T (b.k) */
            for (int i = 0; i < dk; ++i) {
                double acc = 0.0, bk = bt[i] * kt[i];
                for (int j = 0; j < dv; ++j) {
                    acc += Sp[i * dv + j] * dr[j];
                    dS[i * dv + j] += bk * dr[j];
                }
                dbk[i] = acc;
            }
            for (int i = 0; i < dk; ++i) {
                dbt[i] = dbk[i] * kt[i];
                dkt[i] += dbk[i] * bt[i];
            }
            /* decay */
            for (int i = 0; i < dk; ++i) {
                double acc = 0.0, a = exp(gt[i]);
                for (int j = 0; j < dv; ++j) {
                    acc += dS[i * dv + j] * Sp[i * dv + j];
                    dS[i * dv + j] *= a;
                }
                dgt[i] = acc;
            }
        }
    }
    if (c->dS0) memcpy(c->dS0 + state_off(d, bi, h), dS, sizeof(double) * KV);
    free(ck); free(seg); free(segp); free(segd); free(S); free(dS);
    free(ddelta); free(dr); free(dbk);
}

/* Token-wise reverse mode.  S0 and dST may be NULL (zero); dS0 may be NULL.
 * ckpt >= 1 is the replay segment length. */
int gdn2_oracle_backward(const double *q, const double *k, const double *v, const double *g,
                         const double *b, const double *w, const double *S0, const double *dO,
                         const double *dST, double *dq, double *dk, double *dv, double *dg,
                         double *db, double *dw, double *dS0, int B, int T, int H, int dk_,
                         int dv_, int ckpt, int nthreads) {
    if (B < 1 || T < 0 || H < 1 || dk_ < 1 || dv_ < 1 || ckpt < 1) return 1;
    bwd_ctx c = {{B, T, H, dk_, dv_}, q, k, v, g, b, w, S0, dO, dST,
                 dq, dk, dv, dg, db, dw, dS0, ckpt};
    for_each_pair(bwd_pair, &c, B, H, nthreads);
    return 0;
}

/* ------------------------------------- KDA and Gated DeltaNet (for ties) */

/* KDA (Kimi Delta Attention), as the matrix product it is written as:
 *   S_t = (I - beta_t k_t k_t^T) Diag(exp g_t) S_{t-1} + beta_t k_t v_t^T.
 * Gated DeltaNet, likewise:
 *   S_t = exp(a_t) (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,
 * with one scalar log-decay a_t per token and head.  The erase operator
 * E = I - beta k k^T is formed explicitly (dk x dk) and applied as a matrix
 * product, unlike the rank-one read-subtract-write of the loop above.
 * beta is [B, T, H]; for Gated DeltaNet g is [B, T, H] too. */
typedef struct {
    dims_t d;
    const double *q, *k, *v, *g, *beta, *S0;
    double *o, *ST;
    int scalar_decay;
} tie_ctx;

static void tie_pair(void *p, int bi, int h) {
    tie_ctx *c = (tie_ctx *)p;
    const dims_t *d = &c->d;
    const int dk = d->dk, dv = d->dv;
    const size_t KV = (size_t)dk * dv;
    double *S = (double *)calloc(KV, sizeof(double));
    double *M = (double *)malloc(sizeof(double) * KV);
    double *E = (double *)malloc(sizeof(double) * (size_t)dk * dk);
    if (c->S0) memcpy(S, c->S0 + state_off(d, bi, h), sizeof(double) * KV);
    for (int t = 0; t < d->T; ++t) {
        size_t ok = tok_off(d, bi, t, h, dk), ov = tok_off(d, bi, t, h, dv);
        size_t os = tok_off(d, bi, t, h, 1);
        const double *kt = c->k + ok, *vt = c->v + ov;
        double beta = c->beta[os];
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dk; ++j) E[i * dk + j] = (i == j ? 1.0 : 0.0) - beta * kt[i] * kt[j];
        if (c->scalar_decay) {
            double a = exp(c->g[os]);
            /* M = E S, then S = a M + beta k v^T */
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int l = 0; l < dk; ++l) acc += E[i * dk + l] * S[l * dv + j];
                    M[i * dv + j] = acc;
                }
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) S[i * dv + j] = a * M[i * dv + j] + beta * kt[i] * vt[j];
        } else {
            const double *gt = c->g + ok;
            /* M = Diag(exp g) S, then S = E M + beta k v^T */
            for (int i = 0; i < dk; ++i) {
                double a = exp(gt[i]);
                for (int j = 0; j < dv; ++j) M[i * dv + j] = a * S[i * dv + j];
            }
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int l = 0; l < dk; ++l) acc += E[i * dk + l] * M[l * dv + j];
                    S[i * dv + j] = acc + beta * kt[i] * vt[j];
                }
        }
        if (c->o) {
            const double *qt = c->q + ok;
            double *ot = c->o + ov;
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += qt[i] * S[i * dv + j];
                ot[j] = acc;
            }
        }
    }
    if (c->ST) memcpy(c->ST + state_off(d, bi, h), S, sizeof(double) * KV);
    free(S); free(M); free(E);
}

int kda_oracle_forward(const double *q, const double *k, const double *v, const double *g,
                       const double *beta, const double *S0, double *o, double *ST,
                       int B, int T, int H, int dk, int dv, int nthreads) {
    if (B < 1 || T < 0 || H < 1 || dk < 1 || dv < 1) return 1;
    tie_ctx c = {{B, T, H, dk, dv}, q, k, v, g, beta, S0, o, ST, 0};
    for_each_pair(tie_pair, &c, B, H, nthreads);
    return 0;
}

int gdn_oracle_forward(const double *q, const double *k, const double *v, const double *alpha_log,
                       const double *beta, const double *S0, double *o, double *ST,
                       int B, int T, int H, int dk, int dv, int nthreads) {
    if (B < 1 || T < 0 || H < 1 || dk < 1 || dv < 1) return 1;
    tie_ctx c = {{B, T, H, dk, dv}, q, k, v, alpha_log, beta, S0, o, ST, 1};
    for_each_pair(tie_pair, &c, B, H, nthreads);
    return 0;
}
