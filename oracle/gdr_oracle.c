/*
 * gdr_oracle.c -- plain fp64 CPU oracle for the gated delta rule forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path calls this file: it is
 * used by tests/, by the smoke check and by the benchmark's CPU-baseline leg.
 * It shares no code with the CUDA library.
 *
 * What it computes (per sequence-head, independently, in double precision):
 *
 *   Gated DeltaNet-2 update (Gated DeltaNet-2 Q&A page, Q3 "update equation";
 *   Gated DeltaNet-2 Review §3-1):
 *       S_t = (I - k_t (b_t . k_t)^T) D_t S_{t-1} + k_t (w_t . v_t)^T,
 *       D_t = diag(exp(g_t)),  S in R^{dk x dv}
 *   read-out with the current state (Gated DeltaNet explainer, "Mechanism":
 *   y = S^T q):
 *       o_t = S_t^T q_t
 *
 *   The loop applies the same product term by term:
 *       S <- D_t S                      (decay)
 *       r  = S^T (b_t . k_t)            (read along b.k from the decayed state)
 *       S <- S + k_t (w_t . v_t - r)^T  (erase along k and write w.v along k)
 *       o_t = S^T q_t
 *   because (I - k (b.k)^T) D S + k (w.v)^T = D S - k ((b.k)^T D S) + k (w.v)^T.
 *
 *   Tied modes (Gated DeltaNet-2 Q&A page, Q3; Gated DeltaNet explainer):
 *     mode 1 (KDA): b_t = w_t = beta_t * 1, channel-wise g_t.
 *     mode 2 (GDN): additionally a scalar decay g_t, i.e.
 *                   S_t = alpha_t (I - beta_t k k^T) S_{t-1} + beta_t k v^T,
 *                   alpha_t = exp(g_t).
 *   Gate-ablation variants (Gated DeltaNet-2 Review §5, "Gate ablation" table), the
 *   same update with one gate a per-token scalar times the all-ones vector:
 *     mode 3 (b-only): channel erase b_t [dk], scalar write w_t.
 *     mode 4 (w-only): scalar erase b_t, channel write w_t [dv].
 *
 * Layouts (row-major): q,k,b [B,H,T,dk]; v,w,o [B,H,T,dv]; g [B,H,T,dk]
 * (mode 2: [B,H,T]); beta (modes 1,2) is passed in b as [B,H,T]; the scalar gate of
 * modes 3 and 4 (w, resp. b) is [B,H,T]; S0, S_T [B,H,dk,dv].  S0 == NULL means a zero
 * initial state; S_T == NULL skips it.
 * Sequence-heads are distributed over `nthreads` POSIX threads.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    const double *q, *k, *v, *g, *b, *w, *S0;
    double *o, *ST;
    int B, H, T, dk, dv, mode;
    int lo, hi; /* [lo, hi) range of sequence-head indices */
} job_t;

/* elements of b and w per token, by mode */
static int b_width(int mode, int dk) { return (mode == 0 || mode == 3) ? dk : 1; }
static int w_width(int mode, int dv) { return (mode == 0 || mode == 4) ? dv : (mode == 3 ? 1 : 0); }

/* One recurrence step on state S (dk x dv); writes o (dv).  b holds b_width values, w
 * w_width values (NULL when 0: the write gate is then beta = b[0]). */
static void step(double *S, const double *q, const double *k, const double *v,
                 const double *g, const double *b, const double *w,
                 int dk, int dv, int mode, double *o, double *r, double *u) {
    /* decay: S <- diag(exp(g)) S */
    for (int i = 0; i < dk; ++i) {
        double a = exp(mode == 2 ? g[0] : g[i]);
        double *row = S + (size_t)i * dv;
        for (int j = 0; j < dv; ++j) row[j] *= a;
    }
    /* r = S^T (b . k) */
    for (int j = 0; j < dv; ++j) r[j] = 0.0;
    for (int i = 0; i < dk; ++i) {
        double bk = (mode == 0 || mode == 3 ? b[i] : b[0]) * k[i];
        const double *row = S + (size_t)i * dv;
        for (int j = 0; j < dv; ++j) r[j] += row[j] * bk;
    }
    /* u = w . v - r */
    for (int j = 0; j < dv; ++j) {
        double wj = (mode == 0 || mode == 4) ? w[j] : (mode == 3 ? w[0] : b[0]);
        u[j] = wj * v[j] - r[j];
    }
    /* S <- S + k u^T */
    for (int i = 0; i < dk; ++i) {
        double *row = S + (size_t)i * dv;
        for (int j = 0; j < dv; ++j) row[j] += k[i] * u[j];
    }
    /* o = S^T q */
    for (int j = 0; j < dv; ++j) o[j] = 0.0;
    for (int i = 0; i < dk; ++i) {
        const double *row = S + (size_t)i * dv;
        for (int j = 0; j < dv; ++j) o[j] += row[j] * q[i];
    }
}

static void *run_fwd(void *arg) {
    job_t *J = (job_t *)arg;
    const int dk = J->dk, dv = J->dv, T = J->T;
    double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    double *r = (double *)malloc(sizeof(double) * dv);
    double *u = (double *)malloc(sizeof(double) * dv);
    const int gw = (J->mode == 2) ? 1 : dk;   /* g elements per token */
    const int bw = b_width(J->mode, dk), ww = w_width(J->mode, dv);
    for (int bh = J->lo; bh < J->hi; ++bh) {
        if (J->S0) memcpy(S, J->S0 + (size_t)bh * dk * dv, sizeof(double) * (size_t)dk * dv);
        else memset(S, 0, sizeof(double) * (size_t)dk * dv);
        for (int t = 0; t < T; ++t) {
            size_t tok = (size_t)bh * T + t;
            step(S, J->q + tok * dk, J->k + tok * dk, J->v + tok * dv, J->g + tok * gw,
                 J->b + tok * bw, ww ? J->w + tok * ww : NULL, dk, dv, J->mode,
                 J->o + tok * dv, r, u);
        }
        if (J->ST) memcpy(J->ST + (size_t)bh * dk * dv, S, sizeof(double) * (size_t)dk * dv);
    }
    free(S); free(r); free(u);
    return NULL;
}

static int launch(job_t base, int n_units, int nthreads, void *(*fn)(void *)) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > n_units) nthreads = n_units > 0 ? n_units : 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
    job_t *jobs = (job_t *)malloc(sizeof(job_t) * nthreads);
    int per = n_units / nthreads, rem = n_units % nthreads, lo = 0;
    for (int i = 0; i < nthreads; ++i) {
        jobs[i] = base;
        jobs[i].lo = lo;
        jobs[i].hi = lo + per + (i < rem ? 1 : 0);
        lo = jobs[i].hi;
        pthread_create(&th[i], NULL, fn, &jobs[i]);
    }
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th); free(jobs);
    return 0;
}

/* Full-sequence forward.  Returns 0 on success, -1 on bad arguments. */
int gdr_oracle_fwd(const double *q, const double *k, const double *v, const double *g,
                   const double *b, const double *w, const double *S0, double *o,
                   double *ST, int B, int H, int T, int dk, int dv, int mode, int nthreads) {
    if (!q || !k || !v || !g || !b || !o || B < 0 || H < 0 || T < 0 || dk < 1 || dv < 1)
        return -1;
    if (mode < 0 || mode > 4 || (w_width(mode, dv) && !w)) return -1;
    job_t J = {q, k, v, g, b, w, S0, o, ST, B, H, T, dk, dv, mode, 0, 0};
    if (T == 0) { /* nothing to read out; S_T = S0 */
        if (ST) {
            size_t n = (size_t)B * H * dk * dv;
            if (S0) memcpy(ST, S0, n * sizeof(double)); else memset(ST, 0, n * sizeof(double));
        }
        return 0;
    }
    return launch(J, B * H, nthreads, run_fwd);
}

static void *run_decode(void *arg) {
    job_t *J = (job_t *)arg;
    const int dk = J->dk, dv = J->dv;
    double *r = (double *)malloc(sizeof(double) * dv);
    double *u = (double *)malloc(sizeof(double) * dv);
    const int gw = (J->mode == 2) ? 1 : dk;
    const int bw = b_width(J->mode, dk), ww = w_width(J->mode, dv);
    for (int nh = J->lo; nh < J->hi; ++nh) {
        double *S = J->ST + (size_t)nh * dk * dv;
        step(S, J->q + (size_t)nh * dk, J->k + (size_t)nh * dk, J->v + (size_t)nh * dv,
             J->g + (size_t)nh * gw, J->b + (size_t)nh * bw,
             ww ? J->w + (size_t)nh * ww : NULL, dk, dv, J->mode,
             J->o + (size_t)nh * dv, r, u);
    }
    free(r); free(u);
    return NULL;
}

/* One-token step for N sequences x H heads; S [N,H,dk,dv] updated in place. */
int gdr_oracle_decode(const double *q, const double *k, const double *v, const double *g,
                      const double *b, const double *w, double *S, double *o,
                      int N, int H, int dk, int dv, int mode, int nthreads) {
    if (!q || !k || !v || !g || !b || !S || !o || N < 0 || H < 0 || dk < 1 || dv < 1)
        return -1;
    if (mode < 0 || mode > 4 || (w_width(mode, dv) && !w)) return -1;
    job_t J = {q, k, v, g, b, w, NULL, o, S, N, H, 1, dk, dv, mode, 0, 0};
    return launch(J, N * H, nthreads, run_decode);
}

/* ---------------------------------------------------------------------------------
 * Backward: the gradient of  L = sum_t <o_t, dO_t> + <S_T, dS_T>  with respect to every
 * input, by reverse-mode differentiation of the same sequential recurrence (the
 * gate-aware backward the Gated DeltaNet-2 Review §4-3 and the Q&A page, Q4, call for;
 * the pages give no formulas, so this is the adjoint of the update equation above).
 *
 * Per token, with M = D_t S_{t-1}, r = M^T (b.k), u = w.v - r, S_t = M + k u^T and
 * o_t = S_t^T q_t, walking t = T-1 .. 0 with G the gradient with respect to S_t:
 *     G   += q_t dO_t^T               dq_t = S_t dO_t
 *     uh   = G^T k_t                  dk_t = G u + b.(M rh),  rh = -uh
 *     dw_t = uh . v_t                 dv_t = uh . w_t
 *     Mh   = G + (b.k) rh^T           db_t = k.(M rh)
 *     dg_t = rowsum(Mh . M)           (d exp(g)/dg = exp(g), M = exp(g) S_{t-1})
 *     G   <- D_t Mh                   (the gradient with respect to S_{t-1})
 * and dS0 = G at the end.  The gates are expanded to full vectors for the step; the
 * tied and scalar modes then sum the components that share one parameter (KDA, GDN:
 * dbeta = sum db + sum dw; GDN: dg = sum dg; b-only: domega = sum dw; w-only:
 * dbeta = sum db).  The states S_{t-1} are recomputed from checkpoints every K tokens
 * by the forward step itself (same operations, so the same values).
 * dO and dS_T (NULL = 0) are [B,H,T,dv] and [B,H,dk,dv]; the outputs have the shapes
 * of their inputs (dS0 NULL = not written).
 */
typedef struct {
    job_t f;
    const double *dO, *dST;
    double *dq, *dk, *dv, *dg, *db, *dw, *dS0;
} bjob_t;

enum { CKPT = 32 };

static void *run_bwd(void *arg) {
    bjob_t *J = (bjob_t *)arg;
    const job_t *F = &J->f;
    const int dk = F->dk, dv = F->dv, T = F->T, mode = F->mode;
    const size_t SS = (size_t)dk * dv;
    const int gw = (mode == 2) ? 1 : dk;
    const int bw = b_width(mode, dk), ww = w_width(mode, dv);
    const int nck = (T + CKPT - 1) / CKPT;
    double *ck = (double *)malloc(sizeof(double) * SS * (nck > 0 ? nck : 1)); /* state before token c*K */
    double *blk = (double *)malloc(sizeof(double) * SS * CKPT);  /* states before each token of a block */
    double *S = (double *)malloc(sizeof(double) * SS);
    double *M = (double *)malloc(sizeof(double) * SS);
    double *G = (double *)malloc(sizeof(double) * SS);
    double *Mh = (double *)malloc(sizeof(double) * SS);
    double *r = (double *)malloc(sizeof(double) * dv), *u = (double *)malloc(sizeof(double) * dv);
    double *uh = (double *)malloc(sizeof(double) * dv), *o = (double *)malloc(sizeof(double) * dv);
    double *y = (double *)malloc(sizeof(double) * dk);
    double *bv = (double *)malloc(sizeof(double) * dk), *wv = (double *)malloc(sizeof(double) * dv);
    double *gv = (double *)malloc(sizeof(double) * dk);
    double *dbv = (double *)malloc(sizeof(double) * dk), *dwv = (double *)malloc(sizeof(double) * dv);
    double *dgv = (double *)malloc(sizeof(double) * dk);
    for (int bh = F->lo; bh < F->hi; ++bh) {
        /* forward, keeping checkpoints */
        if (F->S0) memcpy(S, F->S0 + (size_t)bh * SS, sizeof(double) * SS);
        else memset(S, 0, sizeof(double) * SS);
        for (int t = 0; t < T; ++t) {
            size_t tok = (size_t)bh * T + t;
            if (t % CKPT == 0) memcpy(ck + (size_t)(t / CKPT) * SS, S, sizeof(double) * SS);
            step(S, F->q + tok * dk, F->k + tok * dk, F->v + tok * dv, F->g + tok * gw,
                 F->b + tok * bw, ww ? F->w + tok * ww : NULL, dk, dv, mode, o, r, u);
        }
        /* G = dS_T */
        if (J->dST) memcpy(G, J->dST + (size_t)bh * SS, sizeof(double) * SS);
        else memset(G, 0, sizeof(double) * SS);
        for (int c = nck - 1; c >= 0; --c) {
            const int t0 = c * CKPT, t1 = (t0 + CKPT < T) ? t0 + CKPT : T;
            /* recompute the states before each token of the block */
            memcpy(S, ck + (size_t)c * SS, sizeof(double) * SS);
            for (int t = t0; t < t1; ++t) {
                size_t tok = (size_t)bh * T + t;
                memcpy(blk + (size_t)(t - t0) * SS, S, sizeof(double) * SS);
                step(S, F->q + tok * dk, F->k + tok * dk, F->v + tok * dv, F->g + tok * gw,
                     F->b + tok * bw, ww ? F->w + tok * ww : NULL, dk, dv, mode, o, r, u);
            }
            for (int t = t1 - 1; t >= t0; --t) {
                size_t tok = (size_t)bh * T + t;
                const double *q = F->q + tok * dk, *k = F->k + tok * dk, *v = F->v + tok * dv;
                const double *dO = J->dO + tok * dv;
                /* expanded gates of this token */
                for (int i = 0; i < dk; ++i) {
                    gv[i] = (mode == 2) ? F->g[tok] : F->g[tok * dk + i];
                    bv[i] = (bw == dk) ? F->b[tok * dk + i] : F->b[tok];
                }
                for (int j = 0; j < dv; ++j)
                    wv[j] = (ww == dv) ? F->w[tok * dv + j] : (ww == 1 ? F->w[tok] : F->b[tok]);
                /* recompute M, r, u and S_t from S_{t-1} */
                const double *Sp = blk + (size_t)(t - t0) * SS;
                for (int i = 0; i < dk; ++i) {
                    const double e = exp(gv[i]);
                    for (int j = 0; j < dv; ++j) M[(size_t)i * dv + j] = e * Sp[(size_t)i * dv + j];
                }
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i) acc += M[(size_t)i * dv + j] * bv[i] * k[i];
                    r[j] = acc;
                    u[j] = wv[j] * v[j] - r[j];
                }
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] = M[(size_t)i * dv + j] + k[i] * u[j];
                /* G += q dO^T;  dq = S_t dO */
                for (int i = 0; i < dk; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) {
                        G[(size_t)i * dv + j] += q[i] * dO[j];
                        acc += S[(size_t)i * dv + j] * dO[j];
                    }
                    J->dq[tok * dk + i] = acc;
                }
                /* uh = G^T k;  dw, dv */
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i) acc += G[(size_t)i * dv + j] * k[i];
                    uh[j] = acc;
                    dwv[j] = acc * v[j];
                    J->dv[tok * dv + j] = acc * wv[j];
                }
                /* y = M rh = -M uh;  dk = G u + b.y;  db = k.y */
                for (int i = 0; i < dk; ++i) {
                    double my = 0.0, gu = 0.0;
                    for (int j = 0; j < dv; ++j) {
                        my -= M[(size_t)i * dv + j] * uh[j];
                        gu += G[(size_t)i * dv + j] * u[j];
                    }
                    y[i] = my;
                    J->dk[tok * dk + i] = gu + bv[i] * my;
                    dbv[i] = k[i] * my;
                }
                /* Mh = G + (b.k) rh^T;  dg = rowsum(Mh . M);  G <- D Mh */
                for (int i = 0; i < dk; ++i) {
                    const double bk = bv[i] * k[i], e = exp(gv[i]);
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) {
                        const double mh = G[(size_t)i * dv + j] - bk * uh[j];
                        Mh[(size_t)i * dv + j] = mh;
                        acc += mh * M[(size_t)i * dv + j];
                        G[(size_t)i * dv + j] = e * mh;
                    }
                    dgv[i] = acc;
                }
                /* fold the expanded gate gradients into the mode's parameters */
                double sdb = 0.0, sdw = 0.0, sdg = 0.0;
                for (int i = 0; i < dk; ++i) { sdb += dbv[i]; sdg += dgv[i]; }
                for (int j = 0; j < dv; ++j) sdw += dwv[j];
                if (mode == 2) J->dg[tok] = sdg;
                else for (int i = 0; i < dk; ++i) J->dg[tok * dk + i] = dgv[i];
                if (bw == dk) for (int i = 0; i < dk; ++i) J->db[tok * dk + i] = dbv[i];
                else J->db[tok] = (mode == 1 || mode == 2) ? sdb + sdw : sdb;
                if (ww == dv) for (int j = 0; j < dv; ++j) J->dw[tok * dv + j] = dwv[j];
                else if (ww == 1) J->dw[tok] = sdw;
            }
        }
        if (J->dS0) memcpy(J->dS0 + (size_t)bh * SS, G, sizeof(double) * SS);
    }
    free(ck); free(blk); free(S); free(M); free(G); free(Mh); free(r); free(u); free(uh); free(o);
    free(y); free(bv); free(wv); free(gv); free(dbv); free(dwv); free(dgv);
    return NULL;
}

static int launch_bwd(bjob_t base, int n_units, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > n_units) nthreads = n_units > 0 ? n_units : 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
    bjob_t *jobs = (bjob_t *)malloc(sizeof(bjob_t) * nthreads);
    int per = n_units / nthreads, rem = n_units % nthreads, lo = 0;
    for (int i = 0; i < nthreads; ++i) {
        jobs[i] = base;
        jobs[i].f.lo = lo;
        jobs[i].f.hi = lo + per + (i < rem ? 1 : 0);
        lo = jobs[i].f.hi;
        pthread_create(&th[i], NULL, run_bwd, &jobs[i]);
    }
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th); free(jobs);
    return 0;
}

/* Backward of gdr_oracle_fwd.  dw may be NULL only when the mode has no w (KDA, GDN). */
int gdr_oracle_bwd(const double *q, const double *k, const double *v, const double *g,
                   const double *b, const double *w, const double *S0, const double *dO,
                   const double *dST, double *dq, double *dk_, double *dv_, double *dg,
                   double *db, double *dw, double *dS0, int B, int H, int T, int dk, int dv,
                   int mode, int nthreads) {
    if (!q || !k || !v || !g || !b || !dO || !dq || !dk_ || !dv_ || !dg || !db || B < 0 || H < 0 ||
        T < 0 || dk < 1 || dv < 1)
        return -1;
    if (mode < 0 || mode > 4 || (w_width(mode, dv) && (!w || !dw))) return -1;
    bjob_t J;
    job_t f = {q, k, v, g, b, w, S0, NULL, NULL, B, H, T, dk, dv, mode, 0, 0};
    J.f = f;
    J.dO = dO; J.dST = dST;
    J.dq = dq; J.dk = dk_; J.dv = dv_; J.dg = dg; J.db = db; J.dw = dw; J.dS0 = dS0;
    if (T == 0) {
        if (dS0) {
            size_t n = (size_t)B * H * dk * dv;
            if (dST) memcpy(dS0, dST, n * sizeof(double)); else memset(dS0, 0, n * sizeof(double));
        }
        return 0;
    }
    return launch_bwd(J, B * H, nthreads);
}
