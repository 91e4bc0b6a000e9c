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
