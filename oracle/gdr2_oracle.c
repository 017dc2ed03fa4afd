/*
 * gdr2_oracle.c -- plain, slow, fp64 CPU oracle for the Gated Delta Rule-2 sequence mixer.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE. Only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark load this file's library. The CUDA library never links, includes or calls
 * it, and this file includes nothing from the CUDA library.
 *
 * Source of every formula: "Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention"
 * (Hatamizadeh, Choi, Kautz), as restated by the long review page (paper-graph-ui), section
 * "The Gated Delta Rule-2 State Update", Steps 1-5 and Eq. 10:
 *
 *     Sbar_t = Diag(alpha_t) S_{t-1}                (Step 1, channel-wise decay on the key axis)
 *     e_t    = b_t (.) k_t,  r_t = Sbar_t^T e_t     (Step 2, gated read)
 *     z_t    = w_t (.) v_t                          (Step 3, gated write target)
 *     S_t    = Sbar_t + k_t (z_t - r_t)^T           (Step 4, delta-rule edit)
 *     o_t    = S_t^T q_t                            (Step 5, output read of the updated state)
 *
 * with alpha_t = exp(log_alpha_t) (section "Gate Parameterization", Eq. 12: alpha = exp(g)).
 * No query scale and no normalisation happen inside the mixer (Step 5 reads S_t^T q_t as is).
 *
 * The backward pass is the explicit adjoint of the five steps above, taken token by token in
 * reverse (the chain rule on Steps 1-5; the review's Appendix D.6 paragraph names a tokenwise
 * fp64 recurrence as the verification reference for all gradients). Per token, with lam = dL/dS_t
 * carried backwards from the future:
 *     lam   += q_t do_t^T                 dq_t = S_t do_t                  (Step 5)
 *     dd     = lam^T k_t                  dk_t = lam (z_t - r_t)           (Step 4, dd = d(z-r))
 *     dw_t   = dd (.) v_t                 dv_t = dd (.) w_t                (Step 3)
 *     mu     = lam - e_t dd^T             de   = -Sbar_t dd                (Step 2, dr = -dd)
 *     db_t   = de (.) k_t                 dk_t += de (.) b_t
 *     dlog_alpha_t[i] = sum_j mu_ij Sbar_t,ij      lam = Diag(alpha_t) mu  (Step 1)
 * and dS0 = lam after the first token. States S_{t-1} are recomputed from checkpoints kept every
 * ORACLE_CKPT tokens (a memory saving only; it changes no arithmetic).
 *
 * Layouts (row-major, contiguous, all double):
 *   q, k, log_alpha, b : [B, T, H, dk]      v, w, o : [B, T, H, dv]
 *   states             : [B, H, dk, dv]     (row index = key channel, column = value channel)
 * Decode tensors drop the T axis: q, k, log_alpha, b : [B, H, dk]; v, w, o : [B, H, dv].
 *
 * Threads: independent (b, h) chains are spread over POSIX threads (nthreads <= 0 means all
 * online cores). Each chain's arithmetic is the same serial loop whatever the thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORACLE_CKPT 64

typedef struct {
    const double *q, *k, *v, *la, *b, *w, *S0;
    const double *dO, *dST;
    double *o, *ST;
    double *dq, *dk, *dv, *dla, *db, *dw, *dS0;
    int B, T, H, dk_, dv_;
    int next;   /* next chain index, taken with an atomic add */
    int fail;   /* set when a worker could not get memory */
} oracle_job;

static size_t tok_off(const oracle_job *J, int bi, int t, int hi, int d) {
    return (((size_t)bi * J->T + t) * J->H + hi) * (size_t)d;
}

/* One token of Steps 1-5 on state S (in place). sbar receives Diag(alpha) S_{t-1}; r, z are
 * scratch of length dv. o may be NULL. */
static void step_forward(int dk, int dv, double *S, double *sbar, double *r, double *z,
                         const double *q, const double *k, const double *v, const double *la,
                         const double *b, const double *w, double *o) {
    for (int i = 0; i < dk; ++i) {                       /* Step 1 */
        double a = exp(la[i]);
        for (int j = 0; j < dv; ++j) sbar[i * dv + j] = a * S[i * dv + j];
    }
    for (int j = 0; j < dv; ++j) r[j] = 0.0;             /* Step 2 */
    for (int i = 0; i < dk; ++i) {
        double e = b[i] * k[i];
        for (int j = 0; j < dv; ++j) r[j] += sbar[i * dv + j] * e;
    }
    for (int j = 0; j < dv; ++j) z[j] = w[j] * v[j];     /* Step 3 */
    for (int i = 0; i < dk; ++i)                         /* Step 4 */
        for (int j = 0; j < dv; ++j) S[i * dv + j] = sbar[i * dv + j] + k[i] * (z[j] - r[j]);
    if (o) {                                             /* Step 5 */
        for (int j = 0; j < dv; ++j) o[j] = 0.0;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) o[j] += S[i * dv + j] * q[i];
    }
}

static void chain_forward(oracle_job *J, int c) {
    const int bi = c / J->H, hi = c % J->H, dk = J->dk_, dv = J->dv_;
    const size_t ss = (size_t)dk * dv;
    double *S = J->ST + (size_t)c * ss;  /* final state buffer doubles as the running state */
    double *sbar = (double *)malloc(sizeof(double) * (ss + 2 * (size_t)dv));
    if (!sbar) { J->fail = 1; return; }
    double *r = sbar + ss, *z = r + dv;
    if (J->S0) memcpy(S, J->S0 + (size_t)c * ss, sizeof(double) * ss);
    else memset(S, 0, sizeof(double) * ss);
    for (int t = 0; t < J->T; ++t) {
        size_t ok = tok_off(J, bi, t, hi, dk), ov = tok_off(J, bi, t, hi, dv);
        step_forward(dk, dv, S, sbar, r, z, J->q + ok, J->k + ok, J->v + ov, J->la + ok,
                     J->b + ok, J->w + ov, J->o + ov);
    }
    free(sbar);
}

static void chain_backward(oracle_job *J, int c) {
    const int bi = c / J->H, hi = c % J->H, dk = J->dk_, dv = J->dv_, T = J->T;
    const size_t ss = (size_t)dk * dv;
    const int nck = (T + ORACLE_CKPT - 1) / ORACLE_CKPT;
    /* checkpoints: S before token m*ORACLE_CKPT; seg: S_{t-1} for each token of one segment */
    double *ck = (double *)malloc(sizeof(double) * ss * (size_t)nck);
    double *seg = (double *)malloc(sizeof(double) * ss * ORACLE_CKPT);
    double *work = (double *)malloc(sizeof(double) * (4 * ss + 3 * (size_t)dv + 2 * (size_t)dk));
    if (!ck || !seg || !work) { free(ck); free(seg); free(work); J->fail = 1; return; }
    double *S = work, *sbar = S + ss, *lam = sbar + ss, *mu = lam + ss;
    double *r = mu + ss, *z = r + dv, *dd = z + dv, *de = dd + dv, *e = de + dk;

    /* forward sweep keeping checkpoints */
    if (J->S0) memcpy(S, J->S0 + (size_t)c * ss, sizeof(double) * ss);
    else memset(S, 0, sizeof(double) * ss);
    for (int t = 0; t < T; ++t) {
        if (t % ORACLE_CKPT == 0) memcpy(ck + (size_t)(t / ORACLE_CKPT) * ss, S, sizeof(double) * ss);
        size_t ok = tok_off(J, bi, t, hi, dk), ov = tok_off(J, bi, t, hi, dv);
        step_forward(dk, dv, S, sbar, r, z, J->q + ok, J->k + ok, J->v + ov, J->la + ok,
                     J->b + ok, J->w + ov, NULL);
    }

    if (J->dST) memcpy(lam, J->dST + (size_t)c * ss, sizeof(double) * ss);
    else memset(lam, 0, sizeof(double) * ss);

    for (int m = nck - 1; m >= 0; --m) {
        const int t0 = m * ORACLE_CKPT;
        const int t1 = (t0 + ORACLE_CKPT < T) ? t0 + ORACLE_CKPT : T;
        memcpy(S, ck + (size_t)m * ss, sizeof(double) * ss);
        for (int t = t0; t < t1; ++t) {   /* recompute S_{t-1} for the segment */
            memcpy(seg + (size_t)(t - t0) * ss, S, sizeof(double) * ss);
            size_t ok = tok_off(J, bi, t, hi, dk), ov = tok_off(J, bi, t, hi, dv);
            step_forward(dk, dv, S, sbar, r, z, J->q + ok, J->k + ok, J->v + ov, J->la + ok,
                         J->b + ok, J->w + ov, NULL);
        }
        for (int t = t1 - 1; t >= t0; --t) {
            size_t ok = tok_off(J, bi, t, hi, dk), ov = tok_off(J, bi, t, hi, dv);
            const double *q = J->q + ok, *k = J->k + ok, *la = J->la + ok, *b = J->b + ok;
            const double *v = J->v + ov, *w = J->w + ov, *dO = J->dO ? J->dO + ov : NULL;
            /* rebuild this token's forward quantities: S holds S_t after the step below */
            memcpy(S, seg + (size_t)(t - t0) * ss, sizeof(double) * ss);
            step_forward(dk, dv, S, sbar, r, z, q, k, v, la, b, w, NULL);
            for (int i = 0; i < dk; ++i) e[i] = b[i] * k[i];

            /* Step 5 adjoint: o = S_t^T q */
            double *dq = J->dq + ok;
            for (int i = 0; i < dk; ++i) {
                double acc = 0.0;
                if (dO)
                    for (int j = 0; j < dv; ++j) acc += S[i * dv + j] * dO[j];
                dq[i] = acc;
            }
            if (dO)
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) lam[i * dv + j] += q[i] * dO[j];

            /* Step 4 adjoint: S_t = Sbar + k (z - r)^T */
            double *dkk = J->dk + ok;
            for (int i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dv; ++j) acc += lam[i * dv + j] * (z[j] - r[j]);
                dkk[i] = acc;
            }
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += lam[i * dv + j] * k[i];
                dd[j] = acc;
            }
            /* Step 3 adjoint: z = w (.) v */
            double *dwp = J->dw + ov, *dvp = J->dv + ov;
            for (int j = 0; j < dv; ++j) { dwp[j] = dd[j] * v[j]; dvp[j] = dd[j] * w[j]; }
            /* Step 2 adjoint: r = Sbar^T e, dr = -dd */
            for (int i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dv; ++j) {
                    mu[i * dv + j] = lam[i * dv + j] - e[i] * dd[j];
                    acc += sbar[i * dv + j] * dd[j];
                }
                de[i] = -acc;
            }
            double *dbp = J->db + ok;
            for (int i = 0; i < dk; ++i) { dbp[i] = de[i] * k[i]; dkk[i] += de[i] * b[i]; }
            /* Step 1 adjoint: Sbar = Diag(exp(la)) S_{t-1} */
            double *dlap = J->dla + ok;
            for (int i = 0; i < dk; ++i) {
                double a = exp(la[i]), acc = 0.0;
                for (int j = 0; j < dv; ++j) {
                    acc += mu[i * dv + j] * sbar[i * dv + j];
                    lam[i * dv + j] = a * mu[i * dv + j];
                }
                dlap[i] = acc;
            }
        }
    }
    if (J->dS0) memcpy(J->dS0 + (size_t)c * ss, lam, sizeof(double) * ss);
    free(ck); free(seg); free(work);
}

typedef struct { oracle_job *J; int mode; } worker_arg;

static void *worker(void *p) {
    worker_arg *a = (worker_arg *)p;
    oracle_job *J = a->J;
    const int n = J->B * J->H;
    for (;;) {
        int c = __atomic_fetch_add(&J->next, 1, __ATOMIC_RELAXED);
        if (c >= n) break;
        if (a->mode == 0) chain_forward(J, c);
        else chain_backward(J, c);
    }
    return NULL;
}

static int run_chains(oracle_job *J, int mode, int nthreads) {
    const int n = J->B * J->H;
    if (nthreads <= 0) {
        long nc = sysconf(_SC_NPROCESSORS_ONLN);
        nthreads = nc > 0 ? (int)nc : 1;
    }
    if (nthreads > n) nthreads = n;
    if (nthreads < 1) nthreads = 1;
    J->next = 0;
    J->fail = 0;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    worker_arg a = {J, mode};
    if (!th) return -1;
    int started = 0;
    for (int i = 1; i < nthreads; ++i)
        if (pthread_create(&th[started], NULL, worker, &a) == 0) ++started;
    worker(&a);  /* the calling thread takes chains too */
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
    return J->fail ? -2 : 0;
}

/* Forward: o [B,T,H,dv] and final state ST [B,H,dk,dv]. S0 may be NULL (zeros). Returns 0, or a
 * negative value when memory runs out. */
int oracle_gdr2_fwd(const double *q, const double *k, const double *v, const double *log_alpha,
                    const double *b, const double *w, const double *S0, double *o, double *ST,
                    int B, int T, int H, int dk, int dv, int nthreads) {
    oracle_job J;
    memset(&J, 0, sizeof(J));
    J.q = q; J.k = k; J.v = v; J.la = log_alpha; J.b = b; J.w = w; J.S0 = S0;
    J.o = o; J.ST = ST;
    J.B = B; J.T = T; J.H = H; J.dk_ = dk; J.dv_ = dv;
    return run_chains(&J, 0, nthreads);
}

/* Backward: given dO [B,T,H,dv] (NULL = zeros) and dST [B,H,dk,dv] (NULL = zeros), writes dq, dk,
 * dlog_alpha, db [B,T,H,dk], dv, dw [B,T,H,dv] and dS0 [B,H,dk,dv] (dS0 may be NULL). */
int oracle_gdr2_bwd(const double *q, const double *k, const double *v, const double *log_alpha,
                    const double *b, const double *w, const double *S0, const double *dO,
                    const double *dST, double *dq, double *dk_out, double *dv_out,
                    double *dlog_alpha, double *db, double *dw, double *dS0,
                    int B, int T, int H, int dk, int dv, int nthreads) {
    oracle_job J;
    memset(&J, 0, sizeof(J));
    J.q = q; J.k = k; J.v = v; J.la = log_alpha; J.b = b; J.w = w; J.S0 = S0;
    J.dO = dO; J.dST = dST;
    J.dq = dq; J.dk = dk_out; J.dv = dv_out; J.dla = dlog_alpha; J.db = db; J.dw = dw;
    J.dS0 = dS0;
    J.B = B; J.T = T; J.H = H; J.dk_ = dk; J.dv_ = dv;
    return run_chains(&J, 1, nthreads);
}

/* Decode: one token per (b, h); state [B,H,dk,dv] is updated in place, o [B,H,dv]. */
int oracle_gdr2_decode(const double *q, const double *k, const double *v, const double *log_alpha,
                       const double *b, const double *w, double *state, double *o,
                       int B, int H, int dk, int dv) {
    const size_t ss = (size_t)dk * dv;
    double *sbar = (double *)malloc(sizeof(double) * (ss + 2 * (size_t)dv));
    if (!sbar) return -2;
    double *r = sbar + ss, *z = r + dv;
    for (int c = 0; c < B * H; ++c)
        step_forward(dk, dv, state + (size_t)c * ss, sbar, r, z, q + (size_t)c * dk,
                     k + (size_t)c * dk, v + (size_t)c * dv, log_alpha + (size_t)c * dk,
                     b + (size_t)c * dk, w + (size_t)c * dv, o + (size_t)c * dv);
    free(sbar);
    return 0;
}
