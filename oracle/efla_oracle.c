/*
 * efla_oracle.c -- plain, sequential fp64 CPU reference of Exact Flow Linear Attention.
 *
 * TEST INFRASTRUCTURE ONLY.  The tests, the smoke check and the bench's CPU-baseline leg
 * call it; the library's compute path never does.  It shares no code, header or constant
 * with the CUDA path.
 *
 * What it computes (row convention: the state S is d_k x d_v and o_t^T = q_t^T S_t,
 * the transpose of the pages' column form S k, S q; both give the same numbers):
 *
 *   lambda_t = ||k_t||^2
 *   alpha_t  = (1 - exp(-beta_t * lambda_t)) / lambda_t      (alpha_t = beta_t when lambda_t == 0)
 *   S_t      = S_{t-1} - alpha_t * k_t (k_t^T S_{t-1} - v_t^T)
 *   o_t      = S_t^T q_t                                      (output read after the write)
 *
 * Sources (Exact Flow Linear Attention, arXiv 2512.12602, summary page):
 *   - Section 2 (Preliminary): the delta rule is a corrective rank-1 write, a first-order
 *     Euler step of continuous-time memory dynamics;
 *   - Section 3.1: zero-order hold, the input and dynamics matrix constant over the step;
 *   - Section 3.2: the closed-form exact flow keeps the delta rule's rank-1 form with
 *     beta_t replaced by alpha_t;
 *   - Section 3.4 (Discussion): the denominator lambda_t is tied to the key's magnitude;
 *   - Section 6 (Conclusion): the dynamics matrix is A_t = k_t k_t^T;
 *   - App. D: A_t is rank 1 and a scaled projection, A_t^2 = lambda_t A_t;
 *   - App. E: the integrating-factor solution of the constant-matrix linear ODE.
 * From these: with dS/dtau = -A S + k v^T on tau in [0, beta], e^{-tau A} = I - ((1 - e^{-tau
 * lambda}) / lambda) A and the input integral collapses to alpha * k v^T, which gives the
 * update above.  The output convention o_t = S_t q_t (after the update) is the method
 * statement's.
 *
 * Mode EFLA_ORACLE_EULER (alpha_t = beta_t) is the plain delta rule of Section 2; the tests
 * use it for the small-step limit of Section 3.4.
 *
 * efla_oracle_bwd is the reverse-mode derivative of the same recurrence, the pass training
 * needs (Section 4.6 reports training throughput on par with DeltaNet; the pages print no
 * backward formulas, so this is the chain rule written out one step at a time in reverse
 * order, from stored states).  With G = dL/dS_t and r_t = S_{t-1}^T k_t - v_t:
 *   G     += q_t dO_t^T              dq_t = S_t dO_t
 *   g      = G^T k_t                 dalpha_t = -g . r_t
 *   dv_t   = alpha_t g               dk_t = -alpha_t (G r_t + S_{t-1} g) + dalpha_t dalpha/dlambda 2 k_t
 *   dbeta_t = dalpha_t dalpha/dbeta  G <- G - alpha_t k_t g^T   (= dL/dS_{t-1})
 * and dS0 = G at the end.  The gate derivatives, from alpha = (1 - e^{-beta lambda})/lambda:
 *   dalpha/dbeta = e^{-beta lambda},   dalpha/dlambda = (beta e^{-beta lambda} - alpha)/lambda,
 * the latter by its Taylor series in x = beta lambda when x is small (its limit at lambda = 0
 * is -beta^2/2).  Euler mode: dalpha/dbeta = 1, dalpha/dlambda = 0.
 *
 * efla_oracle_fwd_gated is the gated variant (Section 3.4 says the method carries over to
 * gated recurrences as "Gated EFLA"; App. F, the exact-flow form of Gated DeltaNet, survives
 * only as a title, so the formula below is this oracle's own reading).  Each token adds a
 * forget gate, a per-token log-decay g_t (g <= 0 decays), to the same zero-order-hold ODE,
 * held constant over the token's unit interval together with the write rate beta_t:
 *   dS/dtau = g S - beta (k k^T S - k v^T),   tau in [0, 1].
 * Its generator g I - beta k k^T has the eigenvalue g - beta*lambda along k and g on the
 * orthogonal complement, so e^{g I - beta k k^T} = e^g (I - alpha k k^T) with the same alpha
 * as above, and the input integral int_0^1 e^{(1-tau)(g - beta lambda)} d tau * beta k v^T
 * collapses to abar k v^T.  With phi1(x) = (1 - e^{-x}) / x (phi1(0) = 1):
 *   alpha_t = beta_t phi1(beta_t lambda_t),   abar_t = beta_t phi1(beta_t lambda_t - g_t),
 *   S_t = e^{g_t} (S_{t-1} - alpha_t k_t (k_t^T S_{t-1})) + abar_t k_t v_t^T,   o_t = S_t^T q_t.
 * g = 0 gives the exact flow above.  Euler mode here is the gated delta rule (Gated
 * DeltaNet): alpha = abar = beta, i.e. the exact decay followed by one Euler step of the
 * delta-rule write.
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>

#define EFLA_ORACLE_EXACT 0
#define EFLA_ORACLE_EULER 1

/* Gate of Section 3.2 with lambda of Section 3.4.  expm1 keeps it exact to rounding when
 * beta*lambda is tiny; lambda == 0 takes the limit alpha = beta. */
double efla_oracle_alpha(double beta, double lambda)
{
    if (lambda == 0.0)
        return beta;
    return -expm1(-beta * lambda) / lambda;
}

/* One recurrence over T tokens of one (b, h) stream.  S (dk x dv) is updated in place;
 * r is scratch of dv doubles.  o may be NULL. */
static void run_stream(const double *q, const double *k, const double *v, const double *beta,
                       double *S, double *o, double *r, long T, long dk, long dv, int mode)
{
    for (long t = 0; t < T; ++t) {
        const double *kt = k + t * dk;
        const double *qt = q + t * dk;
        const double *vt = v + t * dv;
        double lam = 0.0;
        for (long i = 0; i < dk; ++i)
            lam += kt[i] * kt[i];
        const double a = (mode == EFLA_ORACLE_EULER) ? beta[t] : efla_oracle_alpha(beta[t], lam);
        /* r = S^T k - v : what the memory returns for this key, minus the target value */
        for (long j = 0; j < dv; ++j)
            r[j] = -vt[j];
        for (long i = 0; i < dk; ++i)
            for (long j = 0; j < dv; ++j)
                r[j] += kt[i] * S[i * dv + j];
        /* rank-1 corrective write S -= a k r^T */
        for (long i = 0; i < dk; ++i)
            for (long j = 0; j < dv; ++j)
                S[i * dv + j] -= a * kt[i] * r[j];
        /* read-out after the write: o = S^T q */
        if (o) {
            double *ot = o + t * dv;
            for (long j = 0; j < dv; ++j)
                ot[j] = 0.0;
            for (long i = 0; i < dk; ++i)
                for (long j = 0; j < dv; ++j)
                    ot[j] += qt[i] * S[i * dv + j];
        }
    }
}

/*
 * Forward over [B, H, T] streams.
 *   q, k : [B, H, T, dk]   v : [B, H, T, dv]   beta : [B, H, T]
 *   S0   : [B, H, dk, dv] or NULL (zero state)
 *   o    : [B, H, T, dv] or NULL    S_T : [B, H, dk, dv] or NULL (may alias S0)
 * Streams (b, h) are independent; nthreads > 1 runs them on an OpenMP team.
 * Returns 0, or -1 if scratch could not be allocated.
 */
int efla_oracle_fwd(const double *q, const double *k, const double *v, const double *beta,
                    const double *S0, double *o, double *S_T, long B, long H, long T, long dk,
                    long dv, int mode, int nthreads)
{
    const long BH = B * H;
    int failed = 0;
    if (nthreads < 1)
        nthreads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) reduction(| : failed)
    for (long bh = 0; bh < BH; ++bh) {
        double *S = (double *)malloc((size_t)(dk * dv + dv) * sizeof(double));
        if (!S) {
            failed |= 1;
            continue;
        }
        double *r = S + dk * dv;
        if (S0)
            memcpy(S, S0 + bh * dk * dv, (size_t)(dk * dv) * sizeof(double));
        else
            memset(S, 0, (size_t)(dk * dv) * sizeof(double));
        run_stream(q + bh * T * dk, k + bh * T * dk, v + bh * T * dv, beta + bh * T, S,
                   o ? o + bh * T * dv : NULL, r, T, dk, dv, mode);
        if (S_T)
            memcpy(S_T + bh * dk * dv, S, (size_t)(dk * dv) * sizeof(double));
        free(S);
    }
    return failed ? -1 : 0;
}

/* phi1(x) = (1 - e^{-x}) / x, exact to rounding for small |x| through expm1; phi1(0) = 1. */
static double phi1(double x)
{
    if (x == 0.0)
        return 1.0;
    return -expm1(-x) / x;
}

/* The gated recurrence over T tokens of one stream; g is the per-token log-decay. */
static void run_stream_gated(const double *q, const double *k, const double *v, const double *beta,
                             const double *g, double *S, double *o, double *m, long T, long dk,
                             long dv, int mode)
{
    for (long t = 0; t < T; ++t) {
        const double *key = k + t * dk, *query = q + t * dk, *value = v + t * dv;
        double lambda = 0.0;
        for (long i = 0; i < dk; ++i)
            lambda += key[i] * key[i];
        double a = beta[t], ab = beta[t];
        if (mode != EFLA_ORACLE_EULER) {
            a = efla_oracle_alpha(beta[t], lambda);
            ab = beta[t] * phi1(beta[t] * lambda - g[t]);
        }
        const double dec = exp(g[t]);
        /* m = S^T k : what the memory returns for this key */
        for (long j = 0; j < dv; ++j)
            m[j] = 0.0;
        for (long i = 0; i < dk; ++i)
            for (long j = 0; j < dv; ++j)
                m[j] += S[i * dv + j] * key[i];
        /* S <- e^g (S - a k m^T) + ab k v^T */
        for (long i = 0; i < dk; ++i)
            for (long j = 0; j < dv; ++j)
                S[i * dv + j] = dec * (S[i * dv + j] - a * key[i] * m[j]) + ab * key[i] * value[j];
        if (o) {
            double *out = o + t * dv;
            for (long j = 0; j < dv; ++j)
                out[j] = 0.0;
            for (long i = 0; i < dk; ++i)
                for (long j = 0; j < dv; ++j)
                    out[j] += S[i * dv + j] * query[i];
        }
    }
}

/* Gated forward: as efla_oracle_fwd, plus g [B, H, T], the per-token log-decay. */
int efla_oracle_fwd_gated(const double *q, const double *k, const double *v, const double *beta,
                          const double *g, const double *S0, double *o, double *S_T, long B, long H,
                          long T, long dk, long dv, int mode, int nthreads)
{
    const long BH = B * H;
    int failed = 0;
    if (nthreads < 1)
        nthreads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) reduction(| : failed)
    for (long bh = 0; bh < BH; ++bh) {
        double *S = (double *)malloc((size_t)(dk * dv + dv) * sizeof(double));
        if (!S) {
            failed |= 1;
            continue;
        }
        double *r = S + dk * dv;
        if (S0 == NULL)
            memset(S, 0, (size_t)(dk * dv) * sizeof(double));
        else
            memcpy(S, S0 + bh * dk * dv, (size_t)(dk * dv) * sizeof(double));
        run_stream_gated(q + bh * T * dk, k + bh * T * dk, v + bh * T * dv, beta + bh * T, g + bh * T, S,
                         o ? o + bh * T * dv : NULL, r, T, dk, dv, mode);
        if (S_T)
            memcpy(S_T + bh * dk * dv, S, (size_t)(dk * dv) * sizeof(double));
        free(S);
    }
    return failed ? -1 : 0;
}

/*
 * One decode step for N*H streams: the recurrence of efla_oracle_fwd with T = 1.
 *   q, k : [N, H, dk]   v : [N, H, dv]   beta : [N, H]   S : [N, H, dk, dv] in/out
 *   o    : [N, H, dv]
 */
int efla_oracle_step(const double *q, const double *k, const double *v, const double *beta,
                     double *S, double *o, long N, long H, long dk, long dv, int mode,
                     int nthreads)
{
    return efla_oracle_fwd(q, k, v, beta, S, o, S, N, H, 1, dk, dv, mode, nthreads);
}

/* One gated decode step (efla_oracle_fwd_gated with T = 1); g is [N, H]. */
int efla_oracle_step_gated(const double *q, const double *k, const double *v, const double *beta,
                           const double *g, double *S, double *o, long N, long H, long dk, long dv,
                           int mode, int nthreads)
{
    return efla_oracle_fwd_gated(q, k, v, beta, g, S, o, S, N, H, 1, dk, dv, mode, nthreads);
}

/* d alpha / d lambda of the exact gate.  For x = beta*lambda < 1e-3 the difference
 * beta e^{-x} - alpha cancels, so the series beta^2 sum_{n>=1} (-1)^n n x^{n-1}/(n+1)! is used
 * (five terms; the next is below 1e-18 relative). */
double efla_oracle_dalpha_dlambda(double beta, double lambda)
{
    const double x = beta * lambda;
    if (fabs(x) < 1e-3)
        return beta * beta * (-0.5 + x / 3.0 - x * x / 8.0 + x * x * x / 30.0 - x * x * x * x / 144.0);
    const double a = -expm1(-x) / lambda;
    return (beta * exp(-x) - a) / lambda;
}

/* Reverse sweep of one stream.  Ss holds S_0 .. S_T ((T + 1) dk dv doubles); G, r, g are
 * scratch.  Gradients are written (not accumulated). */
static void bwd_stream(const double *q, const double *k, const double *v, const double *beta,
                       const double *dO, const double *dST, double *Ss, double *G, double *r,
                       double *g, double *dq, double *dk, double *dv, double *dbeta, double *dS0,
                       long T, long dk_, long dv_, int mode)
{
    const long D = dk_ * dv_;
    /* forward, keeping every state */
    for (long t = 0; t < T; ++t) {
        const double *kx = k + t * dk_, *vx = v + t * dv_;
        const double *Sp = Ss + t * D;
        double *Sn = Ss + (t + 1) * D;
        double l2 = 0.0;
        for (long i = 0; i < dk_; ++i)
            l2 += kx[i] * kx[i];
        const double at = (mode == EFLA_ORACLE_EULER) ? beta[t] : efla_oracle_alpha(beta[t], l2);
        for (long j = 0; j < dv_; ++j)
            r[j] = -vx[j];
        for (long i = 0; i < dk_; ++i)
            for (long j = 0; j < dv_; ++j)
                r[j] += kx[i] * Sp[i * dv_ + j];
        for (long i = 0; i < dk_; ++i)
            for (long j = 0; j < dv_; ++j)
                Sn[i * dv_ + j] = Sp[i * dv_ + j] - at * kx[i] * r[j];
    }
    /* reverse */
    for (long x = 0; x < D; ++x)
        G[x] = dST ? dST[x] : 0.0;
    for (long t = T - 1; t >= 0; --t) {
        const double *qx = q + t * dk_, *kx = k + t * dk_, *vx = v + t * dv_, *dox = dO + t * dv_;
        const double *Sp = Ss + t * D, *Sc = Ss + (t + 1) * D;
        double l2 = 0.0;
        for (long i = 0; i < dk_; ++i)
            l2 += kx[i] * kx[i];
        const double at = (mode == EFLA_ORACLE_EULER) ? beta[t] : efla_oracle_alpha(beta[t], l2);
        /* o_t = S_t^T q_t */
        for (long i = 0; i < dk_; ++i) {
            double acc = 0.0;
            for (long j = 0; j < dv_; ++j) {
                G[i * dv_ + j] += qx[i] * dox[j];
                acc += Sc[i * dv_ + j] * dox[j];
            }
            dq[t * dk_ + i] = acc;
        }
        /* S_t = S_{t-1} - alpha k r^T with r = S_{t-1}^T k - v */
        for (long j = 0; j < dv_; ++j) {
            double rj = -vx[j], gj = 0.0;
            for (long i = 0; i < dk_; ++i) {
                rj += kx[i] * Sp[i * dv_ + j];
                gj += G[i * dv_ + j] * kx[i];
            }
            r[j] = rj;
            g[j] = gj;
        }
        double da = 0.0;
        for (long j = 0; j < dv_; ++j) {
            da -= g[j] * r[j];
            dv[t * dv_ + j] = at * g[j];
        }
        double dadb, dadl;
        if (mode == EFLA_ORACLE_EULER) {
            dadb = 1.0;
            dadl = 0.0;
        } else if (l2 == 0.0) {
            dadb = 1.0;
            dadl = -0.5 * beta[t] * beta[t];
        } else {
            dadb = exp(-beta[t] * l2);
            dadl = efla_oracle_dalpha_dlambda(beta[t], l2);
        }
        for (long i = 0; i < dk_; ++i) {
            double gr = 0.0, sg = 0.0;
            for (long j = 0; j < dv_; ++j) {
                gr += G[i * dv_ + j] * r[j];
                sg += Sp[i * dv_ + j] * g[j];
            }
            dk[t * dk_ + i] = -at * (gr + sg) + da * dadl * 2.0 * kx[i];
        }
        dbeta[t] = da * dadb;
        for (long i = 0; i < dk_; ++i)
            for (long j = 0; j < dv_; ++j)
                G[i * dv_ + j] -= at * kx[i] * g[j];
    }
    if (dS0)
        memcpy(dS0, G, (size_t)D * sizeof(double));
}

/*
 * Backward over [B, H, T] streams: given dO [B, H, T, dv] and dS_T [B, H, dk, dv] (or NULL,
 * zero), writes dq, dk [B, H, T, dk], dv [B, H, T, dv], dbeta [B, H, T] and dS0 [B, H, dk, dv]
 * (dS0 may be NULL).  S0 as in efla_oracle_fwd.  Keeps all T + 1 states of a stream:
 * (T + 1) dk dv doubles per running stream.  Returns 0, or -1 on allocation failure.
 */
int efla_oracle_bwd(const double *q, const double *k, const double *v, const double *beta,
                    const double *S0, const double *dO, const double *dST, double *dq, double *dk,
                    double *dv, double *dbeta, double *dS0, long B, long H, long T, long dk_,
                    long dv_, int mode, int nthreads)
{
    const long BH = B * H, D = dk_ * dv_;
    int failed = 0;
    if (nthreads < 1)
        nthreads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) reduction(| : failed)
    for (long bh = 0; bh < BH; ++bh) {
        double *Ss = (double *)malloc((size_t)((T + 2) * D + 2 * dv_) * sizeof(double));
        if (!Ss) {
            failed |= 1;
            continue;
        }
        double *G = Ss + (T + 1) * D, *r = G + D, *g = r + dv_;
        if (S0 != NULL)
            memcpy(Ss, S0 + bh * D, (size_t)D * sizeof(double));
        else
            memset(Ss, 0, (size_t)D * sizeof(double));
        bwd_stream(q + bh * T * dk_, k + bh * T * dk_, v + bh * T * dv_, beta + bh * T,
                   dO + bh * T * dv_, dST ? dST + bh * D : NULL, Ss, G, r, g, dq + bh * T * dk_,
                   dk + bh * T * dk_, dv + bh * T * dv_, dbeta + bh * T, dS0 ? dS0 + bh * D : NULL,
                   T, dk_, dv_, mode);
        free(Ss);
    }
    return failed ? -1 : 0;
}
