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

/* alpha_t for n tokens: k is [n, dk], beta is [n]. */
void efla_oracle_gate(const double *k, const double *beta, double *alpha, long n, long dk,
                      int mode)
{
    for (long t = 0; t < n; ++t) {
        double lam = 0.0;
        for (long i = 0; i < dk; ++i)
            lam += k[t * dk + i] * k[t * dk + i];
        alpha[t] = (mode == EFLA_ORACLE_EULER) ? beta[t] : efla_oracle_alpha(beta[t], lam);
    }
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
