/*
 * efla_oracle.c - plain, slow fp64 CPU oracle for the EFLA token mixer.
 *
 * TEST INFRASTRUCTURE ONLY.  The test-suite, the smoke check and the CPU
 * baseline leg of the benchmark load this library; the product path (the
 * CUDA library and its Python binding) never does, and the two share no code.
 *
 * What it follows ("Exact Flow Linear Attention: Exact Solution from
 * Continuous-Time Dynamics", papernotes.org summary of arXiv 2512.12602):
 *   - section 关键设计 1: the delta-rule/Euler update
 *         S_t = (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T
 *     and the ZOH ODE  dS/dt = -A_t S + b_t,  A_t = k_t k_t^T, b_t = k_t v_t^T;
 *   - section 关键设计 2: the exact flow over [0, beta_t]
 *         S_t = e^{-beta_t A_t} S_{t-1} + int_0^beta e^{-(beta-tau)A} b dtau
 *     collapsed by A^n = lambda^{n-1} A (lambda = k^T k) to
 *         S_t = (I - alpha_t k_t k_t^T) S_{t-1} + alpha_t k_t v_t^T,
 *         alpha_t = (1 - e^{-beta_t lambda_t}) / lambda_t;
 *   - section 损失函数 / 训练策略: 1 - e^{-x} evaluated as -expm1(-x), the
 *     denominator lambda clamped from below at 1e-12;
 *   - flowchart of section 整体框架: readout o_t = S_t^T q_t (post-update S_t).
 * The jsqmd.com blog ("EFLA注意力机制：优化挑战与训练策略解析", section 5.3)
 * supplies the RK4 specialisation used as a convergence check.
 *
 * Layouts (all row-major, fp64):
 *   q, k : [B][H][L][dk]      v, o : [B][H][L][dv]      beta : [B][H][L]
 *   S0, SL: [B][H][dk][dv]    (S0 may be NULL = zero state)
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#define EFLA_ORACLE_EPS 1e-12

/* Exact-flow gate (关键设计 2 closed form; numerics per 训练策略):
 * lambda_c = max(lambda, 1e-12), alpha = -expm1(-beta*lambda_c)/lambda_c.
 * euler != 0 selects the DeltaNet/explicit-Euler step size alpha = beta
 * (关键设计 1). */
double efla_oracle_alpha(double beta, double lambda, int euler)
{
    if (euler) return beta;
    double lc = lambda > EFLA_ORACLE_EPS ? lambda : EFLA_ORACLE_EPS;
    return -expm1(-beta * lc) / lc;
}

/* Gate over `rows` keys of length dk: lambda = ||k||^2 (unclamped), alpha as above. */
void efla_oracle_gate(const double *k, const double *beta, long rows, int dk,
                      int euler, double *alpha, double *lambda)
{
    for (long r = 0; r < rows; ++r) {
        const double *kr = k + r * (long)dk;
        double lam = 0.0;
        for (int i = 0; i < dk; ++i) lam += kr[i] * kr[i];
        lambda[r] = lam;
        alpha[r] = efla_oracle_alpha(beta[r], lam, euler);
    }
}

/* One token of the recurrence on a single dk x dv state, in place:
 *   S <- (I - a k k^T) S + a k v^T      (written as S - a k (k^T S) + a k v^T)
 *   o  = S^T q                           (with the updated S)
 * kts is caller scratch of length dv. */
static void one_token(int dk, int dv, const double *q, const double *k,
                      const double *v, double a, double *S, double *o,
                      double *kts)
{
    for (int j = 0; j < dv; ++j) kts[j] = 0.0;
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) kts[j] += k[i] * S[(long)i * dv + j];
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j)
            S[(long)i * dv + j] += -a * k[i] * kts[j] + a * k[i] * v[j];
    if (o) {
        for (int j = 0; j < dv; ++j) o[j] = 0.0;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) o[j] += S[(long)i * dv + j] * q[i];
    }
}

/* Sequential recurrence over L tokens for every (b,h).  This is the oracle
 * proper: o [B,H,L,dv] and the final state SL [B,H,dk,dv]. */
void efla_oracle_recurrence(const double *q, const double *k, const double *v,
                            const double *beta, const double *S0, int B, int H,
                            int L, int dk, int dv, int euler, double *o,
                            double *SL, int nthreads)
{
    long BH = (long)B * H;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads > 0 ? nthreads : 1)
    for (long bh = 0; bh < BH; ++bh) {
        double *S = SL + bh * (long)dk * dv;
        if (S0) memcpy(S, S0 + bh * (long)dk * dv, sizeof(double) * (size_t)dk * dv);
        else memset(S, 0, sizeof(double) * (size_t)dk * dv);
        double *kts = (double *)malloc(sizeof(double) * (size_t)dv);
        for (int t = 0; t < L; ++t) {
            long row = bh * L + t;
            const double *kt = k + row * dk;
            double lam = 0.0;
            for (int i = 0; i < dk; ++i) lam += kt[i] * kt[i];
            double a = efla_oracle_alpha(beta[row], lam, euler);
            one_token(dk, dv, q + row * dk, kt, v + row * dv, a, S,
                      o ? o + row * dv : NULL, kts);
        }
        free(kts);
    }
}

/* Derivatives of the gate alpha(beta, lambda) of efla_oracle_alpha: with
 * x = beta * lambda, d alpha / d beta = e^{-x} and
 *     d alpha / d lambda = (x e^{-x} - (1 - e^{-x})) / lambda^2,
 * summed as its series beta^2 * sum_{n>=2} (-1)^{n+1} (n-1) x^{n-2} / n!
 * for |x| < 1e-3 (the closed form cancels there).  Where the clamp
 * lambda <= 1e-12 is active alpha does not depend on lambda.  Euler: alpha =
 * beta. */
static void alpha_grad(double beta, double lambda, int euler, double *da_db, double *da_dl)
{
    if (euler) { *da_db = 1.0; *da_dl = 0.0; return; }
    if (lambda <= EFLA_ORACLE_EPS) {
        *da_db = exp(-beta * EFLA_ORACLE_EPS);
        *da_dl = 0.0;
        return;
    }
    double x = beta * lambda;
    *da_db = exp(-x);
    if (fabs(x) < 1e-3) {
        double sum = 0.0, xp = 1.0, fact = 2.0;  /* n = 2: x^0 / 2! */
        for (int n = 2; n < 10; ++n) {
            double term = (double)(n - 1) * xp / fact;
            sum += (n % 2 == 1) ? term : -term;  /* (-1)^{n+1} */
            xp *= x;
            fact *= (double)(n + 1);
        }
        *da_dl = beta * beta * sum;
    } else {
        *da_dl = (x * exp(-x) + expm1(-x)) / (lambda * lambda);
    }
}

/* Reverse-mode derivative of the sequential recurrence, for every (b,h),
 * given dO = dL/do [B,H,L,dv] and dSL = dL/dS_L [B,H,dk,dv] (NULL = 0).
 * The forward states S_0..S_L are kept in full.  Backwards over t, with
 * H = dL/dS_t (the readout of step t included, H += q_t do_t^T):
 *   e = v_t - S_{t-1}^T k_t,  g = H^T k_t,
 *   d alpha = g . e,          de = alpha g        (= dv_t)
 *   dq_t = S_t do_t,          dk_t = alpha H e - S_{t-1} de
 *                                    + 2 d alpha (d alpha/d lambda) k_t
 *   dbeta_t = d alpha (d alpha/d beta)
 *   H <- H - k_t de^T         (= (I - alpha k_t k_t^T) H)
 * and dS0 = H at the end.  Outputs: dq, dk [B,H,L,dk], dv [B,H,L,dv],
 * dbeta [B,H,L], dS0 [B,H,dk,dv]. */
void efla_oracle_backward(const double *q, const double *k, const double *v,
                          const double *beta, const double *S0, const double *dO,
                          const double *dSL, int B, int H, int L, int dk, int dv,
                          int euler, double *dq, double *dkk, double *dvv,
                          double *dbeta, double *dS0, int nthreads)
{
    long BH = (long)B * H;
    long SS = (long)dk * dv;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads > 0 ? nthreads : 1)
    for (long bh = 0; bh < BH; ++bh) {
        double *S = (double *)malloc(sizeof(double) * (size_t)(L + 1) * SS);
        double *Hm = (double *)malloc(sizeof(double) * (size_t)SS);
        double *kts = (double *)malloc(sizeof(double) * (size_t)dv);
        double *e = (double *)malloc(sizeof(double) * (size_t)dv);
        double *g = (double *)malloc(sizeof(double) * (size_t)dv);
        double *de = (double *)malloc(sizeof(double) * (size_t)dv);
        if (S0) memcpy(S, S0 + bh * SS, sizeof(double) * (size_t)SS);
        else memset(S, 0, sizeof(double) * (size_t)SS);
        for (int t = 0; t < L; ++t) {
            long row = bh * L + t;
            const double *kt = k + row * dk;
            double lam = 0.0;
            for (int i = 0; i < dk; ++i) lam += kt[i] * kt[i];
            const double at = efla_oracle_alpha(beta[row], lam, euler);
            memcpy(S + (long)(t + 1) * SS, S + (long)t * SS, sizeof(double) * (size_t)SS);
            one_token(dk, dv, q + row * dk, kt, v + row * dv, at, S + (long)(t + 1) * SS, NULL, kts);
        }
        if (dSL) memcpy(Hm, dSL + bh * SS, sizeof(double) * (size_t)SS);
        else memset(Hm, 0, sizeof(double) * (size_t)SS);
        for (int t = L - 1; t >= 0; --t) {
            long row = bh * L + t;
            const double *qt = q + row * dk, *kt = k + row * dk, *vt = v + row * dv, *dot = dO + row * dv;
            const double *Sp = S + (long)t * SS, *Sn = S + (long)(t + 1) * SS;
            double lam = 0.0;
            for (int i = 0; i < dk; ++i) lam += kt[i] * kt[i];
            double a = efla_oracle_alpha(beta[row], lam, euler), da_db, da_dl;
            alpha_grad(beta[row], lam, euler, &da_db, &da_dl);
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) Hm[(long)i * dv + j] += qt[i] * dot[j];
            for (int i = 0; i < dk; ++i) {  /* dq_t = S_t do_t */
                double acc = 0.0;
                for (int j = 0; j < dv; ++j) acc += Sn[(long)i * dv + j] * dot[j];
                dq[row * dk + i] = acc;
            }
            for (int j = 0; j < dv; ++j) {
                double se = 0.0, hg = 0.0;
                for (int i = 0; i < dk; ++i) {
                    se += Sp[(long)i * dv + j] * kt[i];
                    hg += Hm[(long)i * dv + j] * kt[i];
                }
                e[j] = vt[j] - se;
                g[j] = hg;
            }
            double dal = 0.0;
            for (int j = 0; j < dv; ++j) dal += g[j] * e[j];
            for (int j = 0; j < dv; ++j) {
                de[j] = a * g[j];
                dvv[row * dv + j] = de[j];
            }
            for (int i = 0; i < dk; ++i) {
                double he = 0.0, sde = 0.0;
                for (int j = 0; j < dv; ++j) {
                    he += Hm[(long)i * dv + j] * e[j];
                    sde += Sp[(long)i * dv + j] * de[j];
                }
                dkk[row * dk + i] = a * he - sde + 2.0 * dal * da_dl * kt[i];
            }
            dbeta[row] = dal * da_db;
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) Hm[(long)i * dv + j] -= kt[i] * de[j];
        }
        memcpy(dS0 + bh * SS, Hm, sizeof(double) * (size_t)SS);
        free(S); free(Hm); free(kts); free(e); free(g); free(de);
    }
}

/* Chunked (UT-form) evaluation of the same recurrence, in fp64, written
 * independently of the sequential loop above.  It is the scheme the pages
 * cite for training (整体框架: chunks of size C, tensorised products) and is
 * used only to check that chunked algebra against the recurrence.  Per
 * chunk with rows t0..t0+n-1:
 *   A  = strictly-lower(diag(alpha) K K^T)      T = (I + A)^{-1}
 *   W  = T diag(alpha) K       U = T diag(alpha) V
 *   D  = U - W S               O = Q S + lower-incl-diag(Q K^T) D
 *   S <- S + K^T D
 */
void efla_oracle_chunked(const double *q, const double *k, const double *v,
                         const double *beta, const double *S0, int B, int H,
                         int L, int dk, int dv, int C, int euler, double *o,
                         double *SL, int nthreads)
{
    long BH = (long)B * H;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads > 0 ? nthreads : 1)
    for (long bh = 0; bh < BH; ++bh) {
        double *S = SL + bh * (long)dk * dv;
        if (S0) memcpy(S, S0 + bh * (long)dk * dv, sizeof(double) * (size_t)dk * dv);
        else memset(S, 0, sizeof(double) * (size_t)dk * dv);
        double *al = (double *)malloc(sizeof(double) * C);
        double *A = (double *)malloc(sizeof(double) * C * C);
        double *T = (double *)malloc(sizeof(double) * C * C);
        double *W = (double *)malloc(sizeof(double) * (size_t)C * dk);
        double *U = (double *)malloc(sizeof(double) * (size_t)C * dv);
        double *D = (double *)malloc(sizeof(double) * (size_t)C * dv);
        for (int t0 = 0; t0 < L; t0 += C) {
            int n = L - t0 < C ? L - t0 : C;
            const double *Kc = k + (bh * L + t0) * dk;
            const double *Qc = q + (bh * L + t0) * dk;
            const double *Vc = v + (bh * L + t0) * dv;
            for (int r = 0; r < n; ++r) {
                double lam = 0.0;
                for (int i = 0; i < dk; ++i) lam += Kc[r * dk + i] * Kc[r * dk + i];
                al[r] = efla_oracle_alpha(beta[bh * L + t0 + r], lam, euler);
            }
            /* A = strictly lower part of diag(alpha) K K^T */
            for (int r = 0; r < n; ++r)
                for (int c = 0; c < n; ++c) {
                    double g = 0.0;
                    if (c < r)
                        for (int i = 0; i < dk; ++i) g += Kc[r * dk + i] * Kc[c * dk + i];
                    A[r * C + c] = c < r ? al[r] * g : 0.0;
                }
            /* T = (I + A)^{-1}: unit lower triangular, forward substitution
             * on (I + A) T = I, one row at a time. */
            for (int r = 0; r < n; ++r)
                for (int c = 0; c < n; ++c) {
                    double s = (r == c) ? 1.0 : 0.0;
                    for (int m = c; m < r; ++m) s -= A[r * C + m] * T[m * C + c];
                    T[r * C + c] = (c <= r) ? s : 0.0;
                }
            /* W = T diag(alpha) K, U = T diag(alpha) V */
            for (int r = 0; r < n; ++r) {
                for (int i = 0; i < dk; ++i) {
                    double s = 0.0;
                    for (int m = 0; m <= r; ++m) s += T[r * C + m] * al[m] * Kc[m * dk + i];
                    W[r * dk + i] = s;
                }
                for (int j = 0; j < dv; ++j) {
                    double s = 0.0;
                    for (int m = 0; m <= r; ++m) s += T[r * C + m] * al[m] * Vc[m * dv + j];
                    U[r * dv + j] = s;
                }
            }
            /* D = U - W S */
            for (int r = 0; r < n; ++r)
                for (int j = 0; j < dv; ++j) {
                    double s = U[r * dv + j];
                    for (int i = 0; i < dk; ++i) s -= W[r * dk + i] * S[(long)i * dv + j];
                    D[r * dv + j] = s;
                }
            /* O = Q S + tril(Q K^T) D, diagonal included (o_t reads S_t) */
            if (o) {
                double *Oc = o + (bh * L + t0) * dv;
                for (int r = 0; r < n; ++r) {
                    for (int j = 0; j < dv; ++j) {
                        double s = 0.0;
                        for (int i = 0; i < dk; ++i) s += Qc[r * dk + i] * S[(long)i * dv + j];
                        Oc[r * dv + j] = s;
                    }
                    for (int m = 0; m <= r; ++m) {
                        double qk = 0.0;
                        for (int i = 0; i < dk; ++i) qk += Qc[r * dk + i] * Kc[m * dk + i];
                        for (int j = 0; j < dv; ++j) Oc[r * dv + j] += qk * D[m * dv + j];
                    }
                }
            }
            /* S <- S + K^T D */
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) {
                    double s = 0.0;
                    for (int m = 0; m < n; ++m) s += Kc[m * dk + i] * D[m * dv + j];
                    S[(long)i * dv + j] += s;
                }
        }
        free(al); free(A); free(T); free(W); free(U); free(D);
    }
}

/* ---------------------------------------------------------------------
 * Independent machinery for pinning the oracle (no closed form used).
 * ------------------------------------------------------------------- */

static void matmul_ld(int n, int m, int p, const long double *X,
                      const long double *Y, long double *Z)
{
    for (int i = 0; i < n; ++i)
        for (int j = 0; j < p; ++j) {
            long double s = 0.0L;
            for (int r = 0; r < m; ++r) s += X[i * m + r] * Y[r * p + j];
            Z[i * p + j] = s;
        }
}

/* out = e^{t M} for a d x d matrix M, by brute force: scale t M by 2^-s so
 * that its max-row-sum norm is below 0.5, sum the Taylor series until the
 * terms stop changing the sum in long double, then square s times.
 * Nothing here uses the rank-1 structure of M. */
void efla_oracle_expm_taylor(int d, const double *M, double t, double *out)
{
    long double *X = (long double *)malloc(sizeof(long double) * d * d);
    long double *P = (long double *)malloc(sizeof(long double) * d * d);
    long double *R = (long double *)malloc(sizeof(long double) * d * d);
    long double *Z = (long double *)malloc(sizeof(long double) * d * d);
    long double nrm = 0.0L;
    for (int i = 0; i < d; ++i) {
        long double rs = 0.0L;
        for (int j = 0; j < d; ++j) rs += fabsl((long double)t * M[i * d + j]);
        if (rs > nrm) nrm = rs;
    }
    int s = 0;
    while (nrm > 0.5L) { nrm *= 0.5L; ++s; }
    long double scale = ldexpl(1.0L, -s);
    for (int i = 0; i < d * d; ++i) X[i] = (long double)t * M[i] * scale;
    for (int i = 0; i < d * d; ++i) { R[i] = (i % (d + 1) == 0) ? 1.0L : 0.0L; P[i] = R[i]; }
    for (int n = 1; n < 200; ++n) {
        matmul_ld(d, d, d, P, X, Z);
        long double mx = 0.0L;
        for (int i = 0; i < d * d; ++i) { P[i] = Z[i] / n; R[i] += P[i]; if (fabsl(P[i]) > mx) mx = fabsl(P[i]); }
        if (mx < 1e-40L) break;
    }
    for (int q = 0; q < s; ++q) {
        matmul_ld(d, d, d, R, R, Z);
        memcpy(R, Z, sizeof(long double) * d * d);
    }
    for (int i = 0; i < d * d; ++i) out[i] = (double)R[i];
    free(X); free(P); free(R); free(Z);
}

/* out (dk x dv) = int_0^beta e^{-(beta - tau) A} b dtau for A = k k^T and
 * b = k v^T, by composite Gauss-Legendre quadrature (5 nodes per panel,
 * `panels` panels) with the brute-force exponential above at every node.
 * This is the Duhamel term of the exact ZOH flow (关键设计 2). */
void efla_oracle_duhamel(int dk, int dv, const double *k, const double *v,
                         double beta, int panels, double *out)
{
    static const double xg[5] = {-0.9061798459386640, -0.5384693101056831, 0.0,
                                 0.5384693101056831, 0.9061798459386640};
    static const double wg[5] = {0.2369268850561891, 0.4786286704993665,
                                 0.5688888888888889, 0.4786286704993665,
                                 0.2369268850561891};
    double *A = (double *)malloc(sizeof(double) * dk * dk);
    double *E = (double *)malloc(sizeof(double) * dk * dk);
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dk; ++j) A[i * dk + j] = k[i] * k[j];
    for (int i = 0; i < dk * dv; ++i) out[i] = 0.0;
    double h = beta / panels;
    for (int p = 0; p < panels; ++p) {
        double a0 = p * h;
        for (int g = 0; g < 5; ++g) {
            double tau = a0 + 0.5 * h * (xg[g] + 1.0);
            double w = 0.5 * h * wg[g];
            efla_oracle_expm_taylor(dk, A, -(beta - tau), E);
            /* out += w * E b,  b = k v^T  ->  (E k) v^T */
            for (int i = 0; i < dk; ++i) {
                double ek = 0.0;
                for (int m = 0; m < dk; ++m) ek += E[i * dk + m] * k[m];
                for (int j = 0; j < dv; ++j) out[i * dv + j] += w * ek * v[j];
            }
        }
    }
    free(A); free(E);
}

/* RK4 specialisation of the ODE step (jsqmd.com blog, section 5.3):
 *   S_t = (I - bA + b^2A^2/2 - b^3A^3/6 + b^4A^4/24) S
 *       + (b I - b^2 A/2 + b^3 A^2/6 - b^4 A^3/24) k v^T
 * evaluated with explicit matrix powers of A = k k^T (no rank-1 shortcut). */
void efla_oracle_rk4_step(int dk, int dv, const double *k, const double *v,
                          double b, const double *S, double *Snew)
{
    int d = dk;
    long double *A = (long double *)malloc(sizeof(long double) * d * d);
    long double *A2 = (long double *)malloc(sizeof(long double) * d * d);
    long double *A3 = (long double *)malloc(sizeof(long double) * d * d);
    long double *A4 = (long double *)malloc(sizeof(long double) * d * d);
    long double *M = (long double *)malloc(sizeof(long double) * d * d);
    long double *N = (long double *)malloc(sizeof(long double) * d * d);
    for (int i = 0; i < d; ++i)
        for (int j = 0; j < d; ++j) A[i * d + j] = (long double)k[i] * k[j];
    matmul_ld(d, d, d, A, A, A2);
    matmul_ld(d, d, d, A2, A, A3);
    matmul_ld(d, d, d, A3, A, A4);
    long double bl = b;
    for (int i = 0; i < d * d; ++i) {
        long double I = (i % (d + 1) == 0) ? 1.0L : 0.0L;
        M[i] = I - bl * A[i] + bl * bl * A2[i] / 2 - bl * bl * bl * A3[i] / 6 +
               bl * bl * bl * bl * A4[i] / 24;
        N[i] = bl * I - bl * bl * A[i] / 2 + bl * bl * bl * A2[i] / 6 -
               bl * bl * bl * bl * A3[i] / 24;
    }
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) {
            long double s = 0.0L;
            for (int m = 0; m < dk; ++m)
                s += M[i * d + m] * S[m * dv + j] + N[i * d + m] * (long double)k[m] * v[j];
            Snew[i * dv + j] = (double)s;
        }
    free(A); free(A2); free(A3); free(A4); free(M); free(N);
}
