/*
 * attn_jvp_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, fp64 CPU oracle for scaled-dot-product attention and its
 * Jacobian-vector product (forward-mode tangent).  Only the test suite, the
 * smoke check and the benchmark's CPU-baseline leg may load this code; the
 * product path (the CUDA library) never calls it and shares no code with it.
 *
 * What it computes (rCM, "Large-scale diffusion distillation via
 * score-regularized continuous-time consistency", §3.2 and App. C as
 * summarised by the anthology record LIT-783: a FlashAttention-2 forward and
 * its JVP computed together, for self- and cross-attention; the formulas are
 * the plain definition of attention and its directional derivative):
 *
 *   for one head, query row i, keys j < Lk, feature k < d, scale s:
 *     S_ij  = s * sum_k Q_ik K_jk
 *     m_i   = max_j S_ij ,   e_ij = exp(S_ij - m_i),   Z_i = sum_j e_ij
 *     P_ij  = e_ij / Z_i                                (two-pass softmax)
 *     dS_ij = s * sum_k (tQ_ik K_jk + Q_ik tK_jk)       (s is a constant)
 *     mu_i  = sum_j P_ij dS_ij
 *     O_i   = sum_j P_ij V_j
 *     tO_i  = sum_j P_ij (dS_ij - mu_i) V_j + sum_j P_ij tV_j
 *     lse_i = m_i + ln Z_i
 *
 * tO is written in its centred form, which is the derivative of O along the
 * tangent (tQ, tK, tV): dP_ij = P_ij (dS_ij - mu_i).
 *
 * Layout: every tensor is contiguous [BH][L][d] (batch and head flattened),
 * tangents laid out like their primals; lse is [BH][Lq].  Rows are
 * independent, so a caller may pass any gathered subset of query rows as a
 * smaller Lq.
 *
 * Parity status: the pages print no worked values; the tests pin this code
 * against closed forms, central finite differences, a library JVP and
 * invariants instead.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Returns 0 on success, -1 on bad arguments, -2 on allocation failure. */
int oracle_attn_jvp_f64(const double *q, const double *k, const double *v,
                        const double *tq, const double *tk, const double *tv,
                        double *o, double *to, double *lse,
                        int64_t BH, int64_t Lq, int64_t Lk, int64_t d,
                        double scale)
{
    if (BH < 0 || Lq < 0 || Lk < 1 || d < 1) return -1;
    if (!q || !k || !v || !tq || !tk || !tv || !o || !to) return -1;
    int failed = 0;

#pragma omp parallel
    {
        /* per-thread scratch: S, dS and P for one row */
        double *S = (double *)malloc(sizeof(double) * (size_t)Lk);
        double *dS = (double *)malloc(sizeof(double) * (size_t)Lk);
        double *P = (double *)malloc(sizeof(double) * (size_t)Lk);
        if (!S || !dS || !P) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1) collapse(2)
        for (int64_t h = 0; h < BH; ++h) {
            for (int64_t i = 0; i < Lq; ++i) {
                if (failed) continue;
                const double *qi = q + (h * Lq + i) * d;
                const double *tqi = tq + (h * Lq + i) * d;
                const double *K = k + h * Lk * d;
                const double *tK = tk + h * Lk * d;
                const double *V = v + h * Lk * d;
                const double *tV = tv + h * Lk * d;
                double *oi = o + (h * Lq + i) * d;
                double *toi = to + (h * Lq + i) * d;

                /* scores and their tangents */
                for (int64_t j = 0; j < Lk; ++j) {
                    double a = 0.0, b = 0.0;
                    for (int64_t c = 0; c < d; ++c) {
                        a += qi[c] * K[j * d + c];
                        b += tqi[c] * K[j * d + c] + qi[c] * tK[j * d + c];
                    }
                    S[j] = scale * a;
                    dS[j] = scale * b;
                }
                /* two-pass softmax */
                double m = S[0];
                for (int64_t j = 1; j < Lk; ++j)
                    if (S[j] > m) m = S[j];
                double Z = 0.0;
                for (int64_t j = 0; j < Lk; ++j) {
                    P[j] = exp(S[j] - m);
                    Z += P[j];
                }
                for (int64_t j = 0; j < Lk; ++j) P[j] /= Z;
                /* mean score tangent under P */
                double mu = 0.0;
                for (int64_t j = 0; j < Lk; ++j) mu += P[j] * dS[j];
                /* outputs */
                for (int64_t c = 0; c < d; ++c) {
                    double acc_o = 0.0, acc_t = 0.0;
                    for (int64_t j = 0; j < Lk; ++j) {
                        acc_o += P[j] * V[j * d + c];
                        acc_t += P[j] * (dS[j] - mu) * V[j * d + c] + P[j] * tV[j * d + c];
                    }
                    oi[c] = acc_o;
                    toi[c] = acc_t;
                }
                if (lse) lse[h * Lq + i] = m + log(Z);
            }
        }
        free(S);
        free(dS);
        free(P);
    }
    return failed ? -2 : 0;
}

/* Number of OpenMP threads a parallel region of this library would use. */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
