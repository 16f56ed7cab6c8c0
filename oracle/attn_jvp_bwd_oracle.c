/*
 * attn_jvp_bwd_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, fp64 CPU oracle for the backward pass of attention + JVP:
 * the gradients of the scalar
 *
 *     L = sum_i <dO_i, O_i> + sum_i <dtO_i, tO_i>
 *
 * with respect to Q, K, V, tQ, tK, tV, where O and tO are the attention
 * output and its JVP as the forward oracle defines them.  rCM trains
 * through its fused attention + JVP kernel (rCM, "Large-scale diffusion
 * distillation via score-regularized continuous-time consistency", §3.2 and
 * App. C, as summarised by the anthology record LIT-783); the pages give the
 * forward only, so this file is the plain definition of the gradient: the
 * chain rule applied to the forward definition's steps in reverse order.
 * Only the test suite may load this code; the CUDA library shares no code
 * with it.
 *
 * Forward steps (one head, query row i, key j, feature k, scale s):
 *   (1) S_ij  = s sum_k Q_ik K_jk
 *   (2) P_ij  = exp(S_ij - m_i) / sum_l exp(S_il - m_i)      (softmax of row i)
 *   (3) dS_ij = s sum_k (tQ_ik K_jk + Q_ik tK_jk)
 *   (4) mu_i  = sum_j P_ij dS_ij
 *   (5) Pd_ij = P_ij (dS_ij - mu_i)                          (tangent of P)
 *   (6) O_i   = sum_j P_ij V_j
 *   (7) tO_i  = sum_j Pd_ij V_j + sum_j P_ij tV_j
 * Reverse (bars are gradients of L):
 *   (7) Pd_bar_ij  = <dtO_i, V_j>;  P_bar_ij += <dtO_i, tV_j>
 *       V_bar_j += Pd_ij dtO_i;     tV_bar_j += P_ij dtO_i
 *   (6) P_bar_ij += <dO_i, V_j>;    V_bar_j += P_ij dO_i
 *   (5) P_bar_ij += Pd_bar_ij (dS_ij - mu_i);   dS_bar_ij = Pd_bar_ij P_ij
 *       mu_bar_i = -sum_j Pd_bar_ij P_ij
 *   (4) P_bar_ij += mu_bar_i dS_ij;  dS_bar_ij += mu_bar_i P_ij
 *   (3) tQ_bar_i += s sum_j dS_bar_ij K_j;   K_bar_j  += s dS_bar_ij tQ_i
 *       Q_bar_i  += s sum_j dS_bar_ij tK_j;  tK_bar_j += s dS_bar_ij Q_i
 *   (2) S_bar_ij = P_ij (P_bar_ij - sum_l P_il P_bar_il)
 *   (1) Q_bar_i += s sum_j S_bar_ij K_j;     K_bar_j  += s S_bar_ij Q_i
 *
 * Layout: contiguous [BH][L][d] for every tensor (batch and head
 * flattened), cotangents dO, dtO laid out like O.  The query-side gradients
 * (dQ, dtQ) are computed for the listed query rows `qrows` (NULL: all), the
 * key-side ones (dK, dV, dtK, dtV) for the listed keys `krows` (NULL: all),
 * each summing over every query row; outputs are [BH][n rows][d].
 *
 * Parity status: no worked values in the pages; pinned by central finite
 * differences of the forward oracle, a library reverse-over-forward
 * derivative, the standard attention backward (dtO = 0) and invariants.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

static double dot(const double *a, const double *b, int64_t d)
{
    double acc = 0.0;
    for (int64_t k = 0; k < d; ++k) acc += a[k] * b[k];
    return acc;
}

/* Returns 0 on success, -1 on bad arguments, -2 on allocation failure. */
int oracle_attn_jvp_bwd_f64(const double *q, const double *k, const double *v,
                            const double *tq, const double *tk, const double *tv,
                            const double *dout, const double *dtout,
                            double *dq, double *dk, double *dv,
                            double *dtq, double *dtk, double *dtv,
                            int64_t BH, int64_t Lq, int64_t Lk, int64_t d, double scale,
                            const int64_t *qrows, int64_t nqr,
                            const int64_t *krows, int64_t nkr)
{
    if (BH < 0 || Lq < 0 || Lk < 1 || d < 1 || nqr < 0 || nkr < 0) return -1;
    if (!q || !k || !v || !tq || !tk || !tv || !dout || !dtout) return -1;
    if (nqr > 0 && (!dq || !dtq)) return -1;
    if (nkr > 0 && (!dk || !dv || !dtk || !dtv)) return -1;
    if (qrows)
        for (int64_t r = 0; r < nqr; ++r)
            if (qrows[r] < 0 || qrows[r] >= Lq) return -1;
    if (krows)
        for (int64_t r = 0; r < nkr; ++r)
            if (krows[r] < 0 || krows[r] >= Lk) return -1;
    if (!qrows && nqr != 0 && nqr != Lq) return -1;
    if (!krows && nkr != 0 && nkr != Lk) return -1;

    /* per-head storage of the four key-side factors for the listed keys */
    const size_t nmat = (size_t)Lq * (size_t)nkr;
    double *SB = NULL, *DSB = NULL, *PM = NULL, *PDM = NULL;
    int64_t *qpos = NULL; /* query row -> output slot, or -1 */
    if (nkr > 0) {
        SB = (double *)malloc(sizeof(double) * (nmat ? nmat : 1));
        DSB = (double *)malloc(sizeof(double) * (nmat ? nmat : 1));
        PM = (double *)malloc(sizeof(double) * (nmat ? nmat : 1));
        PDM = (double *)malloc(sizeof(double) * (nmat ? nmat : 1));
    }
    qpos = (int64_t *)malloc(sizeof(int64_t) * (size_t)(Lq ? Lq : 1));
    if ((nkr > 0 && (!SB || !DSB || !PM || !PDM)) || !qpos) {
        free(SB); free(DSB); free(PM); free(PDM); free(qpos);
        return -2;
    }
    for (int64_t i = 0; i < Lq; ++i) qpos[i] = -1;
    for (int64_t r = 0; r < nqr; ++r) qpos[qrows ? qrows[r] : r] = r;
    int failed = 0;

    for (int64_t h = 0; h < BH && !failed; ++h) {
        const double *Q = q + (size_t)h * Lq * d, *tQ = tq + (size_t)h * Lq * d;
        const double *K = k + (size_t)h * Lk * d, *tK = tk + (size_t)h * Lk * d;
        const double *V = v + (size_t)h * Lk * d, *tV = tv + (size_t)h * Lk * d;
        const double *dO = dout + (size_t)h * Lq * d, *dtO = dtout + (size_t)h * Lq * d;

        /* query rows: every row when key-side gradients are wanted (their sums
         * run over all rows), otherwise the listed rows only */
#pragma omp parallel
        {
            double *S = (double *)malloc(sizeof(double) * (size_t)Lk);
            double *P = (double *)malloc(sizeof(double) * (size_t)Lk);
            double *dS = (double *)malloc(sizeof(double) * (size_t)Lk);
            double *Pbar = (double *)malloc(sizeof(double) * (size_t)Lk);
            double *Pdbar = (double *)malloc(sizeof(double) * (size_t)Lk);
            double *dSbar = (double *)malloc(sizeof(double) * (size_t)Lk);
            double *Sbar = (double *)malloc(sizeof(double) * (size_t)Lk);
            const int have = S && P && dS && Pbar && Pdbar && dSbar && Sbar;
            if (!have) {
#pragma omp atomic write
                failed = 1;
            }
            {
                const int64_t nrows = nkr > 0 ? Lq : nqr;
                /* every thread takes part in the work-shared loop */
#pragma omp for schedule(dynamic, 4)
                for (int64_t r = 0; r < nrows; ++r) {
                    if (!have) continue;
                    const int64_t i = nkr > 0 ? r : (qrows ? qrows[r] : r);
                    const double *Qi = Q + (size_t)i * d, *tQi = tQ + (size_t)i * d;
                    const double *dOi = dO + (size_t)i * d, *dtOi = dtO + (size_t)i * d;
                    /* forward (1)-(5) for row i */
                    double m = -INFINITY;
                    for (int64_t j = 0; j < Lk; ++j) {
                        S[j] = scale * dot(Qi, K + (size_t)j * d, d);
                        if (S[j] > m) m = S[j];
                    }
                    double Z = 0.0;
                    for (int64_t j = 0; j < Lk; ++j) {
                        P[j] = exp(S[j] - m);
                        Z += P[j];
                    }
                    double mu = 0.0;
                    for (int64_t j = 0; j < Lk; ++j) {
                        P[j] /= Z;
                        dS[j] = scale * (dot(tQi, K + (size_t)j * d, d) + dot(Qi, tK + (size_t)j * d, d));
                        mu += P[j] * dS[j];
                    }
                    /* reverse (7), (6), (5), (4) */
                    double mubar = 0.0;
                    for (int64_t j = 0; j < Lk; ++j) {
                        Pdbar[j] = dot(dtOi, V + (size_t)j * d, d);
                        Pbar[j] = dot(dtOi, tV + (size_t)j * d, d) + dot(dOi, V + (size_t)j * d, d);
                        Pbar[j] += Pdbar[j] * (dS[j] - mu);
                        dSbar[j] = Pdbar[j] * P[j];
                        mubar -= Pdbar[j] * P[j];
                    }
                    for (int64_t j = 0; j < Lk; ++j) {
                        Pbar[j] += mubar * dS[j];
                        dSbar[j] += mubar * P[j];
                    }
                    /* reverse (2) */
                    double ps = 0.0;
                    for (int64_t j = 0; j < Lk; ++j) ps += P[j] * Pbar[j];
                    for (int64_t j = 0; j < Lk; ++j) Sbar[j] = P[j] * (Pbar[j] - ps);
                    /* query-side gradients, reverse (3) and (1) */
                    const int64_t slot = qpos[i];
                    if (slot >= 0) {
                        double *dQi = dq + ((size_t)h * nqr + (size_t)slot) * d;
                        double *dtQi = dtq + ((size_t)h * nqr + (size_t)slot) * d;
                        for (int64_t c = 0; c < d; ++c) {
                            double a = 0.0, b = 0.0;
                            for (int64_t j = 0; j < Lk; ++j) {
                                a += Sbar[j] * K[(size_t)j * d + c] + dSbar[j] * tK[(size_t)j * d + c];
                                b += dSbar[j] * K[(size_t)j * d + c];
                            }
                            dQi[c] = scale * a;
                            dtQi[c] = scale * b;
                        }
                    }
                    /* key-side factors of the listed keys */
                    for (int64_t jj = 0; jj < nkr; ++jj) {
                        const int64_t j = krows ? krows[jj] : jj;
                        const size_t at = (size_t)i * nkr + (size_t)jj;
                        SB[at] = Sbar[j];
                        DSB[at] = dSbar[j];
                        PM[at] = P[j];
                        PDM[at] = P[j] * (dS[j] - mu);
                    }
                }
            }
            free(S); free(P); free(dS); free(Pbar); free(Pdbar); free(dSbar); free(Sbar);
        }
        if (failed) break;

        /* key-side gradients: reverse (7), (6), (3), (1), summed over all rows */
#pragma omp parallel for schedule(dynamic, 4)
        for (int64_t jj = 0; jj < nkr; ++jj) {
            double *dKj = dk + ((size_t)h * nkr + (size_t)jj) * d;
            double *dVj = dv + ((size_t)h * nkr + (size_t)jj) * d;
            double *dtKj = dtk + ((size_t)h * nkr + (size_t)jj) * d;
            double *dtVj = dtv + ((size_t)h * nkr + (size_t)jj) * d;
            for (int64_t c = 0; c < d; ++c) dKj[c] = dVj[c] = dtKj[c] = dtVj[c] = 0.0;
            for (int64_t i = 0; i < Lq; ++i) {
                const size_t at = (size_t)i * nkr + (size_t)jj;
                const double sb = SB[at], dsb = DSB[at], pm = PM[at], pdm = PDM[at];
                const double *Qi = Q + (size_t)i * d, *tQi = tQ + (size_t)i * d;
                const double *dOi = dO + (size_t)i * d, *dtOi = dtO + (size_t)i * d;
                for (int64_t c = 0; c < d; ++c) {
                    dKj[c] += scale * (sb * Qi[c] + dsb * tQi[c]);
                    dtKj[c] += scale * dsb * Qi[c];
                    dVj[c] += pm * dOi[c] + pdm * dtOi[c];
                    dtVj[c] += pm * dtOi[c];
                }
            }
        }
    }
    free(SB); free(DSB); free(PM); free(PDM); free(qpos);
    return failed ? -2 : 0;
}
