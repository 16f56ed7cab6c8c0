/*
 * attn_jvp_bwd_masked_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, fp64 CPU oracle for the backward pass of attention + JVP with
 * a causal mask and/or variable-length (packed) sequences: the gradients of
 *
 *     L = sum_i <dO_i, O_i> + sum_i <dtO_i, tO_i>
 *
 * with respect to Q, K, V, tQ, tK, tV, where O and tO are the masked
 * attention output and its JVP.  The pages describe the fused
 * FlashAttention-2 + JVP forward for self- and cross-attention (rCM,
 * "Large-scale diffusion distillation via score-regularized continuous-time
 * consistency", §3.2 / App. C, as summarised by the anthology record
 * LIT-783); neither masks nor the backward are described there.  This file
 * is the plain definition: the chain rule through the masked forward's steps
 * in reverse order, with every sum over keys taken over the keys the query
 * row may see.
 *
 * Layout and mask (as for the masked forward oracle): every tensor is
 * [H][T][d] (head-major), sequence b holds query rows cu_q[b] .. cu_q[b+1]-1
 * and key rows cu_k[b] .. cu_k[b+1]-1; Lq_b, Lk_b are their lengths.  For
 * local query row i of sequence b, local key j is visible iff
 *     !causal  or  j <= i + (Lk_b - Lq_b)          (bottom-right aligned)
 * A dense [B][H][L][d] problem with a causal mask is the packed layout with
 * B*H "heads" of one sequence each.
 *
 * Forward steps over the visible keys V(i) of row i (scale s):
 *   (1) S_ij  = s <Q_i, K_j>
 *   (2) P_ij  = exp(S_ij - m_i) / sum_{l in V(i)} exp(S_il - m_i)
 *   (3) dS_ij = s (<tQ_i, K_j> + <Q_i, tK_j>)
 *   (4) mu_i  = sum_j P_ij dS_ij
 *   (5) Pd_ij = P_ij (dS_ij - mu_i)
 *   (6) O_i   = sum_j P_ij V_j
 *   (7) tO_i  = sum_j Pd_ij V_j + sum_j P_ij tV_j
 * A row with no visible key has O_i = tO_i = 0 whatever the inputs, so it
 * contributes nothing to any gradient.  Reverse (bars are gradients of L), j
 * in V(i):
 *   (7) Pd_bar_ij = <dtO_i, V_j>;  P_bar_ij = <dtO_i, tV_j>;
 *       V_bar_j += Pd_ij dtO_i;    tV_bar_j += P_ij dtO_i
 *   (6) P_bar_ij += <dO_i, V_j>;   V_bar_j += P_ij dO_i
 *   (5) P_bar_ij += Pd_bar_ij (dS_ij - mu_i);  dS_bar_ij = Pd_bar_ij P_ij;
 *       mu_bar_i = -sum_j Pd_bar_ij P_ij
 *   (4) P_bar_ij += mu_bar_i dS_ij;  dS_bar_ij += mu_bar_i P_ij
 *   (3) tQ_bar_i += s sum_j dS_bar_ij K_j;  K_bar_j  += s dS_bar_ij tQ_i
 *       Q_bar_i  += s sum_j dS_bar_ij tK_j; tK_bar_j += s dS_bar_ij Q_i
 *   (2) S_bar_ij = P_ij (P_bar_ij - sum_l P_il P_bar_il)
 *   (1) Q_bar_i += s sum_j S_bar_ij K_j;    K_bar_j  += s S_bar_ij Q_i
 *
 * Query-side gradients (dQ, dtQ) are computed for the listed packed query
 * rows `qrows` (NULL: all Tq), key-side ones (dK, dV, dtK, dtV) for the
 * listed packed key rows `krows` (NULL: all Tk), each summing over every
 * query row of its sequence; outputs are [H][n rows][d].  Only the test
 * suite may load this code; the CUDA library shares no code with it.
 *
 * Parity status: no worked values in the pages; pinned by central finite
 * differences of the masked forward oracle, a library reverse-over-forward
 * derivative of a masked softmax attention, the unmasked backward oracle on
 * a single unmasked sequence, per-sequence independence and the empty-row
 * rule.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#ifdef _OPENMP
#include <omp.h>
#endif

static double dot(const double *a, const double *b, int64_t d)
{
    double acc = 0.0;
    for (int64_t c = 0; c < d; ++c) acc += a[c] * b[c];
    return acc;
}

/* the sequence holding packed row r (cu: nseq + 1 non-decreasing starts) */
static int64_t seq_of(const int64_t *cu, int64_t nseq, int64_t r)
{
    int64_t b = 0;
    while (b + 1 < nseq && r >= cu[b + 1]) ++b;
    return b;
}

/* number of visible keys (local 0 .. n-1) of local query row i */
static int64_t visible_keys(int64_t i, int64_t Lq, int64_t Lk, int causal)
{
    if (!causal) return Lk;
    const int64_t last = i + (Lk - Lq); /* largest visible local key */
    if (last < 0) return 0;
    return last + 1 < Lk ? last + 1 : Lk;
}

/* Returns 0 on success, -1 on bad arguments, -2 on allocation failure. */
int oracle_attn_jvp_bwd_masked_f64(const double *q, const double *k, const double *v,
                                   const double *tq, const double *tk, const double *tv,
                                   const double *dout, const double *dtout,
                                   double *dq, double *dk, double *dv,
                                   double *dtq, double *dtk, double *dtv,
                                   int64_t H, int64_t Tq, int64_t Tk, int64_t d, double scale,
                                   const int64_t *cu_q, const int64_t *cu_k, int64_t nseq, int causal,
                                   const int64_t *qrows, int64_t nqr,
                                   const int64_t *krows, int64_t nkr)
{
    if (H < 0 || Tq < 0 || Tk < 0 || d < 1 || nseq < 1 || !cu_q || !cu_k || nqr < 0 || nkr < 0) return -1;
    if (!q || !k || !v || !tq || !tk || !tv || !dout || !dtout) return -1;
    if (nqr > 0 && (!dq || !dtq)) return -1;
    if (nkr > 0 && (!dk || !dv || !dtk || !dtv)) return -1;
    if (cu_q[0] != 0 || cu_k[0] != 0 || cu_q[nseq] != Tq || cu_k[nseq] != Tk) return -1;
    for (int64_t b = 0; b < nseq; ++b)
        if (cu_q[b + 1] < cu_q[b] || cu_k[b + 1] < cu_k[b]) return -1;
    if (qrows)
        for (int64_t r = 0; r < nqr; ++r)
            if (qrows[r] < 0 || qrows[r] >= Tq) return -1;
    if (krows)
        for (int64_t r = 0; r < nkr; ++r)
            if (krows[r] < 0 || krows[r] >= Tk) return -1;
    if (!qrows && nqr != 0 && nqr != Tq) return -1;
    if (!krows && nkr != 0 && nkr != Tk) return -1;

    /* per-head key-side factors of the listed keys, one row per query row
     * (zero where the key is not visible to that row or in another sequence) */
    const size_t nmat = (size_t)Tq * (size_t)nkr;
    double *SB = NULL, *DSB = NULL, *PM = NULL, *PDM = NULL;
    int64_t *qpos = (int64_t *)malloc(sizeof(int64_t) * (size_t)(Tq ? Tq : 1));
    int64_t *kseq = (int64_t *)malloc(sizeof(int64_t) * (size_t)(nkr ? nkr : 1));
    if (nkr > 0) {
        SB = (double *)calloc(nmat ? nmat : 1, sizeof(double));
        DSB = (double *)calloc(nmat ? nmat : 1, sizeof(double));
        PM = (double *)calloc(nmat ? nmat : 1, sizeof(double));
        PDM = (double *)calloc(nmat ? nmat : 1, sizeof(double));
    }
    if ((nkr > 0 && (!SB || !DSB || !PM || !PDM)) || !qpos || !kseq) {
        free(SB); free(DSB); free(PM); free(PDM); free(qpos); free(kseq);
        return -2;
    }
    for (int64_t r = 0; r < Tq; ++r) qpos[r] = -1;
    for (int64_t r = 0; r < nqr; ++r) qpos[qrows ? qrows[r] : r] = r;
    for (int64_t jj = 0; jj < nkr; ++jj) kseq[jj] = seq_of(cu_k, nseq, krows ? krows[jj] : jj);
    int failed = 0;

    for (int64_t h = 0; h < H && !failed; ++h) {
        const double *Q = q + (size_t)h * Tq * d, *tQ = tq + (size_t)h * Tq * d;
        const double *dO = dout + (size_t)h * Tq * d, *dtO = dtout + (size_t)h * Tq * d;

        /* query rows: all of them when key-side gradients are wanted (their sums
         * run over every row of the key's sequence), otherwise the listed ones */
#pragma omp parallel
        {
            const size_t nk = (size_t)(Tk ? Tk : 1);
            double *P = (double *)malloc(sizeof(double) * nk);
            double *dS = (double *)malloc(sizeof(double) * nk);
            double *Pbar = (double *)malloc(sizeof(double) * nk);
            double *Pdbar = (double *)malloc(sizeof(double) * nk);
            double *dSbar = (double *)malloc(sizeof(double) * nk);
            double *Sbar = (double *)malloc(sizeof(double) * nk);
            const int have = P && dS && Pbar && Pdbar && dSbar && Sbar;
            if (!have) {
#pragma omp atomic write
                failed = 1;
            }
            const int64_t nrows = nkr > 0 ? Tq : nqr;
#pragma omp for schedule(dynamic, 4)
            for (int64_t rr = 0; rr < nrows; ++rr) {
                if (!have) continue;
                const int64_t r = nkr > 0 ? rr : (qrows ? qrows[rr] : rr);
                const int64_t b = seq_of(cu_q, nseq, r);
                const int64_t i = r - cu_q[b];
                const int64_t Lq = cu_q[b + 1] - cu_q[b], Lk = cu_k[b + 1] - cu_k[b];
                const int64_t nv = visible_keys(i, Lq, Lk, causal);
                const double *K = k + ((size_t)h * Tk + (size_t)cu_k[b]) * d;
                const double *tK = tk + ((size_t)h * Tk + (size_t)cu_k[b]) * d;
                const double *V = v + ((size_t)h * Tk + (size_t)cu_k[b]) * d;
                const double *tV = tv + ((size_t)h * Tk + (size_t)cu_k[b]) * d;
                const double *Qi = Q + (size_t)r * d, *tQi = tQ + (size_t)r * d;
                const double *dOi = dO + (size_t)r * d, *dtOi = dtO + (size_t)r * d;
                /* forward (1)-(5) over the visible keys */
                double m = -INFINITY;
                for (int64_t j = 0; j < nv; ++j) {
                    P[j] = scale * dot(Qi, K + (size_t)j * d, d); /* S_ij for now */
                    if (P[j] > m) m = P[j];
                }
                double Z = 0.0;
                for (int64_t j = 0; j < nv; ++j) {
                    P[j] = exp(P[j] - m);
                    Z += P[j];
                }
                double mu = 0.0;
                for (int64_t j = 0; j < nv; ++j) {
                    P[j] /= Z;
                    dS[j] = scale * (dot(tQi, K + (size_t)j * d, d) + dot(Qi, tK + (size_t)j * d, d));
                    mu += P[j] * dS[j];
                }
                /* reverse (7), (6), (5), (4) */
                double mubar = 0.0;
                for (int64_t j = 0; j < nv; ++j) {
                    Pdbar[j] = dot(dtOi, V + (size_t)j * d, d);
                    Pbar[j] = dot(dtOi, tV + (size_t)j * d, d) + dot(dOi, V + (size_t)j * d, d);
                    Pbar[j] += Pdbar[j] * (dS[j] - mu);
                    dSbar[j] = Pdbar[j] * P[j];
                    mubar -= Pdbar[j] * P[j];
                }
                for (int64_t j = 0; j < nv; ++j) {
                    Pbar[j] += mubar * dS[j];
                    dSbar[j] += mubar * P[j];
                }
                /* reverse (2) */
                double ps = 0.0;
                for (int64_t j = 0; j < nv; ++j) ps += P[j] * Pbar[j];
                for (int64_t j = 0; j < nv; ++j) Sbar[j] = P[j] * (Pbar[j] - ps);
                /* query-side gradients, reverse (3) and (1) */
                const int64_t slot = qpos[r];
                if (slot >= 0) {
                    double *dQi = dq + ((size_t)h * nqr + (size_t)slot) * d;
                    double *dtQi = dtq + ((size_t)h * nqr + (size_t)slot) * d;
                    for (int64_t c = 0; c < d; ++c) {
                        double a = 0.0, e = 0.0;
                        for (int64_t j = 0; j < nv; ++j) {
                            a += Sbar[j] * K[(size_t)j * d + c] + dSbar[j] * tK[(size_t)j * d + c];
                            e += dSbar[j] * K[(size_t)j * d + c];
                        }
                        dQi[c] = scale * a;
                        dtQi[c] = scale * e;
                    }
                }
                /* key-side factors of the listed keys this row sees */
                for (int64_t jj = 0; jj < nkr; ++jj) {
                    if (kseq[jj] != b) continue;
                    const int64_t j = (krows ? krows[jj] : jj) - cu_k[b];
                    if (j >= nv) continue;
                    const size_t at = (size_t)r * nkr + (size_t)jj;
                    SB[at] = Sbar[j];
                    DSB[at] = dSbar[j];
                    PM[at] = P[j];
                    PDM[at] = P[j] * (dS[j] - mu);
                }
            }
            free(P); free(dS); free(Pbar); free(Pdbar); free(dSbar); free(Sbar);
        }
        if (failed) break;

        /* key-side gradients: reverse (7), (6), (3), (1), summed over the query
         * rows of the key's sequence (the factors of every other row are zero) */
#pragma omp parallel for schedule(dynamic, 4)
        for (int64_t jj = 0; jj < nkr; ++jj) {
            double *dKj = dk + ((size_t)h * nkr + (size_t)jj) * d;
            double *dVj = dv + ((size_t)h * nkr + (size_t)jj) * d;
            double *dtKj = dtk + ((size_t)h * nkr + (size_t)jj) * d;
            double *dtVj = dtv + ((size_t)h * nkr + (size_t)jj) * d;
            for (int64_t c = 0; c < d; ++c) dKj[c] = dVj[c] = dtKj[c] = dtVj[c] = 0.0;
            const int64_t b = kseq[jj];
            for (int64_t r = cu_q[b]; r < cu_q[b + 1]; ++r) {
                const size_t at = (size_t)r * nkr + (size_t)jj;
                const double sb = SB[at], dsb = DSB[at], pm = PM[at], pdm = PDM[at];
                const double *Qi = Q + (size_t)r * d, *tQi = tQ + (size_t)r * d;
                const double *dOi = dO + (size_t)r * d, *dtOi = dtO + (size_t)r * d;
                for (int64_t c = 0; c < d; ++c) {
                    dKj[c] += scale * (sb * Qi[c] + dsb * tQi[c]);
                    dtKj[c] += scale * dsb * Qi[c];
                    dVj[c] += pm * dOi[c] + pdm * dtOi[c];
                    dtVj[c] += pm * dtOi[c];
                }
            }
        }
        /* the next head's factors start from zero again */
        if (nkr > 0 && h + 1 < H)
            for (size_t x = 0; x < nmat; ++x) SB[x] = DSB[x] = PM[x] = PDM[x] = 0.0;
    }
    free(SB); free(DSB); free(PM); free(PDM); free(qpos); free(kseq);
    return failed ? -2 : 0;
}
