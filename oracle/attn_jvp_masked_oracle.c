/*
 * attn_jvp_masked_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, fp64 CPU oracle for attention + JVP with a causal mask and/or
 * variable-length (packed) sequences.  The pages describe the fused
 * FlashAttention-2 + JVP pass for self- and cross-attention (rCM, "Large-
 * scale diffusion distillation via score-regularized continuous-time
 * consistency", §3.2 / App. C, as summarised by the anthology record
 * LIT-783); masks and packed batches are not described there.  This file is
 * the plain definition with the keys each query may see restricted:
 *
 *   packed layout: every tensor is [H][T][d] (head-major), sequence b holds
 *   rows cu_q[b] .. cu_q[b+1]-1 of the queries and cu_k[b] .. cu_k[b+1]-1 of
 *   the keys; Lq_b, Lk_b are their lengths.  For local query row i of
 *   sequence b, key j (local, j < Lk_b) is visible iff
 *       !causal  or  j <= i + (Lk_b - Lq_b)       (causal, bottom-right aligned)
 *   and over the visible keys V(i):
 *     S_ij  = s <Q_i, K_j>,  m_i = max S_ij,  P_ij = exp(S_ij - m_i) / sum exp(S_il - m_i)
 *     dS_ij = s (<tQ_i, K_j> + <Q_i, tK_j>),  mu_i = sum P_ij dS_ij
 *     O_i   = sum P_ij V_j,  tO_i = sum P_ij (dS_ij - mu_i) V_j + sum P_ij tV_j
 *     lse_i = m_i + ln sum exp(S_ij - m_i)
 *   A row with no visible key gets O_i = tO_i = 0 and lse_i = -infinity.
 *
 * A dense [B][H][L][d] tensor with a causal mask is the packed layout with
 * B*H "heads" of one sequence each.  Only the test suite may load this code;
 * the CUDA library shares no code with it.
 *
 * Parity status: pinned by the unmasked oracle on the visible keys (prefix
 * property, per-sequence independence), a library masked-softmax JVP and the
 * empty-row rule.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Returns 0 on success, -1 on bad arguments, -2 on allocation failure. */
int oracle_attn_jvp_masked_f64(const double *q, const double *k, const double *v,
                               const double *tq, const double *tk, const double *tv,
                               double *o, double *to, double *lse,
                               int64_t H, int64_t Tq, int64_t Tk, int64_t d, double scale,
                               const int64_t *cu_q, const int64_t *cu_k, int64_t nseq, int causal)
{
    if (H < 0 || Tq < 0 || Tk < 0 || d < 1 || nseq < 1 || !cu_q || !cu_k) return -1;
    if (!q || !k || !v || !tq || !tk || !tv || !o || !to || !lse) return -1;
    if (cu_q[0] != 0 || cu_k[0] != 0 || cu_q[nseq] != Tq || cu_k[nseq] != Tk) return -1;
    for (int64_t b = 0; b < nseq; ++b)
        if (cu_q[b + 1] < cu_q[b] || cu_k[b + 1] < cu_k[b]) return -1;
    int failed = 0;

#pragma omp parallel
    {
        double *S = (double *)malloc(sizeof(double) * (size_t)(Tk ? Tk : 1));
        double *dS = (double *)malloc(sizeof(double) * (size_t)(Tk ? Tk : 1));
        const int have = S && dS;
        if (!have) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 8)
        for (int64_t hr = 0; hr < H * Tq; ++hr) {
            if (!have) continue;
            const int64_t h = hr / Tq, r = hr % Tq;
            int64_t b = 0;
            while (r >= cu_q[b + 1]) ++b; /* the sequence holding query row r */
            const int64_t i = r - cu_q[b];
            const int64_t Lq = cu_q[b + 1] - cu_q[b], Lk = cu_k[b + 1] - cu_k[b];
            int64_t nvis = Lk; /* visible keys are local 0 .. nvis-1 */
            if (causal) {
                const int64_t last = i + (Lk - Lq); /* largest visible local key */
                nvis = last + 1 < Lk ? last + 1 : Lk;
                if (nvis < 0) nvis = 0;
            }
            const double *Qi = q + ((size_t)h * Tq + r) * d, *tQi = tq + ((size_t)h * Tq + r) * d;
            const double *K = k + ((size_t)h * Tk + cu_k[b]) * d, *tK = tk + ((size_t)h * Tk + cu_k[b]) * d;
            const double *V = v + ((size_t)h * Tk + cu_k[b]) * d, *tV = tv + ((size_t)h * Tk + cu_k[b]) * d;
            double *Oi = o + ((size_t)h * Tq + r) * d, *tOi = to + ((size_t)h * Tq + r) * d;
            if (nvis == 0) {
                for (int64_t c = 0; c < d; ++c) Oi[c] = tOi[c] = 0.0;
                lse[(size_t)h * Tq + r] = -INFINITY;
                continue;
            }
            double m = -INFINITY;
            for (int64_t j = 0; j < nvis; ++j) {
                double a = 0.0, bb = 0.0;
                for (int64_t c = 0; c < d; ++c) {
                    a += Qi[c] * K[j * d + c];
                    bb += tQi[c] * K[j * d + c] + Qi[c] * tK[j * d + c];
                }
                S[j] = scale * a;
                dS[j] = scale * bb;
                if (S[j] > m) m = S[j];
            }
            double Z = 0.0;
            for (int64_t j = 0; j < nvis; ++j) {
                S[j] = exp(S[j] - m); /* S now holds the unnormalised weights */
                Z += S[j];
            }
            double mu = 0.0;
            for (int64_t j = 0; j < nvis; ++j) mu += (S[j] / Z) * dS[j];
            for (int64_t c = 0; c < d; ++c) {
                double acc_o = 0.0, acc_t = 0.0;
                for (int64_t j = 0; j < nvis; ++j) {
                    const double P = S[j] / Z;
                    acc_o += P * V[j * d + c];
                    acc_t += P * (dS[j] - mu) * V[j * d + c] + P * tV[j * d + c];
                }
                Oi[c] = acc_o;
                tOi[c] = acc_t;
            }
            lse[(size_t)h * Tq + r] = m + log(Z);
        }
        free(S);
        free(dS);
    }
    return failed ? -2 : 0;
}
