// jvp_f32.cuh -- fused attention + JVP with fp32 I/O and fp32 arithmetic on
// the CUDA cores, for the accuracy-critical fp32 configuration (max-relative
// error ~1e-6 against fp64; tensor-core tf32 has a 10-bit mantissa and would
// not meet a 1e-4 bound reliably).
//
// Same online algorithm as the tensor-core kernel (rCM, anthology record
// LIT-783, §3.2 / App. C: FlashAttention-2 and its JVP in one tiled pass),
// with an exact rescale at every key tile:
//   m' = max(m, max_j s S_ij),  a = exp(m - m')
//   l  = a l + sum_j p_ij,      g = a g + sum_j p_ij s dS'_ij
//   O  = a O + sum_j p_ij V_j,  T = a T + sum_j p_ij s dS'_ij V_j + p_ij tV_j
// then O /= l, mu = g / l, tO = T / l - mu O, lse = m + ln l.
//
// CTA = 16 query rows of one (batch, head), 4 warps x 4 rows; key tiles of
// 32 keys staged in shared memory (rows padded to d + 1 floats so that lane j
// reading key row j is bank-conflict free).  Lane j owns key j for the score
// dot products; lane t owns output columns t, t + 32, ... for the
// accumulation.
#pragma once

#include <cstdint>

namespace ajvp {
namespace f32 {

constexpr int ROWS_PER_WARP = 4;
constexpr int WARPS = 4;
constexpr int BR = ROWS_PER_WARP * WARPS;  // 16
constexpr int BC = 32;
constexpr int DMAX = 256;
constexpr int CPL = DMAX / 32;  // output columns per lane

__host__ __device__ constexpr size_t smem_bytes(int d) {
    return sizeof(float) * ((size_t)4 * BC * (d + 1) + (size_t)2 * BR * d + (size_t)2 * BR * BC);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__global__ void __launch_bounds__(WARPS * 32) attn_jvp_fwd_f32_kernel(
    const float *__restrict__ q, const float *__restrict__ k, const float *__restrict__ v,
    const float *__restrict__ tq, const float *__restrict__ tk, const float *__restrict__ tv,
    float *__restrict__ o, float *__restrict__ to, float *__restrict__ lse, int Lq, int Lk, int d,
    int n_qtiles, float scale) {
    extern __shared__ float sm[];
    const int dp = d + 1;
    float *sK = sm;
    float *sTK = sK + BC * dp;
    float *sV = sTK + BC * dp;
    float *sTV = sV + BC * dp;
    float *sQ = sTV + BC * dp;   // [BR][d]
    float *sTQ = sQ + BR * d;    // [BR][d]
    float *sP = sTQ + BR * d;    // [BR][BC]
    float *sPD = sP + BR * BC;   // [BR][BC]

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int qt = blockIdx.x % n_qtiles;
    const size_t bh = blockIdx.x / n_qtiles;
    const int q0 = qt * BR;
    const float *qh = q + bh * (size_t)Lq * d;
    const float *tqh = tq + bh * (size_t)Lq * d;
    const float *kh = k + bh * (size_t)Lk * d;
    const float *tkh = tk + bh * (size_t)Lk * d;
    const float *vh = v + bh * (size_t)Lk * d;
    const float *tvh = tv + bh * (size_t)Lk * d;

    for (int idx = tid; idx < BR * d; idx += WARPS * 32) {
        const int r = idx / d, c = idx - r * d;
        const int gr = q0 + r;
        sQ[idx] = gr < Lq ? qh[(size_t)gr * d + c] : 0.f;
        sTQ[idx] = gr < Lq ? tqh[(size_t)gr * d + c] : 0.f;
    }

    float m[ROWS_PER_WARP], l[ROWS_PER_WARP], g[ROWS_PER_WARP];
    float O[ROWS_PER_WARP][CPL], T[ROWS_PER_WARP][CPL];
#pragma unroll
    for (int r = 0; r < ROWS_PER_WARP; ++r) {
        m[r] = -INFINITY;
        l[r] = 0.f;
        g[r] = 0.f;
#pragma unroll
        for (int i = 0; i < CPL; ++i) O[r][i] = T[r][i] = 0.f;
    }

    const int nk = (Lk + BC - 1) / BC;
    for (int kt = 0; kt < nk; ++kt) {
        __syncthreads();  // the previous tile's readers are done
        for (int idx = tid; idx < BC * d; idx += WARPS * 32) {
            const int j = idx / d, c = idx - j * d;
            const int gj = kt * BC + j;
            const bool in = gj < Lk;
            const size_t gi = (size_t)gj * d + c;
            sK[j * dp + c] = in ? kh[gi] : 0.f;
            sTK[j * dp + c] = in ? tkh[gi] : 0.f;
            sV[j * dp + c] = in ? vh[gi] : 0.f;
            sTV[j * dp + c] = in ? tvh[gi] : 0.f;
        }
        __syncthreads();
        const bool valid = kt * BC + lane < Lk;
#pragma unroll
        for (int r = 0; r < ROWS_PER_WARP; ++r) {
            const int row = warp * ROWS_PER_WARP + r;
            const float *qr = sQ + row * d;
            const float *tqr = sTQ + row * d;
            const float *kr = sK + lane * dp;
            const float *tkr = sTK + lane * dp;
            float sd = 0.f, dd = 0.f;
            for (int c = 0; c < d; ++c) {
                const float qc = qr[c], kc = kr[c];
                sd = fmaf(qc, kc, sd);
                dd = fmaf(tqr[c], kc, fmaf(qc, tkr[c], dd));
            }
            const float x = valid ? sd * scale : -INFINITY;
            const float ds = dd * scale;
            const float m_new = fmaxf(m[r], warp_max(x));
            const float a = expf(m[r] - m_new);  // 0 on the first tile (m = -inf)
            const float pj = valid ? expf(x - m_new) : 0.f;
            const float t = pj * ds;
            l[r] = fmaf(a, l[r], warp_sum(pj));
            g[r] = fmaf(a, g[r], warp_sum(t));
            m[r] = m_new;
            sP[row * BC + lane] = pj;
            sPD[row * BC + lane] = t;
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                O[r][i] *= a;
                T[r][i] *= a;
            }
        }
        __syncwarp();
#pragma unroll
        for (int r = 0; r < ROWS_PER_WARP; ++r) {
            const int row = warp * ROWS_PER_WARP + r;
            for (int j = 0; j < BC; ++j) {
                const float pj = sP[row * BC + j];
                const float pdj = sPD[row * BC + j];
#pragma unroll
                for (int i = 0; i < CPL; ++i) {
                    const int c = lane + 32 * i;
                    if (c < d) {
                        const float vj = sV[j * dp + c];
                        O[r][i] = fmaf(pj, vj, O[r][i]);
                        T[r][i] = fmaf(pdj, vj, fmaf(pj, sTV[j * dp + c], T[r][i]));
                    }
                }
            }
        }
    }

#pragma unroll
    for (int r = 0; r < ROWS_PER_WARP; ++r) {
        const int gr = q0 + warp * ROWS_PER_WARP + r;
        if (gr >= Lq) continue;
        const float inv = 1.f / l[r];
        const float mu = g[r] * inv;
        float *orow = o + (bh * (size_t)Lq + gr) * d;
        float *trow = to + (bh * (size_t)Lq + gr) * d;
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const int c = lane + 32 * i;
            if (c < d) {
                const float ov = O[r][i] * inv;
                orow[c] = ov;
                trow[c] = fmaf(-mu, ov, T[r][i] * inv);
            }
        }
        if (lse != nullptr && lane == 0) lse[bh * (size_t)Lq + gr] = m[r] + logf(l[r]);
    }
}

}  // namespace f32
}  // namespace ajvp
