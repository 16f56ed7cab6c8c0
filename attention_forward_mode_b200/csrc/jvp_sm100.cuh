// jvp_sm100.cuh -- fused attention + Jacobian-vector product, bf16 I/O,
// fp32 accumulation, for sm_100a (B200): TMA tile loads through an mbarrier
// pipeline, tcgen05 MMAs accumulating in tensor memory, warp-specialised
// roles.
//
// The method (rCM, anthology record LIT-783, §3.2 / App. C): one tiled pass
// computes the FlashAttention-2 forward and its JVP.  Per query row i and
// key tile j the kernel keeps the online-softmax state
//     m  running reference max of s*S (log2 units, lazily raised)
//     l  = sum_j p_ij                    p_ij = exp2(c*S_ij - m), c = s*log2(e)
//     g  = sum_j p_ij * s*dS'_ij         dS' = tQ K^T + Q tK^T
// and two tensor-memory accumulators
//     O_acc = sum_j p_ij V_j
//     T_acc = sum_j (p_ij * s*dS'_ij) V_j + p_ij tV_j
// so that at the end O = O_acc / l, mu = g / l, tO = T_acc / l - mu * O
// (the centred JVP expression, rearranged with rowsum(P) = 1).  P and dS are
// never written to global memory.
//
// CTA = 128 query rows of one (batch, head); 256 threads:
//   warp 0      TMA producer (one lane): Q, tQ once; K|tK and V|tV tiles
//               through two 2-stage rings.
//   warp 1      MMA issuer (one lane), per 64-key tile j:
//                 [S_j | dS'_j]  = Q  [K_j | tK_j]^T      (N = 128)
//                        dS'_j  += tQ K_j^T               (N = 64)
//                 [O | T]       += P_j  [V_j | tV_j]      (N = 256, A in TMEM)
//                        T      += PdS_j V_j              (N = 128, A in TMEM)
//   warp 2      tensor-memory allocation / release.
//   warps 4-7   softmax + JVP statistics (one thread per query row, rows are
//               TMEM lanes), lazy rescale of O and T, epilogue.
//
// Tensor memory (512 columns x 128 lanes of fp32):
//   [0,128) O_acc   [128,256) T_acc   [256,384) S/dS' buffer 0
//   [384,512) S/dS' buffer 1    (S at +0, dS' at +64 inside a buffer)
// bf16 P_j is written over S_j's first 32 columns and bf16 (P.*s dS')_j over
// dS'_j's first 32 columns; they are the A operands of the second MMA pair.
#pragma once

#include "ptx_sm100.cuh"

namespace ajvp {
namespace sm100 {

constexpr int BR = 128;       // query rows per CTA
constexpr int BC = 64;        // keys per tile
constexpr int HD = 128;       // head dimension
constexpr int NTHREADS = 256;

// shared memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t CHUNK_Q = 128 * 128;            // one 64-column chunk of a 128-row tile (bytes)
constexpr uint32_t CHUNK_K = 64 * 128;             // one 64-column chunk of a 64-row tile
constexpr uint32_t SM_Q = 0;                       // Q  [2 chunks][128 rows][128 B]
constexpr uint32_t SM_TQ = SM_Q + 2 * CHUNK_Q;     // tQ
constexpr uint32_t STAGE_BYTES = 4 * CHUNK_K;      // 32 KB
constexpr uint32_t SM_KT = SM_TQ + 2 * CHUNK_Q;    // K|tK ring, 2 stages
constexpr uint32_t SM_VT = SM_KT + 2 * STAGE_BYTES;  // V|tV ring, 2 stages
constexpr uint32_t SM_BAR = SM_VT + 2 * STAGE_BYTES;
constexpr uint32_t SMEM_BYTES = SM_BAR + 256 + 1024;  // + alignment slack

// barrier slots (8 bytes each) inside SM_BAR
enum : int {
    B_Q_FULL = 0,
    B_KT_FULL = 1,   // +stage
    B_KT_EMPTY = 3,  // +stage
    B_VT_FULL = 5,   // +stage
    B_VT_EMPTY = 7,  // +stage
    B_SD_FULL = 9,   // +buffer
    B_P_FULL = 11,   // +buffer
    B_PV_DONE = 13,   // one phase per P.V pair (rescale waits on the previous tile's)
    B_O_FULL = 14,    // single use: every MMA of the CTA has completed
    B_MMA_DRAIN = 15,
    N_BARS = 16
};
constexpr uint32_t OFF_TMEM_SLOT = 8 * N_BARS;   // u32
constexpr uint32_t OFF_ABORT = OFF_TMEM_SLOT + 4;  // int

constexpr uint32_t TM_O = 0, TM_T = 128, TM_BUF = 256;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units: P entries stay <= 256

struct Params {
    CUtensorMap tm_q, tm_tq, tm_k, tm_tk, tm_v, tm_tv, tm_o, tm_to;
    float *lse;
    int Lq, Lk, n_qtiles;
    float scale;       // s
    float scale_log2;  // s * log2(e)
    unsigned long long bound_ns;
};

__global__ void __launch_bounds__(NTHREADS, 1) attn_jvp_fwd_kernel(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int qt = blockIdx.x % p.n_qtiles;
    const int bh = blockIdx.x / p.n_qtiles;
    const int q0 = qt * BR;
    const int nk = (p.Lk + BC - 1) / BC;
    const uint64_t bound = p.bound_ns;

    const uint32_t bars = base + SM_BAR;
    auto BAR = [&](int i) -> uint32_t { return bars + 8u * (uint32_t)i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + SM_BAR + OFF_TMEM_SLOT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + SM_BAR + OFF_ABORT);

    if (threadIdx.x == 0) {
        mbar_init(BAR(B_Q_FULL), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(BAR(B_KT_FULL + s), 1);
            mbar_init(BAR(B_KT_EMPTY + s), 1);
            mbar_init(BAR(B_VT_FULL + s), 1);
            mbar_init(BAR(B_VT_EMPTY + s), 1);
            mbar_init(BAR(B_SD_FULL + s), 1);
            mbar_init(BAR(B_P_FULL + s), 128);
        }
        mbar_init(BAR(B_PV_DONE), 1);
        mbar_init(BAR(B_O_FULL), 1);
        mbar_init(BAR(B_MMA_DRAIN), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&p.tm_q);
        tma_prefetch_desc(&p.tm_tq);
        tma_prefetch_desc(&p.tm_k);
        tma_prefetch_desc(&p.tm_tk);
        tma_prefetch_desc(&p.tm_v);
        tma_prefetch_desc(&p.tm_tv);
    }
    if (warp == 2) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            bool ok = true;
            int kt_last[2] = {-1, -1}, vt_last[2] = {-1, -1};
            mbar_arrive_expect_tx(BAR(B_Q_FULL), 4 * CHUNK_Q);
            tma_load_3d(base + SM_Q, &p.tm_q, BAR(B_Q_FULL), 0, q0, bh);
            tma_load_3d(base + SM_Q + CHUNK_Q, &p.tm_q, BAR(B_Q_FULL), 64, q0, bh);
            tma_load_3d(base + SM_TQ, &p.tm_tq, BAR(B_Q_FULL), 0, q0, bh);
            tma_load_3d(base + SM_TQ + CHUNK_Q, &p.tm_tq, BAR(B_Q_FULL), 64, q0, bh);
            // order of use by the MMA warp: KT_0, KT_1, VT_0, KT_2, VT_1, ...
            for (int t = 0; t <= nk && ok; ++t) {
                if (t < nk) {
                    const int s = t & 1;
                    if (!mbar_wait(BAR(B_KT_EMPTY + s), ((t >> 1) & 1) ^ 1, abort_flag, bound)) {
                        ok = false;
                        break;
                    }
                    const uint32_t st = base + SM_KT + s * STAGE_BYTES;
                    const uint32_t fb = BAR(B_KT_FULL + s);
                    const int y = t * BC;
                    mbar_arrive_expect_tx(fb, STAGE_BYTES);
                    // chunk c: K rows then tK rows, so [K | tK] is one N = 128 operand
                    tma_load_3d(st, &p.tm_k, fb, 0, y, bh);
                    tma_load_3d(st + CHUNK_K, &p.tm_tk, fb, 0, y, bh);
                    tma_load_3d(st + 2 * CHUNK_K, &p.tm_k, fb, 64, y, bh);
                    tma_load_3d(st + 3 * CHUNK_K, &p.tm_tk, fb, 64, y, bh);
                    kt_last[s] = t;
                }
                if (t >= 1) {
                    const int i = t - 1;
                    const int s = i & 1;
                    if (!mbar_wait(BAR(B_VT_EMPTY + s), ((i >> 1) & 1) ^ 1, abort_flag, bound)) {
                        ok = false;
                        break;
                    }
                    const uint32_t st = base + SM_VT + s * STAGE_BYTES;
                    const uint32_t fb = BAR(B_VT_FULL + s);
                    const int y = i * BC;
                    mbar_arrive_expect_tx(fb, STAGE_BYTES);
                    // [V c0 | V c1 | tV c0 | tV c1]: N-chunks 64 columns apart (LBO)
                    tma_load_3d(st, &p.tm_v, fb, 0, y, bh);
                    tma_load_3d(st + CHUNK_K, &p.tm_v, fb, 64, y, bh);
                    tma_load_3d(st + 2 * CHUNK_K, &p.tm_tv, fb, 0, y, bh);
                    tma_load_3d(st + 3 * CHUNK_K, &p.tm_tv, fb, 64, y, bh);
                    vt_last[s] = i;
                }
            }
            // let every copy already issued land before shared memory is released
            mbar_wait_drain(BAR(B_Q_FULL), 0, bound);
            for (int s = 0; s < 2; ++s) {
                if (kt_last[s] >= 0) mbar_wait_drain(BAR(B_KT_FULL + s), (kt_last[s] >> 1) & 1, bound);
                if (vt_last[s] >= 0) mbar_wait_drain(BAR(B_VT_FULL + s), (vt_last[s] >> 1) & 1, bound);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // -------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t ID_SD = idesc_bf16_f32(128, 128, 0);  // Q [K|tK]^T
            constexpr uint32_t ID_D = idesc_bf16_f32(128, 64, 0);    // tQ K^T
            constexpr uint32_t ID_OT = idesc_bf16_f32(128, 256, 1);  // P [V|tV]
            constexpr uint32_t ID_T = idesc_bf16_f32(128, 128, 1);   // PdS V
            bool ok = mbar_wait(BAR(B_Q_FULL), 0, abort_flag, bound);
            auto issue_sd = [&](int j) -> bool {
                const int s = j & 1;
                if (!mbar_wait(BAR(B_KT_FULL + s), (j >> 1) & 1, abort_flag, bound)) return false;
                tc_fence_after();
                const uint32_t kst = base + SM_KT + s * STAGE_BYTES;
                const uint32_t t_s = tbase + TM_BUF + 128u * s;
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * 2 * CHUNK_K + (kk & 3) * 32;
                    const uint32_t offq = (kk >> 2) * CHUNK_Q + (kk & 3) * 32;
                    mma_ss(t_s, smem_desc_sw128(base + SM_Q + offq, 16, 1024),
                           smem_desc_sw128(kst + off, 16, 1024), ID_SD, kk > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * 2 * CHUNK_K + (kk & 3) * 32;
                    const uint32_t offq = (kk >> 2) * CHUNK_Q + (kk & 3) * 32;
                    mma_ss(t_s + 64, smem_desc_sw128(base + SM_TQ + offq, 16, 1024),
                           smem_desc_sw128(kst + off, 16, 1024), ID_D, 1u);
                }
                mma_commit(BAR(B_SD_FULL + s));
                mma_commit(BAR(B_KT_EMPTY + s));
                return true;
            };
            auto issue_pv = [&](int i) -> bool {
                const int s = i & 1;
                if (!mbar_wait(BAR(B_P_FULL + s), (i >> 1) & 1, abort_flag, bound)) return false;
                if (!mbar_wait(BAR(B_VT_FULL + s), (i >> 1) & 1, abort_flag, bound)) return false;
                tc_fence_after();
                const uint32_t vst = base + SM_VT + s * STAGE_BYTES;
                const uint32_t t_s = tbase + TM_BUF + 128u * s;
#pragma unroll
                for (int kk = 0; kk < BC / 16; ++kk) {
                    mma_ts(tbase + TM_O, t_s + 8u * kk, smem_desc_sw128(vst + kk * 2048, CHUNK_K, 1024), ID_OT,
                           (i > 0 || kk > 0) ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < BC / 16; ++kk) {
                    mma_ts(tbase + TM_T, t_s + 64 + 8u * kk, smem_desc_sw128(vst + kk * 2048, CHUNK_K, 1024),
                           ID_T, 1u);
                }
                mma_commit(BAR(B_VT_EMPTY + s));
                mma_commit(BAR(B_PV_DONE));
                return true;
            };
            if (ok) ok = issue_sd(0);
            for (int j = 1; j < nk && ok; ++j) {
                ok = issue_sd(j);
                if (ok) ok = issue_pv(j - 1);
            }
            if (ok) ok = issue_pv(nk - 1);
            // O and T are final once everything issued so far completes.  (A parity wait
            // on B_PV_DONE for the last tile would be ambiguous: that barrier may still be
            // two phases behind when the softmax warps finish their last tile.)
            if (ok) mma_commit(BAR(B_O_FULL));
            // every MMA issued must finish before tensor memory is released
            mma_commit(BAR(B_MMA_DRAIN));
            mbar_wait_drain(BAR(B_MMA_DRAIN), 0, bound);
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ---------------------------------------- softmax, JVP statistics, epilogue
        const int wl = warp - 4;
        const int row = wl * 32 + lane;
        const uint32_t lane_off = (uint32_t)(wl * 32) << 16;
        const float c = p.scale_log2;
        const float s_lin = p.scale;
        float m_ref = -INFINITY, l = 0.f, g = 0.f;
        bool ok = true;

        for (int j = 0; j < nk; ++j) {
            const int b = j & 1;
            const uint32_t t_s = tbase + lane_off + TM_BUF + 128u * b;
            ok = mbar_wait(BAR(B_SD_FULL + b), (j >> 1) & 1, abort_flag, bound);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();

            float x[BC];
            {
                uint32_t r0[32], r1[32];
                tmem_ld32(t_s, r0);
                tmem_ld32(t_s + 32, r1);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    x[i] = __uint_as_float(r0[i]);
                    x[i + 32] = __uint_as_float(r1[i]);
                }
            }
            const int valid = p.Lk - j * BC;  // >= 1
            if (valid < BC) {
#pragma unroll
                for (int i = 1; i < BC; ++i)
                    if (i >= valid) x[i] = x[0];  // neutral for the max; p forced to 0 below
            }
            // row max (min for a negative scale) over 8 independent chains
            float m8[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) m8[k] = x[k];
            if (c >= 0.f) {
#pragma unroll
                for (int i = 8; i < BC; ++i) m8[i & 7] = fmaxf(m8[i & 7], x[i]);
#pragma unroll
                for (int k = 0; k < 4; ++k) m8[k] = fmaxf(m8[k], m8[k + 4]);
                m8[0] = fmaxf(fmaxf(m8[0], m8[2]), fmaxf(m8[1], m8[3]));
            } else {
#pragma unroll
                for (int i = 8; i < BC; ++i) m8[i & 7] = fminf(m8[i & 7], x[i]);
#pragma unroll
                for (int k = 0; k < 4; ++k) m8[k] = fminf(m8[k], m8[k + 4]);
                m8[0] = fminf(fminf(m8[0], m8[2]), fminf(m8[1], m8[3]));
            }
            const float mx = m8[0];
            const float m_tile = mx * c;
            if (j == 0) {
                m_ref = m_tile;
            } else {
                const bool need = m_tile > m_ref + RESCALE_THRESHOLD;
                if (__any_sync(0xffffffffu, need)) {
                    float alpha = 1.f;
                    if (need) {
                        alpha = ex2_approx(m_ref - m_tile);
                        m_ref = m_tile;
                    }
                    l *= alpha;
                    g *= alpha;
                    // O and T may only be touched once PV_{j-1} is complete
                    ok = mbar_wait(BAR(B_PV_DONE), (j - 1) & 1, abort_flag, bound);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll 1
                    for (int cc = 0; cc < 8; ++cc) {
                        uint32_t r[32];
                        const uint32_t ta = tbase + lane_off + TM_O + 32u * cc;
                        tmem_ld32(ta, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                        tmem_st32(ta, r);
                    }
                }
            }
            const float neg_m = -m_ref;
#pragma unroll
            for (int i = 0; i < BC; ++i) x[i] = ex2_approx(fmaf(x[i], c, neg_m));
            if (valid < BC) {
#pragma unroll
                for (int i = 1; i < BC; ++i)
                    if (i >= valid) x[i] = 0.f;
            }
            // dS' is loaded while P is packed and stored (different columns)
            uint32_t d0[32], d1[32];
            tmem_ld32(t_s + 64, d0);
            tmem_ld32(t_s + 96, d1);
            float lsum;
            {
                float ls[4] = {0.f, 0.f, 0.f, 0.f};
                uint32_t pk[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    ls[i & 3] += x[2 * i] + x[2 * i + 1];
                    pk[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
                }
                tmem_st32(t_s, pk);  // P over S's first 32 columns
                lsum = (ls[0] + ls[1]) + (ls[2] + ls[3]);
            }
            float gsum;
            {
                tmem_wait_ld();
                float gs[4] = {0.f, 0.f, 0.f, 0.f};
                uint32_t pd[32];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float t0 = x[2 * i] * __uint_as_float(d0[2 * i]) * s_lin;
                    const float t1 = x[2 * i + 1] * __uint_as_float(d0[2 * i + 1]) * s_lin;
                    gs[i & 3] += t0 + t1;
                    pd[i] = pack_bf16x2(t0, t1);
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float t0 = x[32 + 2 * i] * __uint_as_float(d1[2 * i]) * s_lin;
                    const float t1 = x[32 + 2 * i + 1] * __uint_as_float(d1[2 * i + 1]) * s_lin;
                    gs[i & 3] += t0 + t1;
                    pd[16 + i] = pack_bf16x2(t0, t1);
                }
                tmem_st32(t_s + 64, pd);  // P.*s dS' over dS''s first 32 columns
                gsum = (gs[0] + gs[1]) + (gs[2] + gs[3]);
            }
            l += lsum;
            g += gsum;
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(BAR(B_P_FULL + b));
        }

        if (ok) {
            ok = mbar_wait(BAR(B_O_FULL), 0, abort_flag, bound);
            ok = __all_sync(0xffffffffu, ok);
        }
        if (ok) {
            tc_fence_after();
            const float inv_l = 1.f / l;
            const float mu = g * inv_l;
            // stage O into the Q tile's shared memory and tO into tQ's, in the
            // 128-byte-swizzled layout of the store tensor maps
#pragma unroll 1
            for (int pc = 0; pc < 4; ++pc) {
                uint32_t ro[32], rt[32];
                tmem_ld32(tbase + lane_off + TM_O + 32u * pc, ro);
                tmem_ld32(tbase + lane_off + TM_T + 32u * pc, rt);
                tmem_wait_ld();
                uint32_t wo[16], wt[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float o0 = __uint_as_float(ro[2 * i]) * inv_l;
                    const float o1 = __uint_as_float(ro[2 * i + 1]) * inv_l;
                    const float t0 = fmaf(-mu, o0, __uint_as_float(rt[2 * i]) * inv_l);
                    const float t1 = fmaf(-mu, o1, __uint_as_float(rt[2 * i + 1]) * inv_l);
                    wo[i] = pack_bf16x2(o0, o1);
                    wt[i] = pack_bf16x2(t0, t1);
                }
                const uint32_t chunk_off = (uint32_t)(pc >> 1) * CHUNK_Q + (uint32_t)row * 128u;
                const uint32_t unit0 = (uint32_t)(pc & 1) * 4u;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const uint32_t phys = (((unit0 + u) ^ (uint32_t)(row & 7)) * 16u);
                    st_shared_v4(base + SM_Q + chunk_off + phys, wo[4 * u], wo[4 * u + 1], wo[4 * u + 2],
                                 wo[4 * u + 3]);
                    st_shared_v4(base + SM_TQ + chunk_off + phys, wt[4 * u], wt[4 * u + 1], wt[4 * u + 2],
                                 wt[4 * u + 3]);
                }
            }
            if (p.lse != nullptr && q0 + row < p.Lq) {
                p.lse[(size_t)bh * (size_t)p.Lq + (size_t)(q0 + row)] =
                    (m_ref + __log2f(l)) * 0.69314718055994531f;
            }
        }
        fence_proxy_async_smem();
        // all four softmax warps reach this barrier on every path (a warp that
        // gave up skips only the work), so it cannot hang
        named_bar_sync(1, 128);
        if (wl == 0 && lane == 0 && ok && *abort_flag == 0) {
            tma_store_3d(&p.tm_o, base + SM_Q, 0, q0, bh);
            tma_store_3d(&p.tm_o, base + SM_Q + CHUNK_Q, 64, q0, bh);
            tma_store_3d(&p.tm_to, base + SM_TQ, 0, q0, bh);
            tma_store_3d(&p.tm_to, base + SM_TQ + CHUNK_Q, 64, q0, bh);
            tma_store_commit();
            tma_store_wait_all();
        }
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tbase, 512);
    }
}

}  // namespace sm100
}  // namespace ajvp
