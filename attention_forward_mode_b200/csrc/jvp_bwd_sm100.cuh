// jvp_bwd_sm100.cuh -- backward pass of the fused attention + JVP for sm_100a
// (B200): the gradients of L = <dO, O> + <dtO, tO> with respect to Q, K, V
// and the tangents tQ, tK, tV, for bf16 I/O with fp32 accumulation.
//
// rCM (anthology record LIT-783, §3.2 / App. C) trains through its fused
// FlashAttention-2 JVP kernel; the pages describe the forward only.  With
// (one head, query row i, key j, s the softmax scale)
//     S = Q K^T,  P_ij = exp(s S_ij - lse_i),  u = s (tQ K^T + Q tK^T),
//     mu_i = sum_j P_ij u_ij,   A = dtO V^T,   B = dO V^T + dtO tV^T,
//     a_i = <dtO_i, O_i>,       D_i = <dO_i, O_i> + <dtO_i, tO_i> - a_i mu_i,
// the chain rule through the forward gives
//     dS_bar = P .* (A - a)                         (gradient of the score tangent)
//     S_bar  = P .* (B + A .* (u - mu) - a u - D)   (gradient of the scores)
//     dQ  = s (S_bar K + dS_bar tK)       dtQ = s dS_bar K
//     dK  = s (S_bar^T Q + dS_bar^T tQ)   dtK = s dS_bar^T Q
//     dV  = P^T dO + (P .* (u - mu))^T dtO          dtV = P^T dtO
// (a and D use sum_j P_ij A_ij = a_i and rowsum(P .* P_bar) = D_i, so no
// pass over the keys is needed for them).  lse and mu come from the forward
// (attn_jvp_fwd_stats), O and tO are the forward's outputs.
//
// Kernels:
//   bwd_rowstats_kernel   one warp per query row: {lse log2(e), mu, a, D}.
//   attn_jvp_bwd_kernel<ROLE>, one CTA per 128 "row-side" items, streaming
//   64-wide tiles of the other side:
//     ROLE_Q  rows = queries, streams keys     -> dQ, dtQ
//     ROLE_K  rows = keys,    streams queries  -> dK, dtK
//     ROLE_V  rows = keys,    streams queries  -> dV, dtV
//   Every product is computed with the row side as the MMA's M = 128
//   dimension, so each role's result is an accumulation over the streamed
//   side into tensor memory, with no atomics and no transposed stores.
//
// Per streamed tile (64 columns), warp 1 issues
//   G1:  [X | Y] = R0 [C0; C1]^T  (N = 128),  Y += R1 C0^T  (N = 64)
//        [Z | W] = R2 [C2; C3]^T  (N = 128),  W += R3 C2^T  (N = 64)   (not ROLE_V)
//   then, once the elementwise warps have written E1, E2 (bf16, in tensor
//   memory over X and Y),
//   G2:  acc0 += E1 C0' + E2 C1',  acc1 += E? C?'  (A from tensor memory)
// with these operands (R* resident, C* streamed, ' = the same tile read
// MN-major):
//            R0 R1  R2  R3   C0 C1  C2  C3   X   Y   Z  W    E1     E2
//   ROLE_Q   Q  tQ  dtO dO   K  tK  V   tV   S   u'  A  B    S_bar  dS_bar
//   ROLE_K   K  tK  V   tV   Q  tQ  dtO dO   S^T u'^T A^T B^T (transposed)
//   ROLE_V   K  tK  -   -    Q  tQ  dO  dtO  S^T u'^T -  -   P^T    (P.*(u-mu))^T
// (u' = tQ K^T + Q tK^T without the scale).  G2: ROLE_Q/K acc0 += E1 C0 +
// E2 C1, acc1 += E2 C0; ROLE_V acc0 += E1 C2 + E2 C3, acc1 += E1 C3.
//
// Warp roles (384 threads): warp 0 TMA producer, warp 1 MMA issuer, warp 2
// tensor-memory allocation, warps 4-11 elementwise in two groups of four
// warps (group g takes columns 32g .. 32g+31 of each tile; one thread per
// row and group), which also run the epilogue (acc * scale -> bf16 -> TMA
// store).  Tensor memory: acc0 [0,128), acc1 [128,256), X [256,320),
// Y [320,384), Z [384,448), W [448,512).
#pragma once

#include "ptx_sm100.cuh"

namespace ajvp {
namespace bwd {

enum Role : int { ROLE_Q = 0, ROLE_K = 1, ROLE_V = 2 };

constexpr int BM = 128;  // row-side items per CTA
constexpr int BN = 64;   // streamed items per tile
constexpr int HD = 128;  // head dimension
constexpr int NTHREADS = 384;
constexpr int EW_THREADS = 256;
constexpr int LSTAGES = 2;  // ring of the streamed tiles the G2 products read

constexpr uint32_t CHUNK_R = 128 * 128;  // one 64-column chunk of a 128-row tile (bytes)
constexpr uint32_t CHUNK_C = 64 * 128;   // one 64-column chunk of a 64-row tile
constexpr uint32_t R_TILE = 2 * CHUNK_R;
constexpr uint32_t C_STAGE = 4 * CHUNK_C;  // [Cx c0 | Cy c0 | Cx c1 | Cy c1]
constexpr uint32_t C_CHUNK = 2 * CHUNK_C;  // stride between the two 64-column chunks of one tile
constexpr uint32_t STATS_TILE = BN * 16;  // {lse2, mu, a, D} per streamed query
constexpr uint32_t SM_R = 0;              // R0..R3
constexpr uint32_t SM_L = SM_R + 4 * R_TILE;       // "long" ring: the tiles G2 reads
constexpr uint32_t SM_S = SM_L + LSTAGES * C_STAGE;  // "short" stage: tiles only G1 reads
constexpr uint32_t SM_ST = SM_S + C_STAGE;           // stats of the long ring's tiles
constexpr uint32_t SM_BAR = SM_ST + LSTAGES * STATS_TILE;
constexpr uint32_t SMEM_BYTES = SM_BAR + 256;  // the base is 1024-byte aligned (checked)
static_assert(SMEM_BYTES <= 232448, "exceeds the opt-in shared memory of one CTA");

enum : int {
    B_R_FULL = 0,
    B_L_FULL = 1,   // + stage
    B_S_FULL = 3,
    B_G1_DONE = 4,  // X, Y, Z, W of the current tile complete; short stage free
    B_E_DONE = 5,   // E1, E2 written (256 arrivals)
    B_G2_DONE = 6,  // + long stage: the stage's G2 products complete
    B_ACC_FULL = 8,
    B_MMA_DRAIN = 9,
    N_BARS = 10
};
constexpr uint32_t OFF_TMEM_SLOT = 8 * N_BARS;
constexpr uint32_t OFF_ABORT = OFF_TMEM_SLOT + 4;

constexpr uint32_t TM_ACC0 = 0, TM_ACC1 = 128, TM_X = 256, TM_Y = 320, TM_Z = 384, TM_W = 448;
constexpr uint32_t NB_EPI = 1;

struct Params {
    CUtensorMap tm_r[4], tm_c[4], tm_out[2];
    const float4 *stats;  // [B*H][Lq] {lse*log2(e), mu, a, D}, plus BN rows of padding
    int Lrow, Lcol;       // row-side and streamed lengths
    int Lq;               // query rows per (batch, head): the stats row stride
    int n_rtiles;         // 128-row tiles per (batch, head)
    float scale;          // s
    float scale_log2;     // s * log2(e)
    float out_scale;      // s (ROLE_Q, ROLE_K) or 1 (ROLE_V)
    unsigned long long bound_ns;
};

// {lse log2(e), mu, a, D} per query row; one warp per row, 4 features per lane.
__global__ void __launch_bounds__(256) bwd_rowstats_kernel(const __nv_bfloat16 *__restrict__ o,
                                                           const __nv_bfloat16 *__restrict__ to,
                                                           const __nv_bfloat16 *__restrict__ dout,
                                                           const __nv_bfloat16 *__restrict__ dtout,
                                                           const float *__restrict__ lse,
                                                           const float *__restrict__ mu, float4 *__restrict__ stats,
                                                           long long rows) {
    const int lane = threadIdx.x & 31;
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
        const size_t off = (size_t)r * HD + 4 * lane;
        const uint2 uo = *reinterpret_cast<const uint2 *>(o + off);
        const uint2 ut = *reinterpret_cast<const uint2 *>(to + off);
        const uint2 ud = *reinterpret_cast<const uint2 *>(dout + off);
        const uint2 ue = *reinterpret_cast<const uint2 *>(dtout + off);
        float a = 0.f, b = 0.f;
        const uint32_t wo[2] = {uo.x, uo.y}, wt[2] = {ut.x, ut.y}, wd[2] = {ud.x, ud.y}, we[2] = {ue.x, ue.y};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float2 fo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&wo[h]));
            const float2 ft = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&wt[h]));
            const float2 fd = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&wd[h]));
            const float2 fe = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&we[h]));
            a = fmaf(fe.x, fo.x, fmaf(fe.y, fo.y, a));                          // <dtO, O>
            b = fmaf(fd.x, fo.x, fmaf(fd.y, fo.y, fmaf(fe.x, ft.x, fmaf(fe.y, ft.y, b))));  // <dO,O>+<dtO,tO>
        }
#pragma unroll
        for (int sh = 16; sh > 0; sh >>= 1) {
            a += __shfl_xor_sync(0xffffffffu, a, sh);
            b += __shfl_xor_sync(0xffffffffu, b, sh);
        }
        if (lane == 0) {
            const float m = mu[r];
            stats[r] = make_float4(lse[r] * 1.4426950408889634f, m, a, b - a * m);
        }
    }
}

template <int ROLE>
__global__ void __launch_bounds__(NTHREADS, 1) attn_jvp_bwd_kernel(const __grid_constant__ Params p) {
    extern __shared__ __align__(1024) uint8_t bwd_smem[];
    const uint32_t base = smem_u32(bwd_smem);
    if (base & 1023u) {  // the tile layout needs 1024-byte alignment and leaves no slack
        if (threadIdx.x == 0) atomicOr(&g_status_word, 2);
        return;
    }
    uint8_t *gbase = bwd_smem;
    constexpr bool kV = ROLE == ROLE_V;
    constexpr bool kColStats = ROLE != ROLE_Q;  // per-column (query) statistics

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int rt = blockIdx.x % p.n_rtiles;
    const int bh = blockIdx.x / p.n_rtiles;
    const int r0 = rt * BM;
    const int nt = (p.Lcol + BN - 1) / BN;
    const uint64_t bound = p.bound_ns;

    const uint32_t bars = base + SM_BAR;
    auto BAR = [&](int i) -> uint32_t { return bars + 8u * (uint32_t)i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + SM_BAR + OFF_TMEM_SLOT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + SM_BAR + OFF_ABORT);

    if (threadIdx.x == 0) {
        mbar_init(BAR(B_R_FULL), 1);
        for (int s = 0; s < LSTAGES; ++s) {
            mbar_init(BAR(B_L_FULL + s), 1);
            mbar_init(BAR(B_G2_DONE + s), 1);
        }
        mbar_init(BAR(B_S_FULL), 1);
        mbar_init(BAR(B_G1_DONE), 1);
        mbar_init(BAR(B_E_DONE), EW_THREADS);
        mbar_init(BAR(B_ACC_FULL), 1);
        mbar_init(BAR(B_MMA_DRAIN), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane < (kV ? 2 : 4)) {
        tma_prefetch_desc(&p.tm_r[lane]);
        tma_prefetch_desc(&p.tm_c[lane]);
    }
    if (warp == 2) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    // streamed tensors in the long ring (read by G2) and the short stage (G1 only)
    constexpr int L0 = kV ? 2 : 0, L1 = kV ? 3 : 1;  // C indices of the long ring
    constexpr int S0 = kV ? 0 : 2, S1 = kV ? 1 : 3;  // C indices of the short stage

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            bool ok = true;
            int l_last[LSTAGES] = {-1, -1}, s_last = -1;
            const int nr = kV ? 2 : 4;
            mbar_arrive_expect_tx(BAR(B_R_FULL), nr * R_TILE);
            for (int i = 0; i < nr; ++i) {
                tma_load_3d(base + SM_R + i * R_TILE, &p.tm_r[i], BAR(B_R_FULL), 0, r0, bh);
                tma_load_3d(base + SM_R + i * R_TILE + CHUNK_R, &p.tm_r[i], BAR(B_R_FULL), 64, r0, bh);
            }
            for (int t = 0; t < nt && ok; ++t) {
                const int y = t * BN;
                {   // long ring, stage t % 2: free once the G2 products of tile t - 2 are complete
                    const int s = t % LSTAGES;
                    if (t >= LSTAGES &&
                        !mbar_wait(BAR(B_G2_DONE + s), ((t - LSTAGES) / LSTAGES) & 1, abort_flag, bound)) {
                        ok = false;
                        break;
                    }
                    const uint32_t st = base + SM_L + s * C_STAGE;
                    const uint32_t fb = BAR(B_L_FULL + s);
                    mbar_arrive_expect_tx(fb, C_STAGE + (kColStats ? STATS_TILE : 0));
                    tma_load_3d(st, &p.tm_c[L0], fb, 0, y, bh);
                    tma_load_3d(st + CHUNK_C, &p.tm_c[L1], fb, 0, y, bh);
                    tma_load_3d(st + 2 * CHUNK_C, &p.tm_c[L0], fb, 64, y, bh);
                    tma_load_3d(st + 3 * CHUNK_C, &p.tm_c[L1], fb, 64, y, bh);
                    if (kColStats)  // padded by BN rows past the last head: never out of bounds
                        bulk_load(base + SM_ST + s * STATS_TILE, p.stats + (size_t)bh * p.Lq + y, STATS_TILE, fb);
                    l_last[s] = t;
                }
                {   // short stage: free once G1 of tile t - 1 is complete
                    if (t >= 1 && !mbar_wait(BAR(B_G1_DONE), (t - 1) & 1, abort_flag, bound)) {
                        ok = false;
                        break;
                    }
                    const uint32_t st = base + SM_S;
                    const uint32_t fb = BAR(B_S_FULL);
                    mbar_arrive_expect_tx(fb, C_STAGE);
                    tma_load_3d(st, &p.tm_c[S0], fb, 0, y, bh);
                    tma_load_3d(st + CHUNK_C, &p.tm_c[S1], fb, 0, y, bh);
                    tma_load_3d(st + 2 * CHUNK_C, &p.tm_c[S0], fb, 64, y, bh);
                    tma_load_3d(st + 3 * CHUNK_C, &p.tm_c[S1], fb, 64, y, bh);
                    s_last = t;
                }
            }
            // every copy already issued lands before shared memory is released
            mbar_wait_drain(BAR(B_R_FULL), 0, bound);
            for (int s = 0; s < LSTAGES; ++s)
                if (l_last[s] >= 0) mbar_wait_drain(BAR(B_L_FULL + s), (l_last[s] / LSTAGES) & 1, bound);
            if (s_last >= 0) mbar_wait_drain(BAR(B_S_FULL), s_last & 1, bound);
        }
        __syncwarp();
    } else if (warp == 1) {
        // -------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t ID_G1W = idesc_bf16_f32(128, 128, 0);  // R [Cx; Cy]^T
            constexpr uint32_t ID_G1N = idesc_bf16_f32(128, 64, 0);   // R Cx^T
            constexpr uint32_t ID_G2 = idesc_bf16_f32(128, 128, 1);   // E C (C read MN-major)
            uint64_t dr[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) dr[i] = smem_desc_sw128(base + SM_R + i * R_TILE, 16, 1024);
            const uint64_t dl0 = smem_desc_sw128(base + SM_L, 16, 1024);  // K-major view
            const uint64_t ds = smem_desc_sw128(base + SM_S, 16, 1024);
            // MN-major views of a long-ring tile: 64-column chunks C_CHUNK apart, 8 rows 1024 B apart
            const uint64_t dm0 = smem_desc_sw128(base + SM_L, C_CHUNK, 1024);
            const uint32_t t_x = tbase + TM_X, t_y = tbase + TM_Y, t_z = tbase + TM_Z;
            bool ok = mbar_wait(BAR(B_R_FULL), 0, abort_flag, bound);
            for (int j = 0; j < nt && ok; ++j) {
                const int s = j % LSTAGES;
                ok = mbar_wait(BAR(B_L_FULL + s), (j / LSTAGES) & 1, abort_flag, bound) &&
                     mbar_wait(BAR(B_S_FULL), j & 1, abort_flag, bound);
                if (!ok) break;
                tc_fence_after();
                // G1: the [C0; C1] pair sits in the long ring (ROLE_Q/K) or the short stage (ROLE_V)
                const uint64_t dc01 = kV ? ds : desc_add(dl0, s * C_STAGE);
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint32_t offr = (kk >> 2) * CHUNK_R + (kk & 3) * 32;
                    const uint32_t offc = (kk >> 2) * C_CHUNK + (kk & 3) * 32;
                    mma_ss(t_x, desc_add(dr[0], offr), desc_add(dc01, offc), ID_G1W, kk > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint32_t offr = (kk >> 2) * CHUNK_R + (kk & 3) * 32;
                    const uint32_t offc = (kk >> 2) * C_CHUNK + (kk & 3) * 32;
                    mma_ss(t_y, desc_add(dr[1], offr), desc_add(dc01, offc), ID_G1N, 1u);
                }
                if (!kV) {
#pragma unroll
                    for (int kk = 0; kk < HD / 16; ++kk) {
                        const uint32_t offr = (kk >> 2) * CHUNK_R + (kk & 3) * 32;
                        const uint32_t offc = (kk >> 2) * C_CHUNK + (kk & 3) * 32;
                        mma_ss(t_z, desc_add(dr[2], offr), desc_add(ds, offc), ID_G1W, kk > 0 ? 1u : 0u);
                    }
#pragma unroll
                    for (int kk = 0; kk < HD / 16; ++kk) {
                        const uint32_t offr = (kk >> 2) * CHUNK_R + (kk & 3) * 32;
                        const uint32_t offc = (kk >> 2) * C_CHUNK + (kk & 3) * 32;
                        mma_ss(t_z + 64, desc_add(dr[3], offr), desc_add(ds, offc), ID_G1N, 1u);
                    }
                }
                mma_commit(BAR(B_G1_DONE));
                // G2, once E1 (over X) and E2 (over Y) are written
                if (!(ok = mbar_wait(BAR(B_E_DONE), j & 1, abort_flag, bound))) break;
                tc_fence_after();
                const uint64_t b0 = desc_add(dm0, s * C_STAGE);  // long-ring tile x (C0, or C2 for ROLE_V)
                const uint64_t b1 = desc_add(b0, CHUNK_C);       // long-ring tile y (C1, or C3)
                const uint64_t b_acc1 = kV ? b1 : b0;
                const uint32_t e_acc1 = kV ? t_x : t_y;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    // streamed items 16kk..16kk+15: group kk/2's columns, 8 columns per K-step
                    const uint32_t a_col = (kk >> 1) * 32 + (kk & 1) * 8;
                    mma_ts(tbase + TM_ACC0, t_x + a_col, desc_add(b0, kk * 2048), ID_G2, (j > 0 || kk > 0) ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    const uint32_t a_col = (kk >> 1) * 32 + (kk & 1) * 8;
                    mma_ts(tbase + TM_ACC0, t_y + a_col, desc_add(b1, kk * 2048), ID_G2, 1u);
                }
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    const uint32_t a_col = (kk >> 1) * 32 + (kk & 1) * 8;
                    mma_ts(tbase + TM_ACC1, e_acc1 + a_col, desc_add(b_acc1, kk * 2048), ID_G2,
                           (j > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(BAR(B_G2_DONE + s));
            }
            if (ok) mma_commit(BAR(B_ACC_FULL));
            mma_commit(BAR(B_MMA_DRAIN));
            mbar_wait_drain(BAR(B_MMA_DRAIN), 0, bound);
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ------------------------------------------------ elementwise, epilogue
        const int grp = (warp - 4) >> 2;  // streamed columns 32*grp .. 32*grp+31 of each tile
        const int wl = warp & 3;          // tensor-memory lane quadrant
        const int row = wl * 32 + lane;
        const uint32_t lane_off = (uint32_t)(wl * 32) << 16;
        const uint32_t col0 = 32u * (uint32_t)grp;
        const float2 c2 = make_float2(p.scale_log2, p.scale_log2);
        const float2 s2 = make_float2(p.scale, p.scale);
        float4 rs = make_float4(0.f, 0.f, 0.f, 0.f);  // ROLE_Q: this row's {lse2, mu, a, D}
        if (!kColStats && r0 + row < p.Lrow) rs = p.stats[(size_t)bh * p.Lq + (size_t)(r0 + row)];
        bool failed = false;

        for (int j = 0; j < nt; ++j) {
            const int s = j % LSTAGES;
            if (!failed) failed = !mbar_wait_warp(BAR(B_G1_DONE), j & 1, abort_flag, bound);
            // the statistics came with the long-ring stage (bulk copy): observe its barrier too
            if (kColStats && !failed) failed = !mbar_wait_warp(BAR(B_L_FULL + s), (j / LSTAGES) & 1, abort_flag, bound);
            if (failed) continue;
            tc_fence_after();
            const int valid = p.Lcol - j * BN - (int)col0;  // this group's columns inside the tensor
            const uint32_t st_base = base + SM_ST + (uint32_t)s * STATS_TILE + col0 * 16u;
            uint32_t e1[16], e2[16];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t xr[16], yr[16], zr[16], wr[16];
                const uint32_t ta = tbase + lane_off + col0 + 16u * h;
                tmem_ld16(ta + TM_X, xr);
                tmem_ld16(ta + TM_Y, yr);
                if (!kV) {
                    tmem_ld16(ta + TM_Z, zr);
                    tmem_ld16(ta + TM_W, wr);
                }
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; i += 2) {
                    const int c = 16 * h + i;  // column inside the group
                    float4 sa = rs, sb = rs;   // statistics of columns c and c + 1
                    if (kColStats) {
                        sa = ld_shared_f4(st_base + 16u * c);
                        sb = ld_shared_f4(st_base + 16u * (c + 1));
                    }
                    const float2 x = make_float2(__uint_as_float(xr[i]), __uint_as_float(xr[i + 1]));
                    const float2 y = make_float2(__uint_as_float(yr[i]), __uint_as_float(yr[i + 1]));
                    const float2 t = __ffma2_rn(x, c2, make_float2(-sa.x, -sb.x));
                    const float2 pp = make_float2(ex2_approx(t.x), ex2_approx(t.y));
                    const float2 u = __fmul2_rn(y, s2);
                    const float2 umu = __fadd2_rn(u, make_float2(-sa.y, -sb.y));  // u - mu
                    float2 r1, r2;
                    if (kV) {
                        r1 = pp;                   // P
                        r2 = __fmul2_rn(pp, umu);  // P .* (u - mu)
                    } else {
                        const float2 z = make_float2(__uint_as_float(zr[i]), __uint_as_float(zr[i + 1]));
                        const float2 w = make_float2(__uint_as_float(wr[i]), __uint_as_float(wr[i + 1]));
                        const float2 na = make_float2(-sa.z, -sb.z);
                        r2 = __fmul2_rn(pp, __fadd2_rn(z, na));  // dS_bar = P (A - a)
                        // P_bar - D = B + A (u - mu) - a u - D
                        float2 pb = __ffma2_rn(z, umu, w);
                        pb = __ffma2_rn(na, u, pb);
                        pb = __fadd2_rn(pb, make_float2(-sa.w, -sb.w));
                        r1 = __fmul2_rn(pp, pb);  // S_bar
                    }
                    if (c >= valid) r1.x = r2.x = 0.f;  // columns past the end of the tensor
                    if (c + 1 >= valid) r1.y = r2.y = 0.f;
                    e1[8 * h + i / 2] = pack_bf16x2(r1.x, r1.y);
                    e2[8 * h + i / 2] = pack_bf16x2(r2.x, r2.y);
                }
            }
            tmem_st16(tbase + lane_off + TM_X + col0, e1);  // over this group's own X columns
            tmem_st16(tbase + lane_off + TM_Y + col0, e2);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(BAR(B_E_DONE));
        }

        if (!failed) failed = !mbar_wait_warp(BAR(B_ACC_FULL), 0, abort_flag, bound);
        const bool any_failed = named_bar_or(NB_EPI, EW_THREADS, failed);
        if (!any_failed) {
            tc_fence_after();
            const float os = p.out_scale;
            // group grp writes output columns 64*grp .. 64*grp+63, staged in R0 (acc0)
            // and R1 (acc1) in the 128-byte-swizzled layout of the store tensor maps
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {
                const int pc = 2 * grp + h;
                uint32_t ra[32], rb[32];
                tmem_ld32(tbase + lane_off + TM_ACC0 + 32u * pc, ra);
                tmem_ld32(tbase + lane_off + TM_ACC1 + 32u * pc, rb);
                tmem_wait_ld();
                uint32_t wa[16], wb[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    wa[i] = pack_bf16x2(__uint_as_float(ra[2 * i]) * os, __uint_as_float(ra[2 * i + 1]) * os);
                    wb[i] = pack_bf16x2(__uint_as_float(rb[2 * i]) * os, __uint_as_float(rb[2 * i + 1]) * os);
                }
                const uint32_t chunk_off = (uint32_t)grp * CHUNK_R + (uint32_t)row * 128u;
                const uint32_t unit0 = (uint32_t)h * 4u;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const uint32_t phys = (((unit0 + u) ^ (uint32_t)(row & 7)) * 16u);
                    st_shared_v4(base + SM_R + chunk_off + phys, wa[4 * u], wa[4 * u + 1], wa[4 * u + 2],
                                 wa[4 * u + 3]);
                    st_shared_v4(base + SM_R + R_TILE + chunk_off + phys, wb[4 * u], wb[4 * u + 1], wb[4 * u + 2],
                                 wb[4 * u + 3]);
                }
            }
        }
        fence_proxy_async_smem();
        named_bar_sync(NB_EPI, EW_THREADS);  // staging complete
        if (warp == 4 && lane == 0 && !any_failed && *abort_flag == 0) {
            tma_store_3d(&p.tm_out[0], base + SM_R, 0, r0, bh);
            tma_store_3d(&p.tm_out[0], base + SM_R + CHUNK_R, 64, r0, bh);
            tma_store_3d(&p.tm_out[1], base + SM_R + R_TILE, 0, r0, bh);
            tma_store_3d(&p.tm_out[1], base + SM_R + R_TILE + CHUNK_R, 64, r0, bh);
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

}  // namespace bwd
}  // namespace ajvp
