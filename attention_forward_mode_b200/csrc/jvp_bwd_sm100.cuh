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
//   attn_jvp_bwd_kernel<VAR>: one CTA per 128 "row-side" items (the MMA's
//   M = 128 dimension, tensor-memory lanes), streaming 64-wide tiles of the
//   other side; each output is an accumulation over the streamed side in
//   tensor memory (no atomics, no transposed stores).  Five variants, so
//   that each fits its score tiles and accumulators in the 512 columns of
//   tensor memory with room to overlap the elementwise work with the MMAs:
//
//   VAR    rows     streams  out       G1 per tile                         E             G2
//   V_DQ   queries  keys     dQ        [X|Y] = Q [K;tK]^T, Y += tQ K^T,    S_bar,        dQ += E1 K + E2 tK
//                                      [Z|W] = dtO [V;tV]^T, W += dO V^T   dS_bar
//   V_DTQ  queries  keys     dtQ       X = Q K^T, Z = dtO V^T              dS_bar        dtQ += E1 K
//   V_DK   keys     queries  dK        [X|Y] = K [Q;tQ]^T, Y += tK Q^T,    S_bar^T,      dK += E1 Q + E2 tQ
//                                      [Z|W] = V [dtO;dO]^T, W += tV dtO^T dS_bar^T
//   V_DKT  keys     queries  dtK, dtV  X = K Q^T, Z = V dtO^T              P^T, dS_bar^T dtK += E2 Q, dtV += E1 dtO
//   V_DV   keys     queries  dV        [X|Y] = K [Q;tQ]^T, Y += tK Q^T     P^T, Pd^T     dV += E1 dO + E2 dtO
//
//   (X = scores, Y = score tangent without the scale, Z = A, W = B, each 64
//   tensor-memory columns per tile; Pd = P .* (u - mu); the elementwise
//   results E1, E2 are bf16, the A operands of G2.)  V_DQ and V_DK hold one
//   set of X, Y, Z, W: their elementwise warps release it as soon as they
//   have read it (so G1 of the next tile runs while they compute) and write
//   E1, E2 to a region of their own.  The other variants double-buffer their
//   score tiles and write E1, E2 over them, as the forward kernel does.  The
//   resident tile R1 (V_DQ, V_DK) or R0 and R1 (V_DTQ, V_DV) are G1's A
//   operands straight from tensor memory, written there once by the
//   elementwise warps; the others are read from shared memory.
//
// Warp roles (384 threads): warp 0 TMA producer, warp 1 MMA issuer, warp 2
// tensor-memory allocation, warps 4-11 elementwise in two groups of four
// warps (group g takes columns 32g .. 32g+31 of each tile; one thread per
// row and group), which also run the epilogue (acc * scale -> bf16 -> TMA
// store).
#pragma once

#include "ptx_sm100.cuh"

namespace ajvp {
namespace bwd {

enum Variant : int { V_DQ = 0, V_DTQ = 1, V_DK = 2, V_DKT = 3, V_DV = 4, N_VARIANTS = 5 };

constexpr int BM = 128;  // row-side items per CTA
constexpr int BN = 64;   // streamed items per tile
constexpr int HD = 128;  // head dimension
constexpr int NTHREADS = 384;
constexpr int EW_THREADS = 256;

constexpr uint32_t CHUNK_R = 128 * 128;  // one 64-column chunk of a 128-row tile (bytes)
constexpr uint32_t CHUNK_C = 64 * 128;   // one 64-column chunk of a 64-row tile
constexpr uint32_t R_TILE = 2 * CHUNK_R;
constexpr uint32_t STATS_TILE = BN * 16;   // {lse2, mu, a, D} per streamed query
constexpr uint32_t SM_R = 0;               // resident tiles R0.., then the rings (per variant)

enum : int {
    B_R_FULL = 0,
    B_L_FULL = 1,    // + long stage (up to 4)
    B_S_FULL = 5,    // + short stage (up to 4)
    B_S_EMPTY = 9,   // + short stage: the G1 products that read it are complete
    B_G1_DONE = 13,  // + score buffer: X..W of the tile complete
    B_X_FREE = 15,   // single-buffer variants: the elementwise warps have read X..W (256 arrivals)
    B_E_DONE = 16,   // + score buffer: E1, E2 of the tile written (256 arrivals)
    B_G2_DONE = 18,  // + long stage: the tile's G2 products complete (the stage is free again)
    B_ACC_FULL = 22,
    B_MMA_DRAIN = 23,
    B_R1_READY = 24,  // R1 (and R0) written into tensor memory (256 arrivals)
    B_ST_FULL = 25,   // + slot: V_DK's own two-slot ring of column statistics
    N_BARS = 27
};
constexpr uint32_t OFF_TMEM_SLOT = 8 * N_BARS;
constexpr uint32_t OFF_ABORT = OFF_TMEM_SLOT + 4;
constexpr uint32_t NB_EPI = 1;

struct Params {
    CUtensorMap tm_r[4], tm_l[2], tm_s[2], tm_out[2];
    const float4 *stats;  // [B*H][Lq] {lse*log2(e), mu, a, D}, plus BN rows of padding
    const __nv_bfloat16 *r0, *r1;  // R0 / R1 ([B*H][Lrow][128]) where they are staged into tensor memory
    int Lrow, Lcol;       // row-side and streamed lengths
    int Lq;               // query rows per (batch, head): the stats row stride
    int n_rtiles;         // 128-row tiles per (batch, head)
    float scale;          // s
    float scale_log2;     // s * log2(e)
    float out_scale[2];   // factor applied to each accumulator at the end (s or 1)
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
            a = fmaf(fe.x, fo.x, fmaf(fe.y, fo.y, a));                                      // <dtO, O>
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

// Compile-time shape of one variant.
template <int VAR>
struct Var {
    static constexpr bool kSingle = VAR == V_DQ || VAR == V_DK;  // one score buffer, E region of its own
    static constexpr bool kTwoAcc = VAR == V_DKT;
    static constexpr bool kColStats = VAR == V_DK || VAR == V_DKT || VAR == V_DV;
    static constexpr bool kL1 = VAR != V_DTQ;                              // second long-ring tensor
    static constexpr int kNS = VAR == V_DKT ? 0 : (VAR == V_DTQ ? 1 : 2);  // short-stage tensors
    static constexpr int kNR = kSingle ? 4 : 2;        // resident tiles R0..R(kNR-1)
    static constexpr int kNB = kSingle ? 1 : 2;        // score buffers
    // streamed-tile rings: "long" (tiles G2 reads, freed when G2 completes) and
    // "short" (tiles only G1 reads, freed when G1 completes), as deep as shared
    // memory allows so that loads run well ahead of the products
    // resident A operands read from tensor memory instead of shared memory (the
    // score products then read only their streamed B tile there): R1 in every
    // variant with 64 free columns, R0 too where 128 are free (dtQ, dV)
    static constexpr bool kR0T = VAR == V_DTQ || VAR == V_DV;
    static constexpr bool kR1T = kSingle || kR0T;
    // single-buffer variants use R1's shared-memory slot as a third long-ring stage
    static constexpr bool kR1Stage = kSingle;
    static constexpr int kLS = kSingle ? 3 : (VAR == V_DV ? 2 : 4);
    // column statistics in shared memory: with the long-ring stage (double-buffer
    // variants), or in a two-slot ring of their own freed by the elementwise warps (V_DK)
    static constexpr bool kStatsSmem = kColStats;
    static constexpr bool kStatsRing = kColStats && kSingle;
    static constexpr int kSS = kNS == 0 ? 0 : (kSingle ? 1 : (VAR == V_DV ? 3 : 4));
    static constexpr int kSSd = kSS > 0 ? kSS : 1;  // divisor for short-ring indices
    // a stage holds one or two [64 rows][128] tiles as [x c0 | y c0 | x c1 | y c1]
    // (c = 64-column chunk); L_CH / S_CH = stride between a tile's two chunks
    static constexpr uint32_t L_CH = (kL1 ? 2u : 1u) * CHUNK_C, S_CH = (kNS > 1 ? 2u : 1u) * CHUNK_C;
    static constexpr uint32_t L_BYTES = 2 * L_CH, S_BYTES = 2 * S_CH;
    static constexpr uint32_t SM_L = SM_R + kNR * R_TILE;
    static constexpr uint32_t SM_S = SM_L + (kR1Stage ? kLS - 1 : kLS) * L_BYTES;
    static constexpr uint32_t SM_ST = SM_S + kSS * S_BYTES;  // statistics of the long-ring tiles
    static constexpr uint32_t SM_BAR = SM_ST + (kStatsRing ? 2 * STATS_TILE : (kStatsSmem ? kLS * STATS_TILE : 0u));
    __device__ static uint32_t long_off(int s) {  // offset of long-ring stage s
        return (kR1Stage && s == kLS - 1) ? SM_R + R_TILE : SM_L + (uint32_t)s * L_BYTES;
    }
    static constexpr uint32_t SMEM_BYTES = SM_BAR + 256;  // the base is 1024-byte aligned (checked)
    static_assert(SMEM_BYTES <= 232448, "exceeds the opt-in shared memory of one CTA");
    static_assert(8 * N_BARS + 8 <= 256, "barrier area");
    // tensor memory: accumulators, then the score buffer(s), then (single) E1, E2
    static constexpr uint32_t BUF0 = kTwoAcc ? 256u : 128u;
    static constexpr uint32_t BUF_COLS = kSingle ? 256u : 128u;
    static constexpr uint32_t X = 0, Y = 64, Z = kSingle ? 128u : 64u, W = 192;  // inside a buffer
    static constexpr uint32_t E1 = BUF0 + 256u, E2 = BUF0 + 288u;               // single only
    static constexpr uint32_t R0T = 384u, R1T = 448u;  // R0, R1 as bf16 pairs (64 columns each)
    static_assert(!kR0T || BUF0 + kNB * BUF_COLS <= R0T, "R0 overlaps the score buffers");
    static_assert(!kR1T || (kSingle ? E2 + 32u : BUF0 + kNB * BUF_COLS) <= R1T, "R1 overlaps");
};

template <int VAR>
__global__ void __launch_bounds__(NTHREADS, 1) attn_jvp_bwd_kernel(const __grid_constant__ Params p) {
    using C = Var<VAR>;
    extern __shared__ __align__(1024) uint8_t bwd_smem[];
    const uint32_t base = smem_u32(bwd_smem);
    if (base & 1023u) {  // the tile layout needs 1024-byte alignment and leaves no slack
        if (threadIdx.x == 0) atomicOr(&g_status_word, 2);
        return;
    }
    uint8_t *gbase = bwd_smem;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int rt = blockIdx.x % p.n_rtiles;
    const int bh = blockIdx.x / p.n_rtiles;
    const int r0 = rt * BM;
    const int nt = (p.Lcol + BN - 1) / BN;
    const uint64_t bound = p.bound_ns;

    const uint32_t bars = base + C::SM_BAR;
    auto BAR = [&](int i) -> uint32_t { return bars + 8u * (uint32_t)i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + C::SM_BAR + OFF_TMEM_SLOT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + C::SM_BAR + OFF_ABORT);

    if (threadIdx.x == 0) {
        mbar_init(BAR(B_R_FULL), 1);
        for (int s = 0; s < 4; ++s) {
            mbar_init(BAR(B_L_FULL + s), 1);
            mbar_init(BAR(B_S_FULL + s), 1);
            mbar_init(BAR(B_S_EMPTY + s), 1);
            mbar_init(BAR(B_G2_DONE + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(BAR(B_G1_DONE + b), 1);
            mbar_init(BAR(B_E_DONE + b), EW_THREADS);
        }
        mbar_init(BAR(B_X_FREE), EW_THREADS);
        mbar_init(BAR(B_R1_READY), EW_THREADS);
        mbar_init(BAR(B_ST_FULL), 1);
        mbar_init(BAR(B_ST_FULL + 1), 1);
        mbar_init(BAR(B_ACC_FULL), 1);
        mbar_init(BAR(B_MMA_DRAIN), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        if (lane < C::kNR) tma_prefetch_desc(&p.tm_r[lane]);
        if (lane < (C::kL1 ? 2 : 1)) tma_prefetch_desc(&p.tm_l[lane]);
        if (lane < C::kNS) tma_prefetch_desc(&p.tm_s[lane]);
    }
    if (warp == 2) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    if (warp == 0 || warp == 3) {
        // ------------------------------------------------------ TMA producers
        // warp 0: resident tiles and the long ring; warp 3: the short ring (the
        // two rings are released at different points, so neither waits on the other)
        const bool lp = warp == 0;
        if (lane == 0 && (lp || C::kSS > 0)) {
            bool ok = true;
            int l_last[4] = {-1, -1, -1, -1}, s_last[4] = {-1, -1, -1, -1}, st_last = -1;
            if (lp) {
                // (a phase that expects no bytes completes on this arrival alone)
                mbar_arrive_expect_tx(BAR(B_R_FULL), (C::kNR - (C::kR1T ? 1 : 0) - (C::kR0T ? 1 : 0)) * R_TILE);
                for (int i = 0; i < C::kNR; ++i) {
                    // R0 / R1 in tensor memory are written by the elementwise warps
                    if ((C::kR1T && i == 1) || (C::kR0T && i == 0)) continue;
                    tma_load_3d(base + SM_R + i * R_TILE, &p.tm_r[i], BAR(B_R_FULL), 0, r0, bh);
                    tma_load_3d(base + SM_R + i * R_TILE + CHUNK_R, &p.tm_r[i], BAR(B_R_FULL), 64, r0, bh);
                }
            }
            for (int t = 0; t < nt && ok; ++t) {
                const int y = t * BN;
                if (lp) {  // long ring, stage t % kLS: free once the G2 products of tile t - kLS are complete
                    const int s = t % C::kLS;
                    if (t >= C::kLS &&
                        !mbar_wait(BAR(B_G2_DONE + s), ((t - C::kLS) / C::kLS) & 1, abort_flag, bound)) {
                        ok = false;
                        break;
                    }
                    const uint32_t st = base + C::long_off(s);
                    const uint32_t fb = BAR(B_L_FULL + s);
                    constexpr bool kWithStats = C::kStatsSmem && !C::kStatsRing;
                    mbar_arrive_expect_tx(fb, (C::kL1 ? 4 : 2) * CHUNK_C + (kWithStats ? STATS_TILE : 0));
                    tma_load_3d(st, &p.tm_l[0], fb, 0, y, bh);
                    tma_load_3d(st + C::L_CH, &p.tm_l[0], fb, 64, y, bh);
                    if (C::kL1) {
                        tma_load_3d(st + CHUNK_C, &p.tm_l[1], fb, 0, y, bh);
                        tma_load_3d(st + C::L_CH + CHUNK_C, &p.tm_l[1], fb, 64, y, bh);
                    }
                    if (kWithStats)  // padded by BN rows past the last head: never out of bounds
                        bulk_load(base + C::SM_ST + s * STATS_TILE, p.stats + (size_t)bh * p.Lq + y, STATS_TILE, fb);
                    l_last[s] = t;
                }
                if (!lp) {  // short ring, stage t % kSS: free once G1 of tile t - kSS is complete
                    const int ss = t % C::kSSd;
                    if (t >= C::kSS &&
                        !mbar_wait(BAR(B_S_EMPTY + ss), ((t - C::kSS) / C::kSSd) & 1, abort_flag, bound)) {
                        ok = false;
                        break;
                    }
                    const uint32_t st = base + C::SM_S + ss * C::S_BYTES;
                    const uint32_t fb = BAR(B_S_FULL + ss);
                    mbar_arrive_expect_tx(fb, C::kNS * 2 * CHUNK_C);
                    tma_load_3d(st, &p.tm_s[0], fb, 0, y, bh);
                    tma_load_3d(st + C::S_CH, &p.tm_s[0], fb, 64, y, bh);
                    if (C::kNS > 1) {
                        tma_load_3d(st + CHUNK_C, &p.tm_s[1], fb, 0, y, bh);
                        tma_load_3d(st + C::S_CH + CHUNK_C, &p.tm_s[1], fb, 64, y, bh);
                    }
                    s_last[ss] = t;
                    if (C::kStatsRing) {
                        // statistics slot t % 2: free once the elementwise warps finished tile t - 2
                        // (E_DONE phases are waited in order, so the parity is unambiguous)
                        if (t >= 2 && !mbar_wait(BAR(B_E_DONE), (t - 2) & 1, abort_flag, bound)) {
                            ok = false;
                            break;
                        }
                        const uint32_t sb = BAR(B_ST_FULL + (t & 1));
                        mbar_arrive_expect_tx(sb, STATS_TILE);  // padded by BN rows: never out of bounds
                        bulk_load(base + C::SM_ST + (t & 1) * STATS_TILE, p.stats + (size_t)bh * p.Lq + y, STATS_TILE, sb);
                        st_last = t;
                    }
                }
            }
            // every copy already issued lands before shared memory is released
            if (lp) mbar_wait_drain(BAR(B_R_FULL), 0, bound);
            for (int s = 0; s < C::kLS; ++s)
                if (l_last[s] >= 0) mbar_wait_drain(BAR(B_L_FULL + s), (l_last[s] / C::kLS) & 1, bound);
            for (int s = 0; s < C::kSS; ++s)
                if (s_last[s] >= 0) mbar_wait_drain(BAR(B_S_FULL + s), (s_last[s] / C::kSSd) & 1, bound);
            for (int u = st_last - 1; u <= st_last; ++u)  // the last two statistics copies
                if (C::kStatsRing && u >= 0) mbar_wait_drain(BAR(B_ST_FULL + (u & 1)), (u >> 1) & 1, bound);
        }
        __syncwarp();
    } else if (warp == 1) {
        // -------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t ID_W = idesc_bf16_f32(128, 128, 0);  // R [Cx; Cy]^T
            constexpr uint32_t ID_N = idesc_bf16_f32(128, 64, 0);   // R Cx^T
            constexpr uint32_t ID_G2 = idesc_bf16_f32(128, 128, 1);  // E C (C read MN-major)
            // descriptors of the resident tiles, as scalars (an array captured by the
            // lambdas below would live in local memory and delay every MMA issue)
            const uint64_t dr0 = smem_desc_sw128(base + SM_R, 16, 1024);
            const uint64_t dr1 = desc_add(dr0, R_TILE), dr2 = desc_add(dr0, 2 * R_TILE), dr3 = desc_add(dr0, 3 * R_TILE);
            // K-x-K products over d = 128: 8 K-steps; a tile's two 64-column chunks are
            // CHUNK_R (resident) and ch (streamed stage) apart
            auto g1 = [&](uint32_t d, uint64_t a, uint64_t b, uint32_t ch, uint32_t id, bool acc) {
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint32_t offr = (kk >> 2) * CHUNK_R + (kk & 3) * 32;
                    const uint32_t offc = (kk >> 2) * ch + (kk & 3) * 32;
                    mma_ss(d, desc_add(a, offr), desc_add(b, offc), id, (acc || kk > 0) ? 1u : 0u);
                }
            };
            // the same with the A operand in tensor memory (column a_col, 8 columns per K-step)
            auto g1t = [&](uint32_t d, uint32_t a_col, uint64_t b, uint32_t ch, uint32_t id, bool acc) {
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk)
                    mma_ts(d, tbase + a_col + 8u * kk, desc_add(b, (kk >> 2) * ch + (kk & 3) * 32), id,
                           (acc || kk > 0) ? 1u : 0u);
            };
            auto wait_full = [&](int bar, int j, int stages) -> bool {
                if (!mbar_wait(BAR(bar + j % stages), (j / stages) & 1, abort_flag, bound)) return false;
                tc_fence_after();
                return true;
            };
            constexpr uint32_t LC = C::L_CH, SC = C::S_CH;
            auto issue_g1 = [&](int j) -> bool {
                const int b = j % C::kNB, s = j % C::kLS, ss = j % C::kSSd;
                const uint32_t tb = tbase + C::BUF0 + (uint32_t)b * C::BUF_COLS;
                const uint64_t dl = smem_desc_sw128(base + C::long_off(s), 16, 1024);
                const uint64_t ds = smem_desc_sw128(base + C::SM_S + ss * C::S_BYTES, 16, 1024);
                if (VAR != V_DV && !wait_full(B_L_FULL, j, C::kLS)) return false;  // V_DV: G1 reads no long tile
                if (VAR == V_DQ || VAR == V_DK) {
                    g1(tb + C::X, dr0, dl, LC, ID_W, false);   // [X | Y] = R0 [L0; L1]^T
                    g1t(tb + C::Y, C::R1T, dl, LC, ID_N, true);  // Y += R1 L0^T, R1 from tensor memory
                    // the short stage is needed only now: its load overlaps the products above
                    if (!wait_full(B_S_FULL, j, C::kSSd)) return false;
                    g1(tb + C::Z, dr2, ds, SC, ID_W, false);  // [Z | W] = R2 [S0; S1]^T
                    g1(tb + C::W, dr3, ds, SC, ID_N, true);   // W += R3 S0^T
                } else if (VAR == V_DTQ) {  // both A operands from tensor memory
                    g1t(tb + C::X, C::R0T, dl, LC, ID_N, false);  // X = R0 L0^T
                    if (!wait_full(B_S_FULL, j, C::kSSd)) return false;
                    g1t(tb + C::Z, C::R1T, ds, SC, ID_N, false);  // Z = R1 S0^T
                } else if (VAR == V_DKT) {
                    g1(tb + C::X, dr0, dl, LC, ID_N, false);                     // X = R0 L0^T
                    g1(tb + C::Z, dr1, desc_add(dl, CHUNK_C), LC, ID_N, false);  // Z = R1 L1^T
                } else {  // V_DV, both A operands from tensor memory
                    if (!wait_full(B_S_FULL, j, C::kSSd)) return false;
                    g1t(tb + C::X, C::R0T, ds, SC, ID_W, false);  // [X | Y] = R0 [S0; S1]^T
                    g1t(tb + C::Y, C::R1T, ds, SC, ID_N, true);   // Y += R1 S0^T
                }
                mma_commit(BAR(B_G1_DONE + b));
                if (C::kSS > 0) mma_commit(BAR(B_S_EMPTY + ss));
                return true;
            };
            auto issue_g2 = [&](int j) -> bool {
                // one E_DONE barrier per score buffer, so the parity is unambiguous: the
                // next phase of buffer j % 2 needs G1 of tile j + 2, issued after this wait
                // (single buffer: the elementwise warps wait for G2 of tile j first)
                if (!wait_full(B_E_DONE, j, C::kNB)) return false;
                if (VAR == V_DV && !wait_full(B_L_FULL, j, C::kLS)) return false;
                const int b = j % C::kNB, s = j % C::kLS;
                const uint32_t tb = tbase + C::BUF0 + (uint32_t)b * C::BUF_COLS;
                // MN-major views of the long-ring tiles: chunks L_CH apart (LBO), 8 rows 1024 B apart
                const uint64_t m0 = smem_desc_sw128(base + C::long_off(s), C::L_CH, 1024);
                const uint64_t m1 = desc_add(m0, CHUNK_C);
                const uint32_t e1 = C::kSingle ? tbase + C::E1 : tb + C::X;
                const uint32_t e2 = C::kSingle ? tbase + C::E2 : tb + (VAR == V_DKT ? C::Z : C::Y);
                auto g2 = [&](uint32_t acc, uint32_t e, uint64_t bm, bool first) {
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk) {
                        // streamed items 16kk..16kk+15: 8 packed columns per K-step
                        const uint32_t a_col = C::kSingle ? 8u * kk : (kk >> 1) * 32u + (kk & 1) * 8u;
                        mma_ts(tbase + acc, e + a_col, desc_add(bm, kk * 2048), ID_G2,
                               (!first || j > 0 || kk > 0) ? 1u : 0u);
                    }
                };
                if (VAR == V_DTQ) {
                    g2(0, e1, m0, true);    // acc0 += E1 L0
                } else if (VAR == V_DKT) {
                    g2(0, e2, m0, true);    // dtK += E2 L0
                    g2(128, e1, m1, true);  // dtV += E1 L1
                } else {
                    g2(0, e1, m0, true);    // acc0 += E1 L0
                    g2(0, e2, m1, false);   //       + E2 L1
                }
                mma_commit(BAR(B_G2_DONE + s));
                return true;
            };
            bool ok = mbar_wait(BAR(B_R_FULL), 0, abort_flag, bound);
            if (ok && C::kR1T) ok = wait_full(B_R1_READY, 0, 1);
            // one call site per issue routine: G1 of tile j + 1, then G2 of tile j
            for (int j = -1; j < nt && ok; ++j) {
                if (j + 1 < nt) {
                    // single buffer: the elementwise warps must have read tile j's X..W first
                    if (C::kSingle && j >= 0 && !(ok = mbar_wait(BAR(B_X_FREE), j & 1, abort_flag, bound))) break;
                    if (!(ok = issue_g1(j + 1))) break;
                }
                if (j >= 0) ok = issue_g2(j);
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
        float4 rs = make_float4(0.f, 0.f, 0.f, 0.f);  // row statistics {lse2, mu, a, D} (query rows)
        if (!C::kColStats && r0 + row < p.Lrow) rs = p.stats[(size_t)bh * p.Lq + (size_t)(r0 + row)];
        bool failed = false;
        if (C::kR1T) {
            // R1 (and R0) row `row` into tensor memory as bf16 pairs (column c = features
            // 2c, 2c+1), the layout of an A operand; group grp writes features 64*grp ..
            // 64*grp+63 (rows past the tensor: zeros)
            auto stage_row = [&](const __nv_bfloat16 *src_t, uint32_t col) {
                uint32_t w[32];
                if (r0 + row < p.Lrow) {
                    const uint4 *src = reinterpret_cast<const uint4 *>(
                        src_t + ((size_t)bh * (size_t)p.Lrow + (size_t)(r0 + row)) * HD + 64u * (uint32_t)grp);
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const uint4 v4 = __ldg(src + u);
                        w[4 * u] = v4.x;
                        w[4 * u + 1] = v4.y;
                        w[4 * u + 2] = v4.z;
                        w[4 * u + 3] = v4.w;
                    }
                } else {
#pragma unroll
                    for (int u = 0; u < 32; ++u) w[u] = 0u;
                }
                tmem_st32(tbase + lane_off + col + 32u * (uint32_t)grp, w);
            };
            stage_row(p.r1, C::R1T);
            if (C::kR0T) stage_row(p.r0, C::R0T);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(BAR(B_R1_READY));
        }

        // one pair of columns (c, c + 1 of this group): x scores, y score tangent,
        // z A, w B -> r1, r2 (see the variant table)
        const float4 *cst = p.stats;  // column statistics of the current tile (read through L1)
        auto pair = [&](int c, int valid, uint32_t st_base, uint32_t xa, uint32_t xb, uint32_t ya, uint32_t yb,
                        uint32_t za, uint32_t zb, uint32_t wa, uint32_t wb, float2 &r1, float2 &r2) {
            float4 sa = rs, sb = rs;  // statistics of columns c and c + 1
            if (C::kStatsSmem) {
                sa = ld_shared_f4(st_base + 16u * c);
                sb = ld_shared_f4(st_base + 16u * (c + 1));
            } else if (C::kColStats) {
                sa = __ldg(cst + c);
                sb = __ldg(cst + c + 1);
            }
            const float2 x = make_float2(__uint_as_float(xa), __uint_as_float(xb));
            const float2 t = __ffma2_rn(x, c2, make_float2(-sa.x, -sb.x));
            const float2 pp = make_float2(ex2_approx(t.x), ex2_approx(t.y));
            if (VAR == V_DV) {
                const float2 u = __fmul2_rn(make_float2(__uint_as_float(ya), __uint_as_float(yb)), s2);
                r1 = pp;                                                          // P
                r2 = __fmul2_rn(pp, __fadd2_rn(u, make_float2(-sa.y, -sb.y)));  // P (u - mu)
            } else {
                const float2 z = make_float2(__uint_as_float(za), __uint_as_float(zb));
                const float2 na = make_float2(-sa.z, -sb.z);
                const float2 dsb = __fmul2_rn(pp, __fadd2_rn(z, na));  // dS_bar = P (A - a)
                if (VAR == V_DTQ) {
                    r1 = dsb;
                    r2 = make_float2(0.f, 0.f);
                } else if (VAR == V_DKT) {
                    r1 = pp;
                    r2 = dsb;
                } else {  // V_DQ, V_DK: S_bar = P (B + A (u - mu) - a u - D)
                    const float2 u = __fmul2_rn(make_float2(__uint_as_float(ya), __uint_as_float(yb)), s2);
                    const float2 umu = __fadd2_rn(u, make_float2(-sa.y, -sb.y));
                    float2 pb = __ffma2_rn(z, umu, make_float2(__uint_as_float(wa), __uint_as_float(wb)));
                    pb = __ffma2_rn(na, u, pb);
                    pb = __fadd2_rn(pb, make_float2(-sa.w, -sb.w));
                    r1 = __fmul2_rn(pp, pb);
                    r2 = dsb;
                }
            }
            if (c >= valid) r1.x = r2.x = 0.f;  // columns past the end of the tensor
            if (c + 1 >= valid) r1.y = r2.y = 0.f;
        };

        for (int j = 0; j < nt; ++j) {
            const int b = j % C::kNB, s = j % C::kLS;
            if (!failed) failed = !mbar_wait_warp(BAR(B_G1_DONE + b), (j / C::kNB) & 1, abort_flag, bound);
            // the statistics came with the long-ring stage (bulk copy): observe its barrier too
            if (C::kStatsRing && !failed)
                failed = !mbar_wait_warp(BAR(B_ST_FULL + (j & 1)), (j >> 1) & 1, abort_flag, bound);
            else if (C::kStatsSmem && !failed)
                failed = !mbar_wait_warp(BAR(B_L_FULL + s), (j / C::kLS) & 1, abort_flag, bound);
            if (failed) continue;
            tc_fence_after();
            cst = p.stats + (size_t)bh * p.Lq + (size_t)j * BN + col0;  // padded: never out of bounds
            const int valid = p.Lcol - j * BN - (int)col0;  // this group's columns inside the tensor
            const uint32_t st_base =
                base + C::SM_ST + (uint32_t)(C::kStatsRing ? (j & 1) : s) * STATS_TILE + col0 * 16u;
            const uint32_t tb = tbase + lane_off + C::BUF0 + (uint32_t)b * C::BUF_COLS;
            uint32_t e1[16], e2[16];
            if (C::kSingle) {
                // all of this group's X..W (4 x 32 columns) at once, so that the buffer
                // is released for the next tile's G1 before any arithmetic
                uint32_t xr[32], yr[32], zr[32], wr[32];
                tmem_ld32(tb + col0 + C::X, xr);
                tmem_ld32(tb + col0 + C::Y, yr);
                tmem_ld32(tb + col0 + C::Z, zr);
                tmem_ld32(tb + col0 + C::W, wr);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(BAR(B_X_FREE));
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    float2 r1, r2;
                    pair(i, valid, st_base, xr[i], xr[i + 1], yr[i], yr[i + 1], zr[i], zr[i + 1], wr[i], wr[i + 1], r1,
                         r2);
                    e1[i / 2] = pack_bf16x2(r1.x, r1.y);
                    e2[i / 2] = pack_bf16x2(r2.x, r2.y);
                }
                // E1, E2 have a region of their own, read by G2 of the previous tile
                if (j >= 1 && !mbar_wait_warp(BAR(B_G2_DONE + (j - 1) % C::kLS), ((j - 1) / C::kLS) & 1, abort_flag,
                                              bound)) {
                    failed = true;
                    continue;
                }
                tc_fence_after();
                tmem_st16(tbase + lane_off + C::E1 + 16u * grp, e1);
                tmem_st16(tbase + lane_off + C::E2 + 16u * grp, e2);
            } else {
                uint32_t xr[32], yr[32];  // X and the second region (Y for V_DV, Z otherwise)
                const uint32_t second = VAR == V_DV ? C::Y : C::Z;
                tmem_ld32(tb + col0 + C::X, xr);
                tmem_ld32(tb + col0 + second, yr);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    float2 r1, r2;
                    pair(i, valid, st_base, xr[i], xr[i + 1], yr[i], yr[i + 1], yr[i], yr[i + 1], 0u, 0u, r1, r2);
                    e1[i / 2] = pack_bf16x2(r1.x, r1.y);
                    e2[i / 2] = pack_bf16x2(r2.x, r2.y);
                }
                // over this group's own columns of X and of the second region
                tmem_st16(tb + col0 + C::X, e1);
                if (VAR != V_DTQ) tmem_st16(tb + col0 + second, e2);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(BAR(B_E_DONE + b));
        }

        if (!failed) failed = !mbar_wait_warp(BAR(B_ACC_FULL), 0, abort_flag, bound);
        const bool any_failed = named_bar_or(NB_EPI, EW_THREADS, failed);
        if (!any_failed) {
            tc_fence_after();
            // group grp writes output columns 64*grp .. 64*grp+63 of each accumulator,
            // staged in R0 (acc0) and R1 (acc1) in the 128-byte-swizzled layout of the
            // store tensor maps
#pragma unroll 1
            for (int a = 0; a < (C::kTwoAcc ? 2 : 1); ++a) {
                const float os = p.out_scale[a];
#pragma unroll 1
                for (int h = 0; h < 2; ++h) {
                    const int pc = 2 * grp + h;
                    uint32_t ra[32];
                    tmem_ld32(tbase + lane_off + 128u * a + 32u * pc, ra);
                    tmem_wait_ld();
                    uint32_t wa[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        wa[i] = pack_bf16x2(__uint_as_float(ra[2 * i]) * os, __uint_as_float(ra[2 * i + 1]) * os);
                    const uint32_t dst = base + SM_R + (uint32_t)a * R_TILE + (uint32_t)grp * CHUNK_R + (uint32_t)row * 128u;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint32_t phys = (((uint32_t)h * 4u + u) ^ (uint32_t)(row & 7)) * 16u;
                        st_shared_v4(dst + phys, wa[4 * u], wa[4 * u + 1], wa[4 * u + 2], wa[4 * u + 3]);
                    }
                }
            }
        }
        fence_proxy_async_smem();
        named_bar_sync(NB_EPI, EW_THREADS);  // staging complete
        if (warp == 4 && lane == 0 && !any_failed && *abort_flag == 0) {
            for (int a = 0; a < (C::kTwoAcc ? 2 : 1); ++a) {
                tma_store_3d(&p.tm_out[a], base + SM_R + a * R_TILE, 0, r0, bh);
                tma_store_3d(&p.tm_out[a], base + SM_R + a * R_TILE + CHUNK_R, 64, r0, bh);
            }
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
