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
//   tensor memory (no atomics, no transposed stores).  Three variants, each
//   with two accumulators and its score tiles in the 512 columns of tensor
//   memory:
//
//   VAR  rows     streams  out       G1 per tile                          E             G2
//   V_Q  queries  keys     dQ, dtQ   [X|Y] = Q [K;tK]^T, Y += tQ K^T,     S_bar,        dQ  += E1 K + E2 tK
//                                    [Z|W] = dtO [V;tV]^T, W += dO V^T    dS_bar        dtQ += E2 K
//   V_K  keys     queries  dK, dtK   [X|Y] = K [Q;tQ]^T, Y += tK Q^T,     S_bar^T,      dK  += E1 Q + E2 tQ
//                                    [Z|W] = V [dtO;dO]^T, W += tV dtO^T  dS_bar^T      dtK += E2 Q
//   V_V  keys     queries  dV, dtV   [X|Y] = K [Q;tQ]^T, Y += tK Q^T      P^T, Pd^T     dV  += E1 dO + E2 dtO
//                                                                                       dtV += E1 dtO
//
//   (V_V issues its G2 as [dV | dtV] += E1 [dO | dtO], one N = 256 product, and
//   dV += E2 dtO.  X = scores, Y = score tangent without the scale, Z = A, W = B, each 64
//   tensor-memory columns per tile; Pd = P .* (u - mu); the elementwise
//   results E1, E2 are bf16, the A operands of G2.)  V_Q and V_K hold one
//   set of X, Y, Z, W next to their accumulators: the elementwise warps read
//   Z and W as soon as the [Z|W] products complete, release them (the next
//   tile's [Z|W] products may then run) and form their statistics terms
//   while the [X|Y] products still run; each group writes its E1 over its own
//   32 columns of X and E2 over its own 32 columns of Y (16 packed columns
//   each), so the next tile's [X|Y] products are issued after this tile's G2
//   (tensor-core operations run in issue order).  V_V double-buffers its two
//   score tiles and writes E1, E2 over them, as the forward kernel does.
//
// Warp roles (384 threads): warps 0 and 3 TMA producers (the long and the
// short ring), warp 1 MMA issuer, warp 2 tensor-memory allocation, warps
// 4-11 elementwise in two groups of four warps (group g takes columns
// 32g .. 32g+31 of each tile; one thread per row and group), which also run
// the epilogue (acc * scale -> bf16 -> tensor store; packed sequences:
// guarded row stores).
#pragma once

#include <type_traits>

#include "ptx_sm100.cuh"

namespace ajvp {
namespace bwd {

enum Variant : int { V_Q = 0, V_K = 1, V_V = 2, N_VARIANTS = 3 };

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
    B_X_FREE = 15,   // V_Q, V_K: the elementwise warps have read Z, W (one arrival per warp)
    B_E_DONE = 16,   // + score buffer: E1, E2 of the tile written (one arrival per warp)
    B_G2_DONE = 18,  // + long stage: the tile's G2 products complete (the stage is free again)
    B_ACC_FULL = 22,
    B_MMA_DRAIN = 23,
    B_ST_FULL = 24,   // + slot: V_K's own two-slot ring of column statistics
    B_ZW_DONE = 26,   // V_Q, V_K: the tile's [Z|W] products complete
    N_BARS = 27
};
constexpr uint32_t OFF_TMEM_SLOT = 8 * N_BARS;
constexpr uint32_t OFF_ABORT = OFF_TMEM_SLOT + 4;
constexpr uint32_t NB_EPI = 1;

// Masks (MASK bits): 1 causal -- key j is visible to query i iff
// j <= i + (Lk - Lq) of its sequence, bottom-right aligned; 2 packed -- the
// tensors are [H][total][128] and sequence b owns row-side rows
// cu_row[b] .. cu_row[b+1]-1 and streamed rows cu_col[b] .. cu_col[b+1]-1.
// 4 split (unmasked key-side variants only) -- the streamed range is cut into
// n_split consecutive parts, one per CTA, each writing its fp32 partial sums
// to partial[split][B*H][Lrow][2][128] (unscaled); bwd_split_reduce_kernel adds
// them up in split order, so the result stays deterministic.
constexpr int MASK_CAUSAL = 1, MASK_PACKED = 2, MASK_SPLIT = 4;

struct Params {
    CUtensorMap tm_r[4], tm_l[2], tm_s[2], tm_out[2];
    CUtensorMap tm_l32, tm_s32;  // pairs: L0 and S0 in boxes of 32 rows (the B2 halves)
    const float4 *stats;  // [B*H][Lq] {lse*log2(e), mu, a, D}, plus BN rows of padding
    int Lrow, Lcol;       // row-side and streamed lengths (packed: the tensors' totals)
    int Lq;               // query rows per (batch, head): the stats row stride
    int n_rtiles;         // 128-row tiles per (batch, head) (packed: of the longest sequence)
    int BH;               // packed: heads (the tensors' outermost extent); split: B*H
    int n_seq;            // packed: sequences per head
    const int *cu_row, *cu_col;  // packed: starts of each sequence's row-side / streamed rows
    __nv_bfloat16 *out[2];       // packed: the outputs as plain pointers (guarded row stores)
    int n_split;                 // split: parts of the streamed range
    float *partial;              // split: [n_split][B*H][Lrow][2][128] fp32 partial sums
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

// Sum of the split parts' fp32 partial sums, in part order, times the
// accumulator's output scale, rounded to bf16: out[a][row][:] for the
// rows x 2 accumulators of one key-side variant.  One thread per 4 columns.
__global__ void __launch_bounds__(256) bwd_split_reduce_kernel(const float4 *__restrict__ partial, int n_split,
                                                               long long rows, __nv_bfloat16 *__restrict__ out0,
                                                               __nv_bfloat16 *__restrict__ out1, float s0, float s1) {
    const long long n4 = rows * 2 * (HD / 4);  // float4s of one part
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
         i += (long long)gridDim.x * blockDim.x) {
        float4 acc = partial[i];
        for (int s = 1; s < n_split; ++s) {
            const float4 v = partial[(size_t)s * (size_t)n4 + (size_t)i];
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
        }
        const long long row = i / (2 * (HD / 4));
        const int a = (int)((i / (HD / 4)) & 1), c4 = (int)(i % (HD / 4));
        const float sc = a ? s1 : s0;
        uint2 w;
        w.x = pack_bf16x2(acc.x * sc, acc.y * sc);
        w.y = pack_bf16x2(acc.z * sc, acc.w * sc);
        *reinterpret_cast<uint2 *>((a ? out1 : out0) + (size_t)row * HD + 4u * c4) = w;
    }
}

// Bounded warp-wide wait of the elementwise warps: all 32 lanes poll the
// barrier together and leave when every lane has seen the phase complete
// (no lane spins alone while the others wait at a reconvergence point, so
// the warp resumes as soon as the phase flips).  The phase cannot move on
// again before this warp releases its stage, so a lane that has seen it keeps
// seeing it and the vote ends.  Lane 0 checks the abort flag and the time
// bound every 32 polls; on failure it raises the flag and the status bit and
// the whole warp returns false.
__device__ __forceinline__ bool ew_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag, uint64_t bound_ns) {
    const uint64_t t0 = global_timer_ns();
    for (uint32_t n = 1;; ++n) {
        if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
        if ((n & 31u) == 0) {
            int bad = 0;
            if ((threadIdx.x & 31) == 0) {
                if (*abort_flag) {
                    bad = 1;
                } else if (global_timer_ns() - t0 > bound_ns) {
                    *abort_flag = 1;
                    atomicOr(&g_status_word, 1);
                    bad = 1;
                }
            }
            if (__shfl_sync(0xffffffffu, bad, 0)) return false;
        }
    }
}

// ------------------------------------------------ CTA pairs (cta_group::2)
// A pair of CTAs on two SMs of one cluster shares each product: the even CTA
// issues M = 256 MMAs whose A rows 0..127 come from its own shared (or tensor)
// memory and rows 128..255 from its peer's, and whose B operand is split by
// N halves, the first half in the even CTA's shared memory and the second in
// the odd CTA's, at the same offsets; each CTA's tensor memory receives the
// accumulator rows of its own A rows, all N columns.
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// shared::cluster address of the same shared-memory offset in CTA `rank`
__device__ __forceinline__ uint32_t cluster_addr(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
// one arrival (release at cluster scope) on a barrier of another CTA of the cluster
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_bar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// bounded wait (acquire at cluster scope) for a barrier that other CTAs arrive on
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                                  uint64_t bound_ns) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t n = 1;; ++n) {
        if (mbar_try_wait_cluster(bar, parity)) return true;
        if ((n & 31u) == 0) {
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > bound_ns) {
                *abort_flag = 1;
                atomicOr(&g_status_word, 1);
                return false;
            }
        }
    }
}
// the odd CTA of a pair announces its part of a load on the even CTA's barrier
// (one arrival plus the bytes its copies will complete there)
__device__ __forceinline__ void mbar_arrive_expect_tx_remote(uint32_t cluster_bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cluster.shared::cluster.b64 _, [%0], %1;" ::"r"(cluster_bar),
                 "r"(bytes)
                 : "memory");
}
// 3-D tiled load global -> this CTA's shared memory whose completion is counted
// (bytes) on a barrier of either CTA of the pair (cta_group::2; this CTA is the only destination)
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const void *tmap, uint32_t cluster_bar, int x, int y,
                                                 int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, "
        "%5}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(cluster_bar), "r"(x), "r"(y), "r"(z)
        : "memory");
}
// every thread of both CTAs (aligned: whole warps)
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void mma_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// one arrival on the barrier at this offset in both CTAs of the pair once the
// pair's tensor-core operations issued so far have completed
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            bar),
        "h"((unsigned short)3)
        : "memory");
}

// Compile-time shape of one variant.  kPair: the dQ / dK variants as CTA
// pairs (the unmasked kernels only).
template <int VAR, bool kPair = false>
struct Var {
    static_assert(!kPair || VAR != V_V, "pairs are built for the dQ and dK variants");
    static constexpr bool kSingle = VAR != V_V;     // one set of X..W (E1, E2 written over X)
    static constexpr bool kColStats = VAR != V_Q;   // statistics per streamed query
    static constexpr int kNR = kSingle ? 4 : 2;     // resident tiles R0..R(kNR-1)
    static constexpr int kNB = kSingle ? 1 : 2;     // score buffers
    // streamed-tile rings: "long" (tiles G2 reads, freed when G2 completes) and
    // "short" (tiles only G1 reads, freed when G1 completes), as deep as shared
    // memory allows so that loads run well ahead of the products
    static constexpr int kLS = 2;
    static constexpr int kSS = kSingle ? 1 : 3;
    // column statistics in shared memory: with the long-ring stage (V_V), or in a
    // two-slot ring of their own freed by the elementwise warps (V_K)
    static constexpr bool kStatsRing = VAR == V_K;
    // a stage holds two [64 rows][128] tiles x, y as [x c0 | y c0 | x c1 | y c1]
    // (c = 64-column chunk), so that [x; y] is one N = 128 operand.
    // Pairs: each CTA holds its halves of the B operands (x: L0 / S0, y: L1 / S1):
    //   B1 [c0 | c1]  the N = 128 product's half: y in the even CTA, x in the odd one
    //   B2 [c0 | c1]  rows 32r .. 32r + 31 of x (CTA r): the N = 64 product's half
    //   B3            x's columns 64r .. 64r + 63 (long stage only): the N = 128 G2
    //                 product's half (B1, read MN-major, is the N = 256 one's)
    static constexpr uint32_t L_CH = 2u * CHUNK_C, S_CH = 2u * CHUNK_C;
    static constexpr uint32_t P_B2 = 2u * CHUNK_C, P_B3 = 3u * CHUNK_C, B2_CH = CHUNK_C / 2;
    static constexpr uint32_t L_BYTES = kPair ? 4u * CHUNK_C : 2 * L_CH;
    static constexpr uint32_t S_BYTES = kPair ? 3u * CHUNK_C : 2 * S_CH;
    static constexpr uint32_t SM_L = SM_R + kNR * R_TILE;
    static constexpr uint32_t SM_S = SM_L + kLS * L_BYTES;
    static constexpr uint32_t SM_ST = SM_S + kSS * S_BYTES;  // column statistics
    static constexpr uint32_t SM_BAR = SM_ST + (kStatsRing ? 2 * STATS_TILE : (kColStats ? kLS * STATS_TILE : 0u));
    __device__ static uint32_t long_off(int s) { return SM_L + (uint32_t)s * L_BYTES; }
    static constexpr uint32_t SMEM_BYTES = SM_BAR + 256;  // the base is 1024-byte aligned (checked)
    static_assert(SMEM_BYTES <= 232448, "exceeds the opt-in shared memory of one CTA");
    static_assert(8 * N_BARS + 8 <= 256, "barrier area");
    // tensor memory: two accumulators, then the score buffer(s)
    static constexpr uint32_t BUF0 = 256u;
    static constexpr uint32_t BUF_COLS = kSingle ? 256u : 128u;
    // inside a buffer (Z, W: V_Q, V_K).  The N = 128 products write [X|Y] and
    // [Z|W]; pairs write [Y|X] and [W|Z] (their first N half is y's), so the
    // N = 64 products, whose halves are rows of x, accumulate into Y and W
    static constexpr uint32_t X = kPair ? 64 : 0, Y = kPair ? 0 : 64, Z = kPair ? 192 : 128, W = kPair ? 128 : 192;
    static constexpr uint32_t G1B_D = 0, G1A_D = 128;  // the N = 128 products' first column
    // E1, E2 (16 packed columns per group) over each group's own columns of X and Y
    static constexpr uint32_t E1 = X, E2 = Y;
    static_assert(BUF0 + kNB * BUF_COLS == 512u, "tensor-memory layout");
};

// Causal: a CTA streams only the tiles that some row of its own sees (V_Q:
// keys 0 .. r0 + 127 + Lk - Lq; V_K, V_V: queries from r0 - (Lk - Lq) on),
// hidden pairs get P = 0, and a CTA whose rows see nothing writes zeros.
// Packed: a CTA is one 128-row tile of one (sequence, head); streamed tiles
// start at the sequence's first streamed row and columns past its end are
// hidden; rows past the sequence's end (the tile may overhang into the next
// sequence) are computed but not stored.
//
// Pairs (kPair, unmasked V_Q / V_K): a cluster of two CTAs takes row tiles
// 2m and 2m + 1 of a head.  The even CTA's MMA warp issues every product of
// the pair (cta_group::2, M = 256) and commits to the barriers of both CTAs;
// each CTA loads its own resident rows and its halves of the streamed
// operands, and the copies of both complete on the even CTA's barriers
// (cta_group::2 loads, each CTA announcing its bytes there); the odd CTA's
// elementwise warps arrive on the even CTA's X_FREE and E_DONE (which count
// both CTAs' warps).
// Both CTAs meet at a cluster barrier after setting up and before releasing
// tensor memory, so neither leaves while the other may still reach it.
template <int VAR, int MASK, bool kPair>
__device__ __forceinline__ void bwd_body(const Params &p) {
    using C = Var<VAR, kPair>;
    constexpr bool kCausal = (MASK & MASK_CAUSAL) != 0, kPacked = (MASK & MASK_PACKED) != 0;
    constexpr bool kSplitK = (MASK & MASK_SPLIT) != 0;
    static_assert(!kSplitK || (MASK == MASK_SPLIT && VAR != V_Q), "the split is for the unmasked key side");
    static_assert(!kPair || MASK == 0, "pairs are built for the unmasked kernels");
    extern __shared__ __align__(1024) uint8_t bwd_smem[];
    const uint32_t base = smem_u32(bwd_smem);
    if (base & 1023u) {  // the tile layout needs 1024-byte alignment and leaves no slack
        // (the same in both CTAs of a pair: both leave here)
        if (threadIdx.x == 0) atomicOr(&g_status_word, 2);
        return;
    }
    uint8_t *gbase = bwd_smem;
    const uint32_t crank = kPair ? cluster_rank() : 0u;  // 0: the CTA that issues the pair's products
    const bool issuer = crank == 0;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // this CTA: local row tile rt of a sequence (dense: the whole tensor) whose row-side
    // rows start at tensor row yr0 and streamed rows at yc0, Lrow_s and Lcol_s of them
    int rt, bh, yr0 = 0, yc0 = 0, Lrow_s = p.Lrow, Lcol_s = p.Lcol;
    if (kPacked) {
        // (sequence, head) major, row tiles fastest (they share the streamed rows in
        // L2); offsets clamped into the tensors so that bad ones stay memory-safe
        const int u = (int)(blockIdx.x % p.n_rtiles), sh = (int)(blockIdx.x / p.n_rtiles);
        const int b = sh / p.BH;
        bh = sh % p.BH;
        rt = (kCausal && VAR == V_Q) ? p.n_rtiles - 1 - u : u;  // causal dQ: late (heavy) tiles first
        yr0 = min(max(p.cu_row[b], 0), p.Lrow);
        Lrow_s = max(min(max(p.cu_row[b + 1], 0), p.Lrow), yr0) - yr0;
        yc0 = min(max(p.cu_col[b], 0), p.Lcol);
        Lcol_s = max(min(max(p.cu_col[b + 1], 0), p.Lcol), yc0) - yc0;
    } else if (kSplitK) {
        // split-major: the n_rtiles * BH tiles of part 0, then of part 1, ...
        const int cta = (int)(blockIdx.x % (unsigned)(p.n_rtiles * p.BH));
        rt = cta % p.n_rtiles;
        bh = cta / p.n_rtiles;
    } else {
        // causal dQ / dtQ: the late (heavy) query tiles of each head first
        rt = (kCausal && VAR == V_Q) ? p.n_rtiles - 1 - (int)(blockIdx.x % p.n_rtiles)
                                     : (int)(blockIdx.x % p.n_rtiles);
        bh = blockIdx.x / p.n_rtiles;
    }
    // split: this CTA's part of the streamed range
    const int sp = kSplitK ? (int)(blockIdx.x / (unsigned)(p.n_rtiles * p.BH)) : 0;
    const int r0 = rt * BM;  // local first row
    if (kPacked && r0 >= Lrow_s) return;  // past the end of this sequence (uniform for the CTA)
    const int yr = yr0 + r0;              // tensor row of the tile's first row
    // pairs: the odd CTA of a head's last pair may lie past the end (an odd tile
    // count); it loads rows 0.. instead, takes its part in the products and stores nothing
    const bool rows_live = r0 < Lrow_s;
    const int yr_load = (kPair && !rows_live) ? 0 : yr;
    // streamed tiles jt0 .. jt0 + nt - 1 (local index j = 0 .. nt - 1)
    int jt0 = 0, nt = (Lcol_s + BN - 1) / BN;
    if (kSplitK) {
        const int chunk = (nt + p.n_split - 1) / p.n_split;
        jt0 = sp * chunk;
        nt = max(0, min(chunk, nt - jt0));
    }
    // koff = Lk - Lq of the sequence: the causal diagonal's offset
    const int koff = VAR == V_Q ? Lcol_s - Lrow_s : Lrow_s - Lcol_s;
    if (kCausal) {
        if (VAR == V_Q) {
            const int kend = min(Lcol_s, r0 + BM + koff);  // keys some row of the tile sees
            nt = kend > 0 ? (kend + BN - 1) / BN : 0;
        } else {
            const int qbeg = max(0, r0 - koff);  // first query that sees a key of the tile
            jt0 = qbeg / BN;
            nt = qbeg < Lcol_s ? nt - jt0 : 0;
        }
    }
    const uint64_t bound = p.bound_ns;

    const uint32_t bars = base + C::SM_BAR;
    auto BAR = [&](int i) -> uint32_t { return bars + 8u * (uint32_t)i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + C::SM_BAR + OFF_TMEM_SLOT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + C::SM_BAR + OFF_ABORT);

    // the even CTA of a pair counts its own loads and the odd CTA's,
    // and both CTAs' elementwise warps
    const uint32_t n_load = (kPair && issuer) ? 2u : 1u, n_ew = (kPair && issuer) ? 2u : 1u;
    if (threadIdx.x == 0) {
        mbar_init(BAR(B_R_FULL), n_load);
        for (int s = 0; s < 4; ++s) {
            mbar_init(BAR(B_L_FULL + s), n_load);
            mbar_init(BAR(B_S_FULL + s), n_load);
            mbar_init(BAR(B_S_EMPTY + s), 1);
            mbar_init(BAR(B_G2_DONE + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(BAR(B_G1_DONE + b), 1);
            mbar_init(BAR(B_E_DONE + b), n_ew * (EW_THREADS / 32));  // one arrival per elementwise warp
        }
        mbar_init(BAR(B_X_FREE), n_ew * (EW_THREADS / 32));
        mbar_init(BAR(B_ZW_DONE), 1);
        mbar_init(BAR(B_ST_FULL), 1);
        mbar_init(BAR(B_ST_FULL + 1), 1);
        mbar_init(BAR(B_ACC_FULL), 1);
        mbar_init(BAR(B_MMA_DRAIN), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        if (lane < C::kNR) tma_prefetch_desc(&p.tm_r[lane]);
        if (lane < 2) {
            tma_prefetch_desc(&p.tm_l[lane]);
            tma_prefetch_desc(&p.tm_s[lane]);
        }
        if (kPair && lane == 2) tma_prefetch_desc(&p.tm_l32);
        if (kPair && lane == 3) tma_prefetch_desc(&p.tm_s32);
    }
    if (warp == 2) {
        if constexpr (kPair) {  // the same columns in both CTAs (warp 2 of each)
            tmem_alloc_pair(smem_u32(tmem_slot), 512);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_u32(tmem_slot), 512);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    if constexpr (kPair)
        cluster_sync_all();  // both CTAs' barriers initialised before any remote arrival
    else
        __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    // the even CTA's copy of one of this CTA's barriers (pairs)
    auto LEAD = [&](int i) -> uint32_t { return cluster_addr(BAR(i), 0u); };

    if (warp == 0 || warp == 3) {
        // ------------------------------------------------------ TMA producers
        // warp 0: resident tiles and the long ring; warp 3: the short ring (the
        // two rings are released at different points, so neither waits on the other)
        const bool lp = warp == 0;
        if (lane == 0) {
            // pairs: both CTAs' copies of the resident tiles and the rings complete on the
            // even CTA's barriers (cta_group::2 loads), each CTA announcing its own bytes
            // there; the odd CTA's own barriers of these kinds stay unused
            auto expect = [&](int bar, uint32_t bytes) {
                if (kPair && !issuer)
                    mbar_arrive_expect_tx_remote(LEAD(bar), bytes);
                else
                    mbar_arrive_expect_tx(BAR(bar), bytes);
            };
            auto load = [&](uint32_t dst, const CUtensorMap *m, int bar, int x, int y) {
                if constexpr (kPair)
                    tma_load_3d_pair(dst, m, LEAD(bar), x, y, bh);
                else
                    tma_load_3d(dst, m, BAR(bar), x, y, bh);
            };
            bool ok = true;
            int l_last[C::kLS], s_last[C::kSS], st_last = -1;
            for (int s = 0; s < C::kLS; ++s) l_last[s] = -1;
            for (int s = 0; s < C::kSS; ++s) s_last[s] = -1;
            if (lp) {
                expect(B_R_FULL, C::kNR * R_TILE);
                for (int i = 0; i < C::kNR; ++i) {
                    load(base + SM_R + i * R_TILE, &p.tm_r[i], B_R_FULL, 0, yr_load);
                    load(base + SM_R + i * R_TILE + CHUNK_R, &p.tm_r[i], B_R_FULL, 64, yr_load);
                }
            }
            // a stage [x c0 | y c0 | x c1 | y c1] of two streamed tensors, rows y..y+63
            auto load_pair = [&](uint32_t st, const CUtensorMap *mx, const CUtensorMap *my, uint32_t fb, int y) {
                tma_load_3d(st, mx, fb, 0, y, bh);
                tma_load_3d(st + CHUNK_C, my, fb, 0, y, bh);
                tma_load_3d(st + 2 * CHUNK_C, mx, fb, 64, y, bh);
                tma_load_3d(st + 3 * CHUNK_C, my, fb, 64, y, bh);
            };
            for (int t = 0; t < nt && ok; ++t) {
                const int y = yc0 + (jt0 + t) * BN;  // tensor row of the streamed tile
                if (lp) {  // long ring, stage t % kLS: free once the G2 products of tile t - kLS are complete
                    const int s = t % C::kLS;
                    if (t >= C::kLS &&
                        !mbar_wait(BAR(B_G2_DONE + s), ((t - C::kLS) / C::kLS) & 1, abort_flag, bound)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = BAR(B_L_FULL + s);
                    constexpr bool kWithStats = C::kColStats && !C::kStatsRing;
                    if (!kPair) mbar_arrive_expect_tx(fb, 4 * CHUNK_C + (kWithStats ? STATS_TILE : 0));
                    if constexpr (kPair) {
                        // B1: y (even CTA) or x (odd CTA); B2: rows 32r.. of x; B3: x's columns 64r..
                        const uint32_t st = base + C::long_off(s);
                        const CUtensorMap *b1 = issuer ? &p.tm_l[1] : &p.tm_l[0];
                        const int fi = B_L_FULL + s;
                        expect(fi, 4 * CHUNK_C);
                        load(st, b1, fi, 0, y);
                        load(st + CHUNK_C, b1, fi, 64, y);
                        load(st + C::P_B2, &p.tm_l32, fi, 0, y + 32 * (int)crank);
                        load(st + C::P_B2 + C::B2_CH, &p.tm_l32, fi, 64, y + 32 * (int)crank);
                        load(st + C::P_B3, &p.tm_l[0], fi, 64 * (int)crank, y);
                    } else if (VAR == V_V) {
                        // only G2 reads it, as one N = 256 operand [x | y]: [x c0 | x c1 | y c0 | y c1]
                        const uint32_t st = base + C::long_off(s);
                        tma_load_3d(st, &p.tm_l[0], fb, 0, y, bh);
                        tma_load_3d(st + CHUNK_C, &p.tm_l[0], fb, 64, y, bh);
                        tma_load_3d(st + 2 * CHUNK_C, &p.tm_l[1], fb, 0, y, bh);
                        tma_load_3d(st + 3 * CHUNK_C, &p.tm_l[1], fb, 64, y, bh);
                    } else {
                        load_pair(base + C::long_off(s), &p.tm_l[0], &p.tm_l[1], fb, y);
                    }
                    if (kWithStats)  // padded by BN rows past the last head: never out of bounds
                        bulk_load(base + C::SM_ST + s * STATS_TILE, p.stats + (size_t)bh * p.Lq + y, STATS_TILE, fb);
                    l_last[s] = t;
                } else {  // short ring, stage t % kSS: free once G1 of tile t - kSS is complete
                    // (V_Q, V_K: one stage, freed by the [Z|W] products' own completion barrier)
                    const int ss = t % C::kSS;
                    const int free_bar = C::kSingle ? (int)B_ZW_DONE : (int)B_S_EMPTY + ss;
                    if (t >= C::kSS &&
                        !mbar_wait(BAR(free_bar), ((t - C::kSS) / C::kSS) & 1, abort_flag, bound)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = BAR(B_S_FULL + ss);
                    const uint32_t st = base + C::SM_S + ss * C::S_BYTES;
                    if constexpr (kPair) {  // B1: y (even CTA) or x (odd CTA); B2: rows 32r.. of x
                        const int fi = B_S_FULL + ss;
                        expect(fi, 3 * CHUNK_C);
                        const CUtensorMap *b1 = issuer ? &p.tm_s[1] : &p.tm_s[0];
                        load(st, b1, fi, 0, y);
                        load(st + CHUNK_C, b1, fi, 64, y);
                        load(st + C::P_B2, &p.tm_s32, fi, 0, y + 32 * (int)crank);
                        load(st + C::P_B2 + C::B2_CH, &p.tm_s32, fi, 64, y + 32 * (int)crank);
                    } else {
                        mbar_arrive_expect_tx(fb, 4 * CHUNK_C);
                        load_pair(st, &p.tm_s[0], &p.tm_s[1], fb, y);
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
            // every copy already issued lands before shared memory is released (pairs: the
            // even CTA drains both CTAs' copies, and the cluster barrier at the end keeps the
            // odd CTA's shared memory until then; the statistics copies stay local)
            if (kPair && !issuer) {
                for (int s = 0; s < C::kLS; ++s) l_last[s] = -1;
                for (int s = 0; s < C::kSS; ++s) s_last[s] = -1;
            }
            if (lp && (!kPair || issuer)) mbar_wait_drain(BAR(B_R_FULL), 0, bound);
            for (int s = 0; s < C::kLS; ++s)
                if (l_last[s] >= 0) mbar_wait_drain(BAR(B_L_FULL + s), (l_last[s] / C::kLS) & 1, bound);
            for (int s = 0; s < C::kSS; ++s)
                if (s_last[s] >= 0) mbar_wait_drain(BAR(B_S_FULL + s), (s_last[s] / C::kSS) & 1, bound);
            for (int u = st_last - 1; u <= st_last; ++u)  // the last two statistics copies
                if (C::kStatsRing && u >= 0) mbar_wait_drain(BAR(B_ST_FULL + (u & 1)), (u >> 1) & 1, bound);
        }
        __syncwarp();
    } else if (warp == 1) {
        // -------------------------------------------------------- MMA issuer
        // (pairs: the even CTA's; the odd CTA's warp 1 has nothing to do)
        if (lane == 0 && (!kPair || issuer)) {
            constexpr uint32_t M = kPair ? 256 : 128;
            constexpr uint32_t ID_W = idesc_bf16_f32(M, 128, 0);  // R [Cx; Cy]^T
            constexpr uint32_t ID_N = idesc_bf16_f32(M, 64, 0);   // R Cx^T
            constexpr uint32_t ID_G2 = idesc_bf16_f32(M, 128, 1);  // E C (C read MN-major)
            constexpr uint32_t ID_G2W = idesc_bf16_f32(M, 256, 1);  // V_V: E1 [L0 | L1]; pairs: E2 [L1 | L0]
            auto commit = [&](int bar) {
                if constexpr (kPair)
                    mma_commit_pair(BAR(bar));
                else
                    mma_commit(BAR(bar));
            };
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
                    if constexpr (kPair)
                        mma_ss_pair(d, desc_add(a, offr), desc_add(b, offc), id, (acc || kk > 0) ? 1u : 0u);
                    else
                        mma_ss(d, desc_add(a, offr), desc_add(b, offc), id, (acc || kk > 0) ? 1u : 0u);
                }
            };
            // (pairs: the odd CTA arrives on these barriers too; acquire at cluster scope)
            auto wait_bar = [&](int bar, uint32_t parity) -> bool {
                if constexpr (kPair)
                    return mbar_wait_cluster(BAR(bar), parity, abort_flag, bound);
                else
                    return mbar_wait(BAR(bar), parity, abort_flag, bound);
            };
            auto wait_full = [&](int bar, int j, int stages) -> bool {
                if (!wait_bar(bar + j % stages, (j / stages) & 1)) return false;
                tc_fence_after();
                return true;
            };
            constexpr uint32_t LC = C::L_CH, SC = C::S_CH;
            // G1, first part: V_Q, V_K [Z|W] = R2 [S0; S1]^T, W += R3 S0^T (the short
            // stage, released here); V_V all of its G1, [X|Y] = R0 [S0; S1]^T, Y += R1 S0^T
            auto issue_g1a = [&](int j) -> bool {
                const int b = j % C::kNB, ss = j % C::kSS;
                const uint32_t tb = tbase + C::BUF0 + (uint32_t)b * C::BUF_COLS;
                const uint64_t ds = smem_desc_sw128(base + C::SM_S + ss * C::S_BYTES, 16, 1024);
                if (!wait_full(B_S_FULL, j, C::kSS)) return false;
                // V_Q, V_K: ZW_DONE also frees the (single) short stage
                if (kPair) {  // [W|Z] = R2 [S1 | S0]^T by halves, W += R3 S0^T by row halves
                    g1(tb + C::G1A_D, dr2, ds, CHUNK_C, ID_W, false);
                    g1(tb + C::W, dr3, desc_add(ds, C::P_B2), C::B2_CH, ID_N, true);
                    commit(B_ZW_DONE);
                } else if (C::kSingle) {
                    g1(tb + C::Z, dr2, ds, SC, ID_W, false);
                    g1(tb + C::W, dr3, ds, SC, ID_N, true);
                    commit(B_ZW_DONE);
                } else {
                    g1(tb + C::X, dr0, ds, SC, ID_W, false);
                    g1(tb + C::Y, dr1, ds, SC, ID_N, true);
                    commit(B_G1_DONE + b);
                    commit(B_S_EMPTY + ss);
                }
                return true;
            };
            // G1, second part (V_Q, V_K): [X|Y] = R0 [L0; L1]^T, Y += R1 L0^T, over the X
            // region that the previous tile's G2 read (issued after it) and the Y region
            // the elementwise warps read before E_DONE
            auto issue_g1b = [&](int j) -> bool {
                const uint32_t tb = tbase + C::BUF0;
                const uint64_t dl = smem_desc_sw128(base + C::long_off(j % C::kLS), 16, 1024);
                if (!wait_full(B_L_FULL, j, C::kLS)) return false;
                if (kPair) {  // [Y|X] = R0 [L1 | L0]^T by halves, Y += R1 L0^T by row halves
                    g1(tb + C::G1B_D, dr0, dl, CHUNK_C, ID_W, false);
                    g1(tb + C::Y, dr1, desc_add(dl, C::P_B2), C::B2_CH, ID_N, true);
                } else {
                    g1(tb + C::X, dr0, dl, LC, ID_W, false);
                    g1(tb + C::Y, dr1, dl, LC, ID_N, true);
                }
                commit(B_G1_DONE);
                return true;
            };
            auto issue_g2 = [&](int j) -> bool {
                // one E_DONE barrier per score buffer, so the parity is unambiguous: the
                // next phase of buffer j % kNB needs G1 of tile j + kNB, issued after this
                if (!wait_full(B_E_DONE, j, C::kNB)) return false;
                if (!C::kSingle && !wait_full(B_L_FULL, j, C::kLS)) return false;  // V_V: only G2 reads it
                const int b = j % C::kNB, s = j % C::kLS;
                const uint32_t tb = tbase + C::BUF0 + (uint32_t)b * C::BUF_COLS;
                const uint32_t e1 = tb + C::E1, e2 = tb + C::E2;
                auto g2 = [&](uint32_t acc, uint32_t e, uint64_t bm, uint32_t id, bool first) {
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk) {
                        // streamed items 16kk..16kk+15: group kk / 2's columns, 8 packed per K-step
                        const uint32_t a_col = (kk >> 1) * 32u + (kk & 1) * 8u;
                        const uint32_t en = (!first || j > 0 || kk > 0) ? 1u : 0u;
                        if constexpr (kPair)
                            mma_ts_pair(tbase + acc, e + a_col, desc_add(bm, kk * 2048), id, en);
                        else
                            mma_ts(tbase + acc, e + a_col, desc_add(bm, kk * 2048), id, en);
                    }
                };
                if (kPair) {
                    // B1 read MN-major (two 64-column chunks CHUNK_C apart, 8 rows 1024 B apart):
                    // [acc0 | acc1] += E2 [L1 | L0] (the first product of the tile: it starts
                    // both accumulators), then acc0 += E1 L0 with B3 (x's columns by halves)
                    const uint64_t mw = smem_desc_sw128(base + C::long_off(s), CHUNK_C, 1024);
                    g2(0, e2, mw, ID_G2W, true);
                    g2(0, e1, desc_add(mw, C::P_B3), ID_G2, false);
                } else if (VAR == V_V) {
                    // MN-major [L0 | L1]: 64-column chunks CHUNK_C apart (LBO), 8 rows 1024 B apart
                    const uint64_t mw = smem_desc_sw128(base + C::long_off(s), CHUNK_C, 1024);
                    g2(0, e1, mw, ID_G2W, true);                         // [dV | dtV] += E1 [L0 | L1]
                    g2(0, e2, desc_add(mw, 2 * CHUNK_C), ID_G2, false);  // dV += E2 L1
                } else {
                    // MN-major views of the long-ring tiles: chunks L_CH apart (LBO), 8 rows 1024 B apart
                    const uint64_t m0 = smem_desc_sw128(base + C::long_off(s), C::L_CH, 1024);
                    const uint64_t m1 = desc_add(m0, CHUNK_C);
                    g2(0, e1, m0, ID_G2, true);    // acc0 += E1 L0
                    g2(0, e2, m1, ID_G2, false);   //       + E2 L1
                    g2(128, e2, m0, ID_G2, true);  // dtQ / dtK += E2 L0
                }
                commit(B_G2_DONE + s);
                return true;
            };
            bool ok = wait_bar(B_R_FULL, 0);
            // one call site per issue routine.  V_Q, V_K: [X|Y] of tile j, [Z|W] of tile
            // j + 1 once the elementwise warps have read tile j's Z and W (they do so as
            // soon as tile j's [Z|W] completes, long before its [X|Y]), then G2 of tile j.
            // V_V: G1 of tile j + 1, then G2 of tile j.
            for (int j = -1; j < nt && ok; ++j) {
                if (C::kSingle && j >= 0 && !(ok = issue_g1b(j))) break;
                if (j + 1 < nt) {
                    if (C::kSingle && j >= 0 && !(ok = wait_bar(B_X_FREE, j & 1))) break;
                    if (!(ok = issue_g1a(j + 1))) break;
                }
                if (j >= 0 && !(ok = issue_g2(j))) break;
            }
            if (ok) commit(B_ACC_FULL);
            commit(B_MMA_DRAIN);
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
        if (!C::kColStats && r0 + row < Lrow_s) rs = p.stats[(size_t)bh * p.Lq + (size_t)(yr + row)];
        bool failed = false;
        // one arrival per warp for the MMA warp (pairs: on the even CTA's barrier; the
        // odd CTA's warps also arrive on their own E_DONE, which frees the column
        // statistics slot for this CTA's producer)
        auto arrive_mma = [&](int bar, bool local_too) {
            if constexpr (kPair) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (issuer) {
                        mbar_arrive(BAR(bar));
                    } else {
                        mbar_arrive_remote(LEAD(bar));
                        if (local_too) mbar_arrive(BAR(bar));
                    }
                }
            } else {
                warp_arrive_after_tc(BAR(bar));
            }
        };
        // one pair of columns (c, c + 1 of this group): x scores, y score tangent,
        // z A, w B -> r1, r2 (see the variant table)
        auto pair = [&](int c, int lo, int hi, bool masked, uint32_t st_base, uint32_t xa, uint32_t xb, uint32_t ya,
                        uint32_t yb, uint32_t za, uint32_t zb, uint32_t wa, uint32_t wb, float2 &r1, float2 &r2) {
            float4 sa = rs, sb = rs;  // statistics of columns c and c + 1
            if (C::kColStats) {
                sa = ld_shared_f4(st_base + 16u * c);
                sb = ld_shared_f4(st_base + 16u * (c + 1));
            }
            const float2 x = make_float2(__uint_as_float(xa), __uint_as_float(xb));
            const float2 t = __ffma2_rn(x, c2, make_float2(-sa.x, -sb.x));
            const float2 pp = make_float2(ex2_approx(t.x), ex2_approx(t.y));
            if (VAR == V_V) {
                // u - mu = s Y - mu in one packed FMA
                const float2 umu = __ffma2_rn(make_float2(__uint_as_float(ya), __uint_as_float(yb)), s2,
                                              make_float2(-sa.y, -sb.y));
                r1 = pp;                     // P
                r2 = __fmul2_rn(pp, umu);    // P (u - mu)
            } else {  // dS_bar = P (A - a), S_bar = P (B + A (u - mu) - a u - D)
                const float2 z = make_float2(__uint_as_float(za), __uint_as_float(zb));
                const float2 na = make_float2(-sa.z, -sb.z);
                const float2 dsb = __fmul2_rn(pp, __fadd2_rn(z, na));
                const float2 u = __fmul2_rn(make_float2(__uint_as_float(ya), __uint_as_float(yb)), s2);
                const float2 umu = __fadd2_rn(u, make_float2(-sa.y, -sb.y));
                float2 pb = __ffma2_rn(z, umu, make_float2(__uint_as_float(wa), __uint_as_float(wb)));
                pb = __ffma2_rn(na, u, pb);
                pb = __fadd2_rn(pb, make_float2(-sa.w, -sb.w));
                r1 = __fmul2_rn(pp, pb);
                r2 = dsb;
            }
            // columns past the end of the tensor, or hidden by the causal mask
            if (masked) {
                if (c >= hi || c < lo) r1.x = r2.x = 0.f;
                if (c + 1 >= hi || c + 1 < lo) r1.y = r2.y = 0.f;
            }
        };

        for (int j = 0; j < nt; ++j) {
            const int b = j % C::kNB, s = j % C::kLS;
            // V_Q, V_K: Z and W first (complete well before X and Y)
            const int g1bar = C::kSingle ? (int)B_ZW_DONE : (int)B_G1_DONE + b;
            if (!failed) failed = !ew_wait(BAR(g1bar), (j / C::kNB) & 1, abort_flag, bound);
            // the statistics came with the long-ring stage (bulk copy): observe its barrier too
            if (C::kStatsRing && !failed)
                failed = !ew_wait(BAR(B_ST_FULL + (j & 1)), (j >> 1) & 1, abort_flag, bound);
            else if (C::kColStats && !failed)
                failed = !ew_wait(BAR(B_L_FULL + s), (j / C::kLS) & 1, abort_flag, bound);
            if (failed) continue;
            tc_fence_after();
            // this group's columns lo .. hi - 1 are inside the tensor and visible
            const int y0 = (jt0 + j) * BN + (int)col0;  // the group's first streamed item
            int lo = 0, hi = Lcol_s - y0;
            if (kCausal) {
                if (VAR == V_Q)
                    hi = min(hi, r0 + row + koff - y0 + 1);  // keys <= query + (Lk - Lq)
                else
                    lo = r0 + row - koff - y0;  // queries >= key - (Lk - Lq)
            }
            const uint32_t st_base =
                base + C::SM_ST + (uint32_t)(C::kStatsRing ? (j & 1) : s) * STATS_TILE + col0 * 16u;
            const uint32_t tb = tbase + lane_off + C::BUF0 + (uint32_t)b * C::BUF_COLS;
            const float *stf = reinterpret_cast<const float *>(gbase + (st_base - base));
            uint32_t e1[16], e2[16];
            if (C::kSingle) {
                // this group's Z and W as soon as the tile's [Z|W] products complete (the
                // next tile's [Z|W] products overwrite only them and start once they are
                // read), and their statistics terms formed while [X|Y] still runs:
                //   za = A - a,  wz = B - D - A mu,
                // so that once X and Y arrive only P = ex2(c S - lse2), u = s Y,
                // S_bar = P (u za + wz) and dS_bar = P za remain (the critical path of
                // the tile: the next [X|Y] products follow this tile's G2, which waits
                // for E_DONE)
                float za[32], wz[32];
                {
                    uint32_t zr[32], wr[32];
                    tmem_ld32(tb + col0 + C::Z, zr);
                    tmem_ld32(tb + col0 + C::W, wr);
                    tmem_wait_ld();
                    arrive_mma(B_X_FREE, false);
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {  // two columns per packed instruction
                        const float4 sa = C::kColStats ? ld_shared_f4(st_base + 16u * i) : rs;
                        const float4 sb = C::kColStats ? ld_shared_f4(st_base + 16u * (i + 1)) : rs;
                        const float2 z = make_float2(__uint_as_float(zr[i]), __uint_as_float(zr[i + 1]));
                        const float2 w = make_float2(__uint_as_float(wr[i]), __uint_as_float(wr[i + 1]));
                        const float2 d = __fadd2_rn(z, make_float2(-sa.z, -sb.z));
                        const float2 e = __ffma2_rn(make_float2(-z.x, -z.y), make_float2(sa.y, sb.y),
                                                    __fadd2_rn(w, make_float2(-sa.w, -sb.w)));
                        za[i] = d.x;
                        za[i + 1] = d.y;
                        wz[i] = e.x;
                        wz[i + 1] = e.y;
                    }
                }
                if (!ew_wait(BAR(B_G1_DONE), j & 1, abort_flag, bound)) {
                    failed = true;
                    continue;
                }
                tc_fence_after();
                // X and Y in two halves of 16 columns; each half's E1, E2 (8 packed columns
                // each) go over columns of X and Y that half has already read.  The
                // per-column mask only for tiles that reach past the end or cross the
                // causal diagonal: most tiles see all their columns and take a copy of the
                // loop without the tests.
                auto e_halves = [&](auto masked_c) {
                    constexpr bool kMasked = decltype(masked_c)::value;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        uint32_t xr[16], yr[16], h1[8], h2[8];
                        tmem_ld16(tb + col0 + C::X + 16u * hh, xr);
                        tmem_ld16(tb + col0 + C::Y + 16u * hh, yr);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 16; i += 2) {
                            const int c = 16 * hh + i;
                            // lse2 of columns c, c + 1 (column statistics: read again from the
                            // slot, which stays valid until E_DONE)
                            const float2 ls =
                                C::kColStats ? make_float2(stf[4 * c], stf[4 * c + 4]) : make_float2(rs.x, rs.x);
                            const float2 x = make_float2(__uint_as_float(xr[i]), __uint_as_float(xr[i + 1]));
                            const float2 tt = __ffma2_rn(x, c2, make_float2(-ls.x, -ls.y));
                            const float2 pp = make_float2(ex2_approx(tt.x), ex2_approx(tt.y));
                            const float2 u =
                                __fmul2_rn(make_float2(__uint_as_float(yr[i]), __uint_as_float(yr[i + 1])), s2);
                            const float2 zz = make_float2(za[c], za[c + 1]);
                            const float2 pb = __ffma2_rn(u, zz, make_float2(wz[c], wz[c + 1]));
                            float2 r1 = __fmul2_rn(pp, pb), r2 = __fmul2_rn(pp, zz);
                            if (kMasked) {  // columns past the end of the tensor, or hidden by the causal mask
                                if (c >= hi || c < lo) r1.x = r2.x = 0.f;
                                if (c + 1 >= hi || c + 1 < lo) r1.y = r2.y = 0.f;
                            }
                            h1[i / 2] = pack_bf16x2(r1.x, r1.y);
                            h2[i / 2] = pack_bf16x2(r2.x, r2.y);
                        }
                        tmem_st8(tb + col0 + C::E1 + 8u * hh, h1);
                        tmem_st8(tb + col0 + C::E2 + 8u * hh, h2);
                    }
                };
                // the choice must be the same for the whole warp: the copies hold
                // warp-collective tensor-memory loads and stores
                if (__all_sync(0xffffffffu, lo <= 0 && hi >= 32))
                    e_halves(std::false_type{});
                else
                    e_halves(std::true_type{});
            } else {
                uint32_t xr[32], yr[32];
                tmem_ld32(tb + col0 + C::X, xr);
                tmem_ld32(tb + col0 + C::Y, yr);
                tmem_wait_ld();
                // the per-column mask only for tiles that reach past the end or cross the
                // causal diagonal (most tiles see all their columns); one choice per warp
                if (__all_sync(0xffffffffu, lo <= 0 && hi >= 32)) {
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        float2 r1, r2;
                        pair(i, lo, hi, false, st_base, xr[i], xr[i + 1], yr[i], yr[i + 1], 0u, 0u, 0u, 0u, r1, r2);
                        e1[i / 2] = pack_bf16x2(r1.x, r1.y);
                        e2[i / 2] = pack_bf16x2(r2.x, r2.y);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        float2 r1, r2;
                        pair(i, lo, hi, true, st_base, xr[i], xr[i + 1], yr[i], yr[i + 1], 0u, 0u, 0u, 0u, r1, r2);
                        e1[i / 2] = pack_bf16x2(r1.x, r1.y);
                        e2[i / 2] = pack_bf16x2(r2.x, r2.y);
                    }
                }
            }
            // over this group's own columns of X and Y (the previous tile's G2, which read
            // E from there, completed before this tile's G1)
            if (!C::kSingle) {
                tmem_st16(tb + col0 + C::E1, e1);
                tmem_st16(tb + col0 + C::E2, e2);
            }
            tmem_wait_st();
            arrive_mma(B_E_DONE + b, true);
        }

        if (!failed) failed = !ew_wait(BAR(B_ACC_FULL), 0, abort_flag, bound);
        const bool any_failed = named_bar_or(NB_EPI, EW_THREADS, failed);
        if (!any_failed) {
            tc_fence_after();
            // group grp writes output columns 64*grp .. 64*grp+63 of each accumulator,
            // staged in R0 (acc0) and R1 (acc1) in the 128-byte-swizzled layout of the
            // store tensor maps
#pragma unroll 1
            for (int a = 0; a < 2; ++a) {
                const float os = p.out_scale[a];
#pragma unroll 1
                for (int h = 0; h < 2; ++h) {
                    const int pc = 2 * grp + h;
                    uint32_t ra[32];
                    if (MASK != 0 && nt == 0) {  // no row of the tile sees anything (or an empty part): zeros
#pragma unroll
                        for (int i = 0; i < 32; ++i) ra[i] = 0u;
                    } else {
                        tmem_ld32(tbase + lane_off + 128u * a + 32u * pc, ra);
                        tmem_wait_ld();
                    }
                    if constexpr (kSplitK) {
                        // this part's fp32 partial sums, unscaled (the reduction scales them)
                        if (r0 + row < Lrow_s) {
                            float4 *dst = reinterpret_cast<float4 *>(
                                p.partial + ((((size_t)sp * (size_t)p.BH + (size_t)bh) * (size_t)p.Lrow +
                                              (size_t)(yr + row)) * 2u + (size_t)a) * HD + 64u * grp + 32u * h);
#pragma unroll
                            for (int u = 0; u < 8; ++u)
                                dst[u] = make_float4(__uint_as_float(ra[4 * u]), __uint_as_float(ra[4 * u + 1]),
                                                     __uint_as_float(ra[4 * u + 2]), __uint_as_float(ra[4 * u + 3]));
                        }
                    } else {
                        uint32_t wa[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            wa[i] = pack_bf16x2(__uint_as_float(ra[2 * i]) * os, __uint_as_float(ra[2 * i + 1]) * os);
                        if (kPacked) {
                            // rows past the sequence's end belong to the next one: not written
                            if (r0 + row < Lrow_s) {
                                uint4 *dst = reinterpret_cast<uint4 *>(
                                    p.out[a] + ((size_t)bh * (size_t)p.Lrow + (size_t)(yr + row)) * HD + 64u * grp +
                                    32u * h);
#pragma unroll
                                for (int u = 0; u < 4; ++u)
                                    dst[u] = make_uint4(wa[4 * u], wa[4 * u + 1], wa[4 * u + 2], wa[4 * u + 3]);
                            }
                            continue;
                        }
                        const uint32_t dst =
                            base + SM_R + (uint32_t)a * R_TILE + (uint32_t)grp * CHUNK_R + (uint32_t)row * 128u;
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const uint32_t phys = (((uint32_t)h * 4u + u) ^ (uint32_t)(row & 7)) * 16u;
                            st_shared_v4(dst + phys, wa[4 * u], wa[4 * u + 1], wa[4 * u + 2], wa[4 * u + 3]);
                        }
                    }  // bf16 outputs
                }
            }
        }
        fence_proxy_async_smem();
        named_bar_sync(NB_EPI, EW_THREADS);  // staging complete
        if (!kPacked && !kSplitK && warp == 4 && lane == 0 && !any_failed && *abort_flag == 0 && rows_live) {
            for (int a = 0; a < 2; ++a) {
                tma_store_3d(&p.tm_out[a], base + SM_R + a * R_TILE, 0, yr, bh);
                tma_store_3d(&p.tm_out[a], base + SM_R + a * R_TILE + CHUNK_R, 64, yr, bh);
            }
            tma_store_commit();
            tma_store_wait_all();
        }
        __syncwarp();
    }

    tc_fence_before();
    if constexpr (kPair)
        cluster_sync_all();  // the peer's loads, arrivals and products are all over
    else
        __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        if constexpr (kPair)
            tmem_dealloc_pair(tbase, 512);
        else
            tmem_dealloc(tbase, 512);
    }
}

template <int VAR, int MASK = 0>
__global__ void __launch_bounds__(NTHREADS, 1) attn_jvp_bwd_kernel(const __grid_constant__ Params p) {
    bwd_body<VAR, MASK, false>(p);
}

// The dQ / dK variants as CTA pairs (grid: an even number of row tiles per head).
template <int VAR>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NTHREADS, 1)
    attn_jvp_bwd_kernel_pair(const __grid_constant__ Params p) {
    bwd_body<VAR, 0, true>(p);
}

}  // namespace bwd
}  // namespace ajvp
