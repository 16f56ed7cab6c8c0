// jvp_sm100.cuh -- fused attention + Jacobian-vector product, bf16 I/O,
// fp32 accumulation, for sm_100a (B200): TMA tile loads through mbarrier
// pipelines, tcgen05 MMAs accumulating in tensor memory, warp-specialised
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
// One CTA owns 128 query rows of one (batch, head); 384 threads:
//   warp 0       TMA producer (one lane): Q, tQ once; K|tK and V|tV tiles
//                through two 2-stage rings.
//   warp 1       MMA issuer (one lane), per 64-key tile j:
//                  [S_j | dS'_j]  = Q  [K_j | tK_j]^T      (N = 128)
//                         dS'_j  += tQ K_j^T               (N = 64)
//                  [O | T]       += P_j  [V_j | tV_j]      (N = 256, A in TMEM)
//                         T      += PdS_j V_j              (N = 128, A in TMEM)
//   warp 2       tensor-memory allocation / release.
//   warps 4-7    softmax group 0: keys 0-31 of every tile,
//   warps 8-11   softmax group 1: keys 32-63 of every tile.
//                One thread per (query row, group); rows are TMEM lanes.  The
//                two groups exchange their partial row maxima through shared
//                memory once per tile, so both keep the same reference max
//                and partial sums l, g that add up at the end.  Each group
//                rescales half of the accumulators (group 0 O, group 1 T) and
//                writes half of the outputs.
//
// Tensor memory (512 columns x 128 lanes of fp32):
//   [0,128) O_acc   [128,256) T_acc   [256,384) S/dS' buffer 0
//   [384,512) S/dS' buffer 1    (S at +0, dS' at +64 inside a buffer)
// bf16 P is written over S and bf16 P.*s dS' over dS', each group inside its
// own 32 columns (group 0 at +0, group 1 at +32), so neither group overwrites
// values the other still has to read.  They are the A operands of the
// second MMA pair: 16 keys = 8 TMEM columns per K-step.
//
// Persistent form (kPersist, unmasked bf16 only; chosen for short key
// sequences such as cross-attention to a few hundred text tokens, where a CTA
// runs only a handful of key tiles): one CTA per SM walks the units
// (query tile, batch*head) blockIdx.x, blockIdx.x + gridDim.x, ..., and every
// ring, buffer and barrier phase follows one CTA-wide tile counter G = n*nk + j
// (unit n, key tile j).  The epilogue stages O and tO in the V-side ring
// (whose tiles are dead once every product of the unit is complete) and warp
// 3 stores them with the tensor-store unit, so Q / tQ shared memory is
// refilled for unit n+1 as soon as the last S/dS' products of unit n are
// complete, and the next unit's first score products run during the
// epilogue; the producer loads unit n+1's first V tiles once the stores have
// read the staging (B_STG_FREE), and the next unit's first P.V waits for the
// epilogue to have read O / T (B_OT_FREE).
#pragma once

#include "ptx_sm100.cuh"

namespace ajvp {
namespace sm100 {

constexpr int BR = 128;  // query rows per CTA
constexpr int BC = 64;   // keys per tile
constexpr int HD = 128;  // head dimension
constexpr int NTHREADS = 384;
constexpr int SOFTMAX_THREADS = 256;
constexpr int STAGES = 2;

constexpr uint32_t CHUNK_Q = 128 * 128;  // one 64-column chunk of a 128-row tile (bytes)
constexpr uint32_t CHUNK_K = 64 * 128;   // one 64-column chunk of a 64-row tile
constexpr uint32_t SM_Q = 0;             // Q  [2 chunks][128 rows][128 B]
constexpr uint32_t SM_TQ = SM_Q + 2 * CHUNK_Q;
constexpr uint32_t KT_STAGE = 4 * CHUNK_K;  // [K c0 | tK c0 | K c1 | tK c1]
constexpr uint32_t VT_STAGE = 4 * CHUNK_K;  // [V c0 | V c1 | tV c0 | tV c1]
constexpr uint32_t KT_CHUNK = 2 * CHUNK_K;  // stride between 64-column chunks of the K side
constexpr uint32_t SM_KT = SM_TQ + 2 * CHUNK_Q;
constexpr uint32_t SM_VT = SM_KT + STAGES * KT_STAGE;
constexpr uint32_t SM_BAR = SM_VT + STAGES * VT_STAGE;
constexpr uint32_t SM_XCH = SM_BAR + 256;  // fp32 [2 buffers][2 groups][128 rows] partial maxima,
                                           // then [l, g][2 groups][128 rows] final sums
constexpr uint32_t XCH_FLOATS = 2 * 2 * 128 + 2 * 2 * 128;
constexpr uint32_t STG_SLOT = 32 * 64;                 // one softmax warp's 32 rows x 32 bf16 columns
constexpr uint32_t SM_STG = SM_XCH + 4 * XCH_FLOATS;  // 8 staging slots for the plain-store epilogue
constexpr uint32_t SMEM_BYTES = SM_STG + 8 * STG_SLOT + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 232448, "dynamic shared memory above the sm_100 per-CTA limit");
// Persistent form: a third V-side stage (the next unit's first V tile never shares a
// stage with the previous unit's staged outputs); the exchange area holds only the
// per-tile maxima, which the final l, g exchange reuses; no staging slots, and no
// alignment slack (the kernel checks that the dynamic shared memory starts on a
// 1024-byte boundary)
constexpr int VSTAGES_P = 3;
constexpr uint32_t SM_BAR_P = SM_VT + VSTAGES_P * VT_STAGE;
constexpr uint32_t SM_XCH_P = SM_BAR_P + 256;
constexpr uint32_t SMEM_BYTES_P = SM_XCH_P + 2 * 2 * 128 * 4;
static_assert(SMEM_BYTES_P <= 232448, "dynamic shared memory above the sm_100 per-CTA limit");

// barrier slots (8 bytes each).  Two MMA commits per key tile:
//   B_SD_FULL[j % 2]  S_j / dS'_j complete: the softmax may read them, and
//                     K-side stage j % 2 (same index) may be refilled
//   B_VT_EMPTY[j % 2] P_j.V_j etc. complete: V-side stage j % 2 may be
//                     refilled, and O / T may be rescaled before P_{j+1}.V
enum : int {
    B_Q_FULL = 0,
    B_KT_FULL = 1,   // + stage
    B_VT_FULL = 3,   // + V-side stage (3 in the persistent form)
    B_VT_EMPTY = 6,  // + V-side stage
    B_SD_FULL = 9,   // + buffer (= K-side stage)
    B_P_FULL = 11,   // + buffer
    B_O_FULL = 13,   // every MMA of the unit has completed (one phase per unit)
    B_MMA_DRAIN = 14,
    B_OT_FREE = 15,   // persistent: the epilogue has read O / T (one arrival per softmax warp)
    B_STG_FULL = 16,  // persistent: O, tO staged in the V-side ring (one arrival per softmax warp)
    B_STG_FREE = 17,  // persistent: + 0 the stores have read O's stage, + 1 tO's as well
    N_BARS = 19
};
static_assert(STAGES == 2, "the K-side ring reuses the two S/dS' buffer barriers");
constexpr uint32_t OFF_TMEM_SLOT = 8 * N_BARS;     // u32
constexpr uint32_t OFF_ABORT = OFF_TMEM_SLOT + 4;  // int

constexpr uint32_t TM_O = 0, TM_T = 128, TM_BUF = 256;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units: P entries stay <= 256
// kSplit: every SPLIT_FOLD_TILES key tiles the O / T accumulators are added
// into the fp32 outputs (round-to-nearest fp32 adds on the CUDA cores) and the
// next tile's products start them afresh in tensor memory, so that no
// accumulator takes more than SPLIT_FOLD_TILES tiles of tensor-core adds
constexpr int SPLIT_FOLD_TILES = 32;

// named barriers of the 256 softmax threads
constexpr uint32_t NB_TILE = 2, NB_EPI = 1;

struct Params {
    CUtensorMap tm_q, tm_tq, tm_k, tm_tk, tm_v, tm_tv, tm_o, tm_to;
    float *o_f32, *to_f32;  // kSplit: fp32 outputs [B*H][Lq][128] (tm_o / tm_to unused)
    float *lse;
    float *mu;  // optional [B*H][Lq]: mu_i = sum_j P_ij s dS'_ij (saved for the backward)
    __nv_bfloat16 *o_bf, *to_bf;  // bf16 outputs as plain pointers (packed rows, empty tiles)
    const int *cu_q, *cu_k;       // packed sequences: starts of each sequence's rows (n_seq + 1)
    int n_seq;                    // packed sequences per head
    int BH;                       // dense: B*H; packed: H (the tensors' outermost extent)
    int Lq, Lk, n_qtiles;  // rows per (batch, head) -- packed: total rows; n_qtiles: 128-row tiles
                           // per (batch, head) -- packed: tiles of the longest sequence
    int n_units;           // persistent: n_qtiles * BH query tiles shared out over the grid
    float scale;           // s
    float scale_log2;      // s * log2(e)
    unsigned long long bound_ns;
};

// Coalesced store of one warp's 32 rows x 32 bf16 columns (lane = row, w = its
// 64 bytes): through the warp's 2 KB shared-memory slot, 16-byte chunk c of row
// r at r*64 + ((c ^ ((r >> 1) & 3)) << 4) (conflict-free for both the row-wise
// writes and the chunk-wise reads), then 8 rows x 64 contiguous bytes per
// global store instruction instead of 32 rows x 16 bytes.  Rows >= rows_left
// are not written; dst: the warp's row 0 at its first column, rows HD apart.
__device__ __forceinline__ void store_rows_32x32(uint32_t slot, const uint32_t (&w)[16], __nv_bfloat16 *dst,
                                                 int rows_left, uint32_t lane) {
#pragma unroll
    for (uint32_t c = 0; c < 4; ++c)
        st_shared_v4(slot + lane * 64u + ((c ^ ((lane >> 1) & 3u)) << 4), w[4 * c], w[4 * c + 1], w[4 * c + 2],
                     w[4 * c + 3]);
    __syncwarp();
#pragma unroll
    for (uint32_t k = 0; k < 4; ++k) {
        const uint32_t r = 8u * k + (lane >> 2), c = lane & 3u;
        const uint4 v = ld_shared_u4(slot + r * 64u + ((c ^ ((r >> 1) & 3u)) << 4));
        if ((int)r < rows_left) *reinterpret_cast<uint4 *>(dst + (size_t)r * HD + 8u * c) = v;
    }
    __syncwarp();  // the slot is free again
}

// Key masks (MASK bits): 1 causal -- key j is visible to query i of a sequence
// iff j <= i + (Lk - Lq), bottom-right aligned; 2 packed -- the tensors are
// [H][total][128] and sequence b owns rows cu_q[b] .. cu_q[b+1]-1 (queries)
// and cu_k[b] .. cu_k[b+1]-1 (keys).  Rows with no visible key give zeros and
// lse = -inf.
constexpr int MASK_CAUSAL = 1, MASK_PACKED = 2;

// kSplit = false: bf16 P and P.*s dS' operands, bf16 outputs.
// kSplit = true : P and P.*s dS' are each split into bf16 hi + lo parts
//                 (x = hi + lo to ~16 significant bits), both multiplied into
//                 O and T, and O, tO are written in fp32; 1.5x the MMA work.
//                 The tensor cores' fp32 accumulation loses a little on every
//                 add into a large accumulator, and over tens of thousands of
//                 keys that loss adds up: so every SPLIT_FOLD_TILES tiles each
//                 softmax thread adds its row's accumulators into the fp32
//                 output rows (the running sums live there until the end) and
//                 the next P.V products overwrite tensor memory instead of
//                 adding to it.  A rescale of the reference max between folds
//                 is carried by one factor per row (opend) applied at the next
//                 fold and in the epilogue.
template <bool kSplit, int MASK = 0, bool kPersist = false>
__global__ void __launch_bounds__(NTHREADS, 1) attn_jvp_fwd_kernel(const __grid_constant__ Params p) {
    static_assert(!kPersist || (!kSplit && MASK == 0), "the persistent form is the unmasked bf16 kernel");
    constexpr bool kCausal = (MASK & MASK_CAUSAL) != 0, kPacked = (MASK & MASK_PACKED) != 0;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);
    // V-side ring depth, barrier area and exchange area of this form
    constexpr int VST = kPersist ? VSTAGES_P : STAGES;
    constexpr uint32_t kBar = kPersist ? SM_BAR_P : SM_BAR, kXch = kPersist ? SM_XCH_P : SM_XCH;
    if (kPersist && base != raw) {  // its layout leaves no alignment slack
        if (threadIdx.x == 0) atomicOr(&g_status_word, 2);
        return;
    }

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // this CTA's tile: outermost tensor index bh, local rows q0.. of a sequence whose
    // rows start at tensor row yq - q0 and keys at yk0, with Lq_s rows and Lk_s keys
    int qt, bh, Lq_s = p.Lq, Lk_s = p.Lk, yk0 = 0, yq0 = 0;
    if (kPacked) {
        // sequence b's rows and keys, clamped into the tensors so that bad offsets stay memory-safe
        auto q_begin = [&](int b) { return min(max(p.cu_q[b], 0), p.Lq); };
        auto k_begin = [&](int b) { return min(max(p.cu_k[b], 0), p.Lk); };
        int b;
        if (!kCausal && p.n_seq <= 32) {
            // without the causal mask a unit costs its sequence's key count whatever its
            // query tile, so the units go out longest sequence first (ties: lower index),
            // which leaves the short ones for the last wave.  Every warp ranks the
            // sequences itself, one per lane; consecutive CTAs take the query tiles of
            // one (sequence, head), which share its keys in L2.
            const int l = threadIdx.x & 31;
            int units = 0, cost = -1;  // lanes past the last sequence: no units, ranked last
            if (l < p.n_seq) {
                const int a0 = q_begin(l), a1 = max(q_begin(l + 1), a0);
                const int k0 = k_begin(l), k1 = max(k_begin(l + 1), k0);
                units = (a1 - a0 + BR - 1) / BR * p.BH;
                cost = k1 - k0;
            }
            int rank = 0;
#pragma unroll 4
            for (int m = 0; m < 32; ++m) {
                const int cm = __shfl_sync(0xffffffffu, cost, m);
                rank += (cm > cost || (cm == cost && m < l)) ? 1 : 0;
            }
            int first = 0;  // units of the sequences ranked before this one
#pragma unroll 4
            for (int m = 0; m < 32; ++m) {
                const int rm = __shfl_sync(0xffffffffu, rank, m), um = __shfl_sync(0xffffffffu, units, m);
                first += rm < rank ? um : 0;
            }
            const int i = (int)blockIdx.x;
            const unsigned own = __ballot_sync(0xffffffffu, i >= first && i < first + units);
            if (own == 0u) return;  // past the last unit (the same for the whole CTA)
            b = __ffs(own) - 1;
            const int local = i - __shfl_sync(0xffffffffu, first, b);
            const int nq = __shfl_sync(0xffffffffu, units, b) / p.BH;
            bh = local / nq;
            qt = local % nq;
        } else {
            // heaviest first for the causal mask: the last tiles of every (sequence, head)
            // go in the first wave
            bh = blockIdx.x % p.BH;
            const int rest = blockIdx.x / p.BH;
            b = rest % p.n_seq;
            qt = p.n_qtiles - 1 - rest / p.n_seq;
        }
        const int a0 = q_begin(b), a1 = max(q_begin(b + 1), a0);
        const int k0 = k_begin(b), k1 = max(k_begin(b + 1), k0);
        yq0 = a0;
        Lq_s = a1 - a0;
        yk0 = k0;
        Lk_s = k1 - k0;
    } else if (kCausal) {
        bh = blockIdx.x % p.BH;
        qt = p.n_qtiles - 1 - blockIdx.x / p.BH;  // heavy (late) query tiles first
    } else {
        qt = blockIdx.x % p.n_qtiles;
        bh = blockIdx.x / p.n_qtiles;
    }
    const int q0 = qt * BR;
    const int yq = yq0 + q0;
    if (kPacked && q0 >= Lq_s) return;  // past the end of this sequence (uniform for the CTA)
    const int koff = Lk_s - Lq_s;        // causal offset of the diagonal
    int kend = Lk_s;                     // keys any row of this tile may see
    if (kCausal) kend = max(0, min(Lk_s, q0 + BR + koff));
    const int nk = (kend + BC - 1) / BC;
    if (MASK != 0 && nk == 0) {
        // no row of the tile sees a key: zeros and lse = -inf, no pipeline at all
        for (int r = threadIdx.x; r < BR && q0 + r < Lq_s; r += blockDim.x) {
            const size_t row = (size_t)bh * (size_t)p.Lq + (size_t)(yq + r);
            // 16-byte words per output row: 128 bf16 or 128 fp32
            constexpr int kWords = kSplit ? HD / 4 : HD / 8;
            uint4 *po = kSplit ? reinterpret_cast<uint4 *>(p.o_f32 + row * HD) : reinterpret_cast<uint4 *>(p.o_bf + row * HD);
            uint4 *pt = kSplit ? reinterpret_cast<uint4 *>(p.to_f32 + row * HD) : reinterpret_cast<uint4 *>(p.to_bf + row * HD);
            for (int u = 0; u < kWords; ++u) po[u] = pt[u] = make_uint4(0u, 0u, 0u, 0u);
            if (p.lse) p.lse[row] = -INFINITY;
            if (p.mu) p.mu[row] = 0.f;
        }
        return;
    }
    const uint64_t bound = p.bound_ns;
    // persistent (nk >= 3): unit n's staged O goes to the V-side stage of unit n + 1's
    // second key tile (G = (n + 1) * nk + 1), tO to that of its third; unit n's last
    // two tiles used those stages, and unit n + 1's first tile has the third stage
    auto stage_o = [&](int n) -> uint32_t { return SM_VT + (uint32_t)(((n + 1) * nk + 1) % VST) * VT_STAGE; };
    auto stage_t = [&](int n) -> uint32_t { return SM_VT + (uint32_t)(((n + 1) * nk + 2) % VST) * VT_STAGE; };
    // persistent: the n-th unit of this CTA (unit 0 is blockIdx.x, decoded above);
    // false past the last one, else its query tile and outer index
    auto next_unit = [&](int n, int &qt_n, int &bh_n) -> bool {
        const long long u = (long long)blockIdx.x + (long long)n * (long long)gridDim.x;
        if (u >= (long long)p.n_units) return false;
        qt_n = (int)(u % p.n_qtiles);
        bh_n = (int)(u / p.n_qtiles);
        return true;
    };

    const uint32_t bars = base + kBar;
    auto BAR = [&](int i) -> uint32_t { return bars + 8u * (uint32_t)i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + kBar + OFF_TMEM_SLOT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + kBar + OFF_ABORT);

    if (threadIdx.x == 0) {
        mbar_init(BAR(B_Q_FULL), 1);
        for (int s = 0; s < STAGES; ++s) mbar_init(BAR(B_KT_FULL + s), 1);
        for (int s = 0; s < VST; ++s) {
            mbar_init(BAR(B_VT_FULL + s), 1);
            mbar_init(BAR(B_VT_EMPTY + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(BAR(B_SD_FULL + b), 1);
            mbar_init(BAR(B_P_FULL + b), SOFTMAX_THREADS / 32);  // one arrival per softmax warp
        }
        mbar_init(BAR(B_O_FULL), 1);
        mbar_init(BAR(B_MMA_DRAIN), 1);
        mbar_init(BAR(B_OT_FREE), SOFTMAX_THREADS / 32);
        mbar_init(BAR(B_STG_FULL), SOFTMAX_THREADS / 32);
        mbar_init(BAR(B_STG_FREE), 1);
        mbar_init(BAR(B_STG_FREE + 1), 1);
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
            int kt_last[STAGES], vt_last[VST], q_last = -1;
            for (int s = 0; s < STAGES; ++s) kt_last[s] = -1;
            for (int s = 0; s < VST; ++s) vt_last[s] = -1;
            int n = 0, qt_n = qt, bh_n = bh;
            do {
                const int G0 = n * nk;  // CTA-wide index of this unit's first key tile
                const int yq_n = yq0 + qt_n * BR;
                // Q / tQ are free once every S / dS' product of the previous unit is complete
                if (n > 0 && !mbar_wait(BAR(B_SD_FULL + ((G0 - 1) & 1)), ((G0 - 1) >> 1) & 1, abort_flag, bound)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(BAR(B_Q_FULL), 4 * CHUNK_Q);
                tma_load_3d(base + SM_Q, &p.tm_q, BAR(B_Q_FULL), 0, yq_n, bh_n);
                tma_load_3d(base + SM_Q + CHUNK_Q, &p.tm_q, BAR(B_Q_FULL), 64, yq_n, bh_n);
                tma_load_3d(base + SM_TQ, &p.tm_tq, BAR(B_Q_FULL), 0, yq_n, bh_n);
                tma_load_3d(base + SM_TQ + CHUNK_Q, &p.tm_tq, BAR(B_Q_FULL), 64, yq_n, bh_n);
                q_last = n;
                // order of use by the MMA warp: KT_0, KT_1, VT_0, KT_2, VT_1, ...
                for (int t = 0; t <= nk && ok; ++t) {
                    if (t < nk) {
                        const int G = G0 + t;
                        const int s = G % STAGES;
                        // stage s is free once S/dS' of tile G - 2 are complete
                        if (!mbar_wait(BAR(B_SD_FULL + s), ((G / STAGES) & 1) ^ 1, abort_flag, bound)) {
                            ok = false;
                            break;
                        }
                        const uint32_t st = base + SM_KT + s * KT_STAGE;
                        const uint32_t fb = BAR(B_KT_FULL + s);
                        const int y = yk0 + t * BC;
                        mbar_arrive_expect_tx(fb, KT_STAGE);
                        // chunk c: K rows then tK rows, so [K | tK] is one N = 128 operand
                        tma_load_3d(st, &p.tm_k, fb, 0, y, bh_n);
                        tma_load_3d(st + CHUNK_K, &p.tm_tk, fb, 0, y, bh_n);
                        tma_load_3d(st + 2 * CHUNK_K, &p.tm_k, fb, 64, y, bh_n);
                        tma_load_3d(st + 3 * CHUNK_K, &p.tm_tk, fb, 64, y, bh_n);
                        kt_last[s] = G;
                    }
                    if (t >= 1) {
                        const int i = G0 + t - 1;
                        const int s = i % VST;
                        if (!mbar_wait(BAR(B_VT_EMPTY + s), ((i / VST) & 1) ^ 1, abort_flag, bound)) {
                            ok = false;
                            break;
                        }
                        // persistent: the previous unit's staged O sits in the stage of this
                        // unit's second V tile (stored first), tO in that of its third; the
                        // first V tile has a stage of its own and loads as soon as the ring
                        // frees it, ahead of the previous unit's epilogue
                        if (kPersist && n > 0 && (t == 2 || t == 3) &&
                            !mbar_wait(BAR(B_STG_FREE + (t - 2)), (n - 1) & 1, abort_flag, bound)) {
                            ok = false;
                            break;
                        }
                        const uint32_t st = base + SM_VT + s * VT_STAGE;
                        const uint32_t fb = BAR(B_VT_FULL + s);
                        const int y = yk0 + (t - 1) * BC;
                        mbar_arrive_expect_tx(fb, VT_STAGE);
                        // [V c0 | V c1 | tV c0 | tV c1]: N-chunks 64 columns apart (LBO)
                        tma_load_3d(st, &p.tm_v, fb, 0, y, bh_n);
                        tma_load_3d(st + CHUNK_K, &p.tm_v, fb, 64, y, bh_n);
                        tma_load_3d(st + 2 * CHUNK_K, &p.tm_tv, fb, 0, y, bh_n);
                        tma_load_3d(st + 3 * CHUNK_K, &p.tm_tv, fb, 64, y, bh_n);
                        vt_last[s] = i;
                    }
                }
            } while (kPersist && ok && next_unit(++n, qt_n, bh_n));
            // let every copy already issued land before shared memory is released
            if (q_last >= 0) mbar_wait_drain(BAR(B_Q_FULL), q_last & 1, bound);
            for (int s = 0; s < STAGES; ++s)
                if (kt_last[s] >= 0) mbar_wait_drain(BAR(B_KT_FULL + s), (kt_last[s] / STAGES) & 1, bound);
            for (int s = 0; s < VST; ++s)
                if (vt_last[s] >= 0) mbar_wait_drain(BAR(B_VT_FULL + s), (vt_last[s] / VST) & 1, bound);
        }
        __syncwarp();
    } else if (warp == 1) {
        // -------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t ID_SD = idesc_bf16_f32(128, 128, 0);  // Q [K|tK]^T
            constexpr uint32_t ID_D = idesc_bf16_f32(128, 64, 0);    // tQ K^T
            constexpr uint32_t ID_OT = idesc_bf16_f32(128, 256, 1);  // P [V|tV]
            constexpr uint32_t ID_T = idesc_bf16_f32(128, 128, 1);   // PdS V
            // K-major operands: 128-byte rows, 8-row groups 1024 B apart; V: 64-column
            // chunks CHUNK_K apart (LBO), 8-key groups 1024 B apart (SBO)
            const uint64_t dq = smem_desc_sw128(base + SM_Q, 16, 1024);
            const uint64_t dtq = smem_desc_sw128(base + SM_TQ, 16, 1024);
            const uint64_t dk0 = smem_desc_sw128(base + SM_KT, 16, 1024);
            const uint64_t dv0 = smem_desc_sw128(base + SM_VT, CHUNK_K, 1024);
            bool ok = true;
            // G: CTA-wide key-tile index (ring stage, buffer and phase)
            auto issue_sd = [&](int G) -> bool {
                const int s = G % STAGES;
                const int b = G & 1;
                if (!mbar_wait(BAR(B_KT_FULL + s), (G / STAGES) & 1, abort_flag, bound)) return false;
                tc_fence_after();
                const uint64_t dk = desc_add(dk0, s * KT_STAGE);
                const uint32_t t_s = tbase + TM_BUF + 128u * b;
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * KT_CHUNK + (kk & 3) * 32;
                    const uint32_t offq = (kk >> 2) * CHUNK_Q + (kk & 3) * 32;
                    mma_ss(t_s, desc_add(dq, offq), desc_add(dk, off), ID_SD, kk > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * KT_CHUNK + (kk & 3) * 32;
                    const uint32_t offq = (kk >> 2) * CHUNK_Q + (kk & 3) * 32;
                    mma_ss(t_s + 64, desc_add(dtq, offq), desc_add(dk, off), ID_D, 1u);
                }
                mma_commit(BAR(B_SD_FULL + b));
                return true;
            };
            // first: the unit's first tile (overwrites O / T); n: the unit
            auto issue_pv = [&](int G, bool first, int n) -> bool {
                const int s = G % VST;  // V-side stage
                const int b = G & 1;
                if (!mbar_wait(BAR(B_P_FULL + b), (G >> 1) & 1, abort_flag, bound)) return false;
                if (!mbar_wait(BAR(B_VT_FULL + s), (G / VST) & 1, abort_flag, bound)) return false;
                // the previous unit's epilogue must have read O / T before they are overwritten
                if (kPersist && first && n > 0 && !mbar_wait(BAR(B_OT_FREE), (n - 1) & 1, abort_flag, bound))
                    return false;
                tc_fence_after();
                const uint64_t dv = desc_add(dv0, s * VT_STAGE);
                const uint32_t t_s = tbase + TM_BUF + 128u * b;
#pragma unroll
                for (int kk = 0; kk < BC / 16; ++kk) {
                    // keys 16kk..16kk+15: group kk/2's columns, 8 columns per K-step
                    const uint32_t a_col = (kk >> 1) * 32 + (kk & 1) * 8;
                    mma_ts(tbase + TM_O, t_s + a_col, desc_add(dv, kk * 2048), ID_OT, (!first || kk > 0) ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < BC / 16; ++kk) {
                    const uint32_t a_col = 64 + (kk >> 1) * 32 + (kk & 1) * 8;
                    mma_ts(tbase + TM_T, t_s + a_col, desc_add(dv, kk * 2048), ID_T, 1u);
                }
                if (kSplit) {  // the lo parts sit 16 columns after the hi parts
#pragma unroll
                    for (int kk = 0; kk < BC / 16; ++kk) {
                        const uint32_t a_col = 16 + (kk >> 1) * 32 + (kk & 1) * 8;
                        mma_ts(tbase + TM_O, t_s + a_col, desc_add(dv, kk * 2048), ID_OT, 1u);
                    }
#pragma unroll
                    for (int kk = 0; kk < BC / 16; ++kk) {
                        const uint32_t a_col = 64 + 16 + (kk >> 1) * 32 + (kk & 1) * 8;
                        mma_ts(tbase + TM_T, t_s + a_col, desc_add(dv, kk * 2048), ID_T, 1u);
                    }
                }
                mma_commit(BAR(B_VT_EMPTY + s));
                return true;
            };
            // key tile t of a unit starts O / T afresh: the unit's first tile and,
            // with kSplit, each tile whose accumulators were just folded out
            auto restarts = [](int t) { return t == 0 || (kSplit && t % SPLIT_FOLD_TILES == 0); };
            int n = 0, qt_n = qt, bh_n = bh;
            do {
                const int G0 = n * nk;
                ok = mbar_wait(BAR(B_Q_FULL), n & 1, abort_flag, bound);
                if (ok) ok = issue_sd(G0);
                for (int j = 1; j < nk && ok; ++j) {
                    ok = issue_sd(G0 + j);
                    if (ok) ok = issue_pv(G0 + j - 1, restarts(j - 1), n);
                }
                if (ok) ok = issue_pv(G0 + nk - 1, restarts(nk - 1), n);
                // O and T are final once everything issued so far completes (a barrier
                // of its own: a parity wait on a per-tile barrier could be ambiguous here)
                if (ok) mma_commit(BAR(B_O_FULL));
            } while (kPersist && ok && next_unit(++n, qt_n, bh_n));
            // every MMA issued must finish before tensor memory is released
            mma_commit(BAR(B_MMA_DRAIN));
            mbar_wait_drain(BAR(B_MMA_DRAIN), 0, bound);
        }
        __syncwarp();
    } else if (kPersist && warp == 3) {
        // ------------------------------------- persistent: output tensor stores
        // each unit's O and tO, staged by the softmax warps in the V-side ring, go out
        // through the tensor-store unit; once the stores have read the staging the
        // producer may load the next unit's V tiles there
        if (lane == 0) {
            int n = 0, qt_n = qt, bh_n = bh;
            do {
                if (!mbar_wait(BAR(B_STG_FULL), n & 1, abort_flag, bound) || *abort_flag != 0) break;
                const int yq_n = yq0 + qt_n * BR;
                const uint32_t so = stage_o(n), st = stage_t(n);
                tma_store_3d(&p.tm_o, base + so, 0, yq_n, bh_n);
                tma_store_3d(&p.tm_o, base + so + CHUNK_Q, 64, yq_n, bh_n);
                tma_store_commit();
                tma_store_3d(&p.tm_to, base + st, 0, yq_n, bh_n);
                tma_store_3d(&p.tm_to, base + st + CHUNK_Q, 64, yq_n, bh_n);
                tma_store_commit();
                tma_store_wait_read_1();  // O's stage read: the next unit's first V tile may land there
                mbar_arrive(BAR(B_STG_FREE));
                tma_store_wait_read_all();
                mbar_arrive(BAR(B_STG_FREE + 1));
            } while (next_unit(++n, qt_n, bh_n));
            tma_store_wait_all();  // the last stores complete before the CTA exits
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ---------------------------------------- softmax, JVP statistics, epilogue
        const int grp = (warp - 4) >> 2;  // key columns 32*grp .. 32*grp+31 of each tile
        const int wl = warp & 3;          // TMEM lane quadrant
        const int row = wl * 32 + lane;
        const uint32_t lane_off = (uint32_t)(wl * 32) << 16;
        const uint32_t col0 = 32u * (uint32_t)grp;
        const float c = p.scale_log2;
        const float2 c2 = make_float2(c, c);
        const float2 s2 = make_float2(p.scale, p.scale);
        const bool up = c >= 0.f;  // row max of c*S is c * max(S) (min(S) for c < 0)
        const float sentinel = up ? -INFINITY : INFINITY;
        float *xch = reinterpret_cast<float *>(gbase + kXch);
        bool failed = false;
        int n = 0, qt_n = qt, bh_n = bh;
        do {
            const int G0 = n * nk;  // CTA-wide index of this unit's first key tile
            const int q0_n = qt_n * BR, yq_n = yq0 + q0_n;
            float m_ref = -INFINITY, l = 0.f, g = 0.f;
            // kSplit: the folded sums in this row's fp32 output columns 64*grp.. of O and
            // tO, to be multiplied by opend (the rescales since the last fold)
            float opend = 1.f;
            // (recomputed where used rather than kept live through the tile loop)
            auto row_ok = [&]() { return q0_n + row < Lq_s; };  // rows past the sequence are never written
            auto out_off = [&]() {
                return ((size_t)bh_n * (size_t)p.Lq + (size_t)(yq_n + row)) * HD + 64u * (uint32_t)grp;
            };
            // keys this row sees (a prefix of the sequence's keys; may be <= 0 when causal)
            const int kcount = kCausal ? min(Lk_s, q0_n + row + koff + 1) : Lk_s;

            for (int j = 0; j < nk; ++j) {
                const int G = G0 + j;  // CTA-wide tile index
                const int b = G & 1;
                const uint32_t t_s = tbase + lane_off + TM_BUF + 128u * b;
                if (!failed) failed = !mbar_wait_warp(BAR(B_SD_FULL + b), (G >> 1) & 1, abort_flag, bound);
                uint32_t xs[32], xd[32];
                const int valid = kcount - j * BC - (int)col0;  // visible keys of this group (may be <= 0)
                float part = sentinel;
                if (!failed) {
                    tc_fence_after();
                    tmem_ld32(t_s + col0, xs);
                    tmem_ld32(t_s + 64 + col0, xd);
                    tmem_wait_ld();
                    if (valid < 32) {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (i >= valid) xs[i] = __float_as_uint(sentinel);
                    }
                    float m4[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) m4[k] = __uint_as_float(xs[k]);
                    if (up) {
#pragma unroll
                        for (int i = 4; i < 28; i += 8)
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                m4[k] = fmax3(m4[k], __uint_as_float(xs[i + k]), __uint_as_float(xs[i + 4 + k]));
#pragma unroll
                        for (int k = 0; k < 4; ++k) m4[k] = fmaxf(m4[k], __uint_as_float(xs[28 + k]));
                        part = fmaxf(fmax3(m4[0], m4[1], m4[2]), m4[3]);
                    } else {
#pragma unroll
                        for (int i = 4; i < 28; i += 8)
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                m4[k] = fmin3(m4[k], __uint_as_float(xs[i + k]), __uint_as_float(xs[i + 4 + k]));
#pragma unroll
                        for (int k = 0; k < 4; ++k) m4[k] = fminf(m4[k], __uint_as_float(xs[28 + k]));
                        part = fminf(fmin3(m4[0], m4[1], m4[2]), m4[3]);
                    }
                    xch[(b * 2 + grp) * 128 + row] = part;
                }
                // both groups' partial maxima are in shared memory; every softmax
                // thread reaches this barrier each tile, and a failure anywhere
                // ends the loop for all of them together
                if (named_bar_or(NB_TILE, SOFTMAX_THREADS, failed)) {
                    failed = true;
                    break;
                }
                const float other = xch[(b * 2 + (grp ^ 1)) * 128 + row];
                const float m_tile = (up ? fmaxf(part, other) : fminf(part, other)) * c;
                if (j == 0) {
                    m_ref = m_tile;
                } else {
                    const bool need = m_tile > m_ref + RESCALE_THRESHOLD;
                    const bool fold = kSplit && j % SPLIT_FOLD_TILES == 0;  // the same for every thread
                    if (fold || __any_sync(0xffffffffu, need)) {
                        float alpha = 1.f;
                        if (need) {
                            alpha = ex2_approx(m_ref - m_tile);
                            m_ref = m_tile;
                        }
                        l *= alpha;
                        g *= alpha;
                        // O and T may only be touched once the P.V products of tile j-1
                        // are complete (the V-side barrier of its stage)
                        failed = !mbar_wait_warp(BAR(B_VT_EMPTY + (G - 1) % VST), ((G - 1) / VST) & 1, abort_flag, bound);
                        if (!failed && fold) {
                            // sums = (sums * opend + acc) * alpha over this thread's 64 O and
                            // 64 T columns (the ones its epilogue writes): the first fold
                            // stores acc * alpha, later ones add acc with fire-and-forget L2
                            // reductions unless a rescale since the last fold makes them
                            // read, scale and write the sums.  Tile j's P.V then overwrites
                            // O / T.  Each 16-column block goes through the warp's staging
                            // slot (row = lane, 16-byte unit u of row r at
                            // r*64 + ((u ^ ((r >> 1) & 3)) << 4), conflict-free both ways) and
                            // out as 8 rows x 64 contiguous bytes per instruction, the lanes
                            // taking the rows' scale factors by shuffle.
                            tc_fence_after();
                            const bool first_fold = j == SPLIT_FOLD_TILES;
                            const uint32_t slot = base + SM_STG + (uint32_t)(warp - 4) * STG_SLOT;
                            const int rows_here = Lq_s - (q0_n + wl * 32);  // rows of this warp in the sequence
                            const size_t warp_row0 = (size_t)bh_n * (size_t)p.Lq + (size_t)(yq_n + wl * 32);
#pragma unroll 1
                            for (int cc = 0; cc < 8; ++cc) {
                                const uint32_t col = 64u * (uint32_t)grp + 16u * (uint32_t)(cc & 3);
                                uint32_t r[16];
                                tmem_ld16(tbase + lane_off + (cc < 4 ? TM_O : TM_T) + col, r);
                                tmem_wait_ld();
#pragma unroll
                                for (int u = 0; u < 4; ++u)
                                    st_shared_v4(slot + (uint32_t)lane * 64u + (((uint32_t)u ^ (((uint32_t)lane >> 1) & 3u)) << 4),
                                                 r[4 * u], r[4 * u + 1], r[4 * u + 2], r[4 * u + 3]);
                                __syncwarp();
                                float *dst0 = (cc < 4 ? p.o_f32 : p.to_f32) + col;
#pragma unroll
                                for (int k = 0; k < 4; ++k) {
                                    const int rr = 8 * k + (lane >> 2);  // this lane's row of the warp
                                    const uint32_t u = (uint32_t)lane & 3u;
                                    const float a_r = __shfl_sync(0xffffffffu, alpha, rr);
                                    const float o_r = __shfl_sync(0xffffffffu, opend, rr);
                                    const float4 v = ld_shared_f4(slot + (uint32_t)rr * 64u + ((u ^ (((uint32_t)rr >> 1) & 3u)) << 4));
                                    if (rr >= rows_here) continue;  // past the sequence: never written
                                    float *d = dst0 + (warp_row0 + (size_t)rr) * HD + 4u * u;
                                    if (first_fold) {
                                        *reinterpret_cast<float4 *>(d) = make_float4(v.x * a_r, v.y * a_r, v.z * a_r, v.w * a_r);
                                    } else if (o_r == 1.f && a_r == 1.f) {
                                        red_add_f32x4(d, v.x, v.y, v.z, v.w);
                                    } else {
                                        const float4 w = __ldcg(reinterpret_cast<const float4 *>(d));
                                        *reinterpret_cast<float4 *>(d) =
                                            make_float4(fmaf(w.x, o_r, v.x) * a_r, fmaf(w.y, o_r, v.y) * a_r,
                                                        fmaf(w.z, o_r, v.z) * a_r, fmaf(w.w, o_r, v.w) * a_r);
                                    }
                                }
                                __syncwarp();  // the slot is free again
                            }
                            opend = 1.f;
                        } else if (!failed) {
                            // group 0 rescales O, group 1 rescales T
                            tc_fence_after();
#pragma unroll 1
                            for (int cc = 0; cc < 4; ++cc) {
                                uint32_t r[32];
                                const uint32_t ta = tbase + lane_off + 128u * (uint32_t)grp + 32u * cc;
                                tmem_ld32(ta, r);
                                tmem_wait_ld();
#pragma unroll
                                for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                                tmem_st32(ta, r);
                            }
                            if (kSplit) opend *= alpha;
                        }
                    }
                }
                if (failed) continue;  // the next tile's barrier carries the failure to everyone
                const float2 nm2 = make_float2(-m_ref, -m_ref);
                float pv[32];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float2 y =
                        __ffma2_rn(make_float2(__uint_as_float(xs[2 * i]), __uint_as_float(xs[2 * i + 1])), c2, nm2);
                    pv[2 * i] = ex2_approx(y.x);
                    pv[2 * i + 1] = ex2_approx(y.y);
                }
                if (valid < 32) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (i >= valid) pv[i] = 0.f;
                }
                float2 ls2a = make_float2(0.f, 0.f), ls2b = ls2a, gs2a = ls2a, gs2b = ls2a;
                uint32_t pk[16], pd[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float2 pp = make_float2(pv[2 * i], pv[2 * i + 1]);
                    const float2 dd = make_float2(__uint_as_float(xd[2 * i]), __uint_as_float(xd[2 * i + 1]));
                    const float2 t = __fmul2_rn(__fmul2_rn(pp, dd), s2);  // p * s dS'
                    if (i & 1) {
                        ls2b = __fadd2_rn(ls2b, pp);
                        gs2b = __fadd2_rn(gs2b, t);
                    } else {
                        ls2a = __fadd2_rn(ls2a, pp);
                        gs2a = __fadd2_rn(gs2a, t);
                    }
                    pk[i] = pack_bf16x2(pp.x, pp.y);
                    pd[i] = pack_bf16x2(t.x, t.y);
                }
                tmem_st16(t_s + col0, pk);       // P over this group's S columns
                tmem_st16(t_s + 64 + col0, pd);  // P.*s dS' over this group's dS' columns
                if (kSplit) {
                    // lo = x - hi, rounded to bf16: hi + lo carries ~16 significant bits
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float2 pp = make_float2(pv[2 * i], pv[2 * i + 1]);
                        const float2 dd = make_float2(__uint_as_float(xd[2 * i]), __uint_as_float(xd[2 * i + 1]));
                        const float2 t = __fmul2_rn(__fmul2_rn(pp, dd), s2);
                        const uint32_t ph = pack_bf16x2(pp.x, pp.y), th = pack_bf16x2(t.x, t.y);
                        pk[i] = pack_bf16x2(pp.x - __uint_as_float(ph << 16), pp.y - __uint_as_float(ph & 0xffff0000u));
                        pd[i] = pack_bf16x2(t.x - __uint_as_float(th << 16), t.y - __uint_as_float(th & 0xffff0000u));
                    }
                    tmem_st16(t_s + col0 + 16, pk);
                    tmem_st16(t_s + 64 + col0 + 16, pd);
                }
                l += (ls2a.x + ls2b.x) + (ls2a.y + ls2b.y);
                g += (gs2a.x + gs2b.x) + (gs2a.y + gs2b.y);
                tmem_wait_st();
                warp_arrive_after_tc(BAR(B_P_FULL + b));
            }

            if (!failed) failed = !mbar_wait_warp(BAR(B_O_FULL), n & 1, abort_flag, bound);
            // [l, g][group][row]; the persistent form reuses the per-tile maxima area, whose
            // last reads (the unit's last tile) precede every P arrival and so O_FULL
            float *lg = kPersist ? xch : xch + 2 * 2 * 128;
            if (!failed) {
                lg[(0 * 2 + grp) * 128 + row] = l;
                lg[(1 * 2 + grp) * 128 + row] = g;
            }
            const bool any_failed = named_bar_or(NB_EPI, SOFTMAX_THREADS, failed);
            if (!any_failed) {
                tc_fence_after();
                const float lt = l + lg[(0 * 2 + (grp ^ 1)) * 128 + row];
                const float gt = g + lg[(1 * 2 + (grp ^ 1)) * 128 + row];
                // persistent: every thread has read the other group's l, g before the next
                // unit's first tile writes its maxima over them
                if (kPersist) named_bar_sync(NB_EPI, SOFTMAX_THREADS);
                // a row that saw no key (masks only) has lt = 0: zeros, lse = -inf
                const float inv_l = (MASK != 0 && !(lt > 0.f)) ? 0.f : 1.f / lt;
                const float mu = gt * inv_l;
                // group grp writes output columns 64*grp .. 64*grp+63
                if (kSplit) {
                    // fp32 outputs straight from registers, 16 bytes per store
                    // (packed: rows past the sequence belong to the next one and are not written);
                    // after folds the row's sums so far sit in the same output words
                    const bool folded = nk > SPLIT_FOLD_TILES;
#pragma unroll 1
                    for (int h = 0; h < 4; ++h) {  // 16 output columns at a time
                        const uint32_t col = 64u * (uint32_t)grp + 16u * (uint32_t)h;
                        float4 *po = reinterpret_cast<float4 *>(p.o_f32 + out_off() + 16 * h);
                        float4 *pt = reinterpret_cast<float4 *>(p.to_f32 + out_off() + 16 * h);
                        float4 so[4], st[4];
                        if (folded && row_ok()) {
#pragma unroll
                            for (int u = 0; u < 4; ++u) {  // (the folds' L2 reductions included)
                                so[u] = __ldcg(po + u);
                                st[u] = __ldcg(pt + u);
                            }
                        }
                        uint32_t ro[16], rt[16];
                        tmem_ld16(tbase + lane_off + TM_O + col, ro);
                        tmem_ld16(tbase + lane_off + TM_T + col, rt);
                        tmem_wait_ld();
                        if (row_ok()) {
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                float ao[4] = {__uint_as_float(ro[4 * u]), __uint_as_float(ro[4 * u + 1]),
                                               __uint_as_float(ro[4 * u + 2]), __uint_as_float(ro[4 * u + 3])};
                                float at[4] = {__uint_as_float(rt[4 * u]), __uint_as_float(rt[4 * u + 1]),
                                               __uint_as_float(rt[4 * u + 2]), __uint_as_float(rt[4 * u + 3])};
                                if (folded) {
                                    const float fo[4] = {so[u].x, so[u].y, so[u].z, so[u].w};
                                    const float ft[4] = {st[u].x, st[u].y, st[u].z, st[u].w};
#pragma unroll
                                    for (int e = 0; e < 4; ++e) {
                                        ao[e] = fmaf(fo[e], opend, ao[e]);
                                        at[e] = fmaf(ft[e], opend, at[e]);
                                    }
                                }
                                float o4[4], t4[4];
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    o4[e] = ao[e] * inv_l;
                                    t4[e] = fmaf(-mu, o4[e], at[e] * inv_l);
                                }
                                po[u] = make_float4(o4[0], o4[1], o4[2], o4[3]);
                                pt[u] = make_float4(t4[0], t4[1], t4[2], t4[3]);
                            }
                        }
                    }
                }
                // bf16 outputs: O into the Q tile's shared memory, tO into tQ's, in
                // the 128-byte-swizzled layout of the store tensor maps (packed rows and
                // the persistent form: plain stores from registers)
#pragma unroll 1
                for (int h = 0; h < (kSplit ? 0 : 2); ++h) {
                    const int pc = 2 * grp + h;
                    uint32_t ro[32], rt[32];
                    tmem_ld32(tbase + lane_off + TM_O + 32u * pc, ro);
                    tmem_ld32(tbase + lane_off + TM_T + 32u * pc, rt);
                    tmem_wait_ld();
                    if (kPersist && h == 1)  // O / T read: the next unit may overwrite them
                        warp_arrive_after_tc(BAR(B_OT_FREE));
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
                    if (kPacked) {
                        // plain stores, staged per warp (rows past the sequence belong to
                        // the next one and are not written)
                        const size_t off =
                            ((size_t)bh_n * (size_t)p.Lq + (size_t)(yq_n + wl * 32)) * HD + 64u * grp + 32u * h;
                        const int rows_left = Lq_s - (q0_n + wl * 32);
                        const uint32_t slot = base + SM_STG + (uint32_t)(warp - 4) * STG_SLOT;
                        store_rows_32x32(slot, wo, p.o_bf + off, rows_left, (uint32_t)lane);
                        store_rows_32x32(slot, wt, p.to_bf + off, rows_left, (uint32_t)lane);
                        continue;
                    }
                    // staging in the store maps' 128-byte-swizzled layout: Q / tQ shared
                    // memory (persistent form: the V-side ring, O in stage 0, tO in stage 1)
                    const uint32_t chunk_off = (uint32_t)grp * CHUNK_Q + (uint32_t)row * 128u;
                    const uint32_t unit0 = (uint32_t)h * 4u;
                    const uint32_t so = kPersist ? stage_o(n) : SM_Q;
                    const uint32_t st = kPersist ? stage_t(n) : SM_TQ;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint32_t phys = (((unit0 + u) ^ (uint32_t)(row & 7)) * 16u);
                        st_shared_v4(base + so + chunk_off + phys, wo[4 * u], wo[4 * u + 1], wo[4 * u + 2],
                                     wo[4 * u + 3]);
                        st_shared_v4(base + st + chunk_off + phys, wt[4 * u], wt[4 * u + 1], wt[4 * u + 2],
                                     wt[4 * u + 3]);
                    }
                }
                if (grp == 0 && p.lse != nullptr && q0_n + row < Lq_s) {
                    p.lse[(size_t)bh_n * (size_t)p.Lq + (size_t)(yq_n + row)] =
                        (MASK != 0 && !(lt > 0.f)) ? -INFINITY : (m_ref + __log2f(lt)) * 0.69314718055994531f;
                }
                if (grp == 1 && p.mu != nullptr && q0_n + row < Lq_s)
                    p.mu[(size_t)bh_n * (size_t)p.Lq + (size_t)(yq_n + row)] = mu;
            }
            if (kPersist) {
                // staging complete: one arrival per warp for the storing warp
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && !any_failed) mbar_arrive(BAR(B_STG_FULL));
            } else {
                fence_proxy_async_smem();
                named_bar_sync(NB_EPI, SOFTMAX_THREADS);  // staging complete (every softmax thread gets here)
                if (!kSplit && !kPacked && warp == 4 && lane == 0 && !any_failed && *abort_flag == 0) {
                    tma_store_3d(&p.tm_o, base + SM_Q, 0, yq_n, bh_n);
                    tma_store_3d(&p.tm_o, base + SM_Q + CHUNK_Q, 64, yq_n, bh_n);
                    tma_store_3d(&p.tm_to, base + SM_TQ, 0, yq_n, bh_n);
                    tma_store_3d(&p.tm_to, base + SM_TQ + CHUNK_Q, 64, yq_n, bh_n);
                    tma_store_commit();
                    tma_store_wait_all();
                }
            }
            if (any_failed) break;  // uniform: an OR over every softmax thread
        } while (kPersist && next_unit(++n, qt_n, bh_n));
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
