// api.cu -- C ABI of the attention + JVP forward library (see
// include/attn_jvp.h for the contract of every entry point).
//
// Host side only: argument checks, tensor-map encoding, launch on the
// caller's stream, error mapping.  No device memory is allocated here.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <initializer_list>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "attn_jvp.h"
#include "jvp_bwd_sm100.cuh"
#include "jvp_f32.cuh"
#include "jvp_sm100.cuh"

namespace {

constexpr int kVersion = 100;  // 0.1.0
constexpr uint64_t kDefaultBoundNs = 2000000000ull;
constexpr int kMaxDevices = 64;

thread_local int t_last_cuda_error = 0;
std::atomic<uint64_t> g_bound_ns{kDefaultBoundNs};

// per-device one-time set-up: capability check and kernel attributes
struct DeviceState {
    std::once_flag once;
    int status = AJVP_OK;
    int cuda_error = 0;
    int sm_count = 0;
};
DeviceState g_dev[kMaxDevices];

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
std::once_flag g_encode_once;
EncodeTiledFn g_encode = nullptr;

int fail_cuda(cudaError_t e) {
    t_last_cuda_error = (int)e;
    return AJVP_ERR_CUDA;
}

// Short key sequences (at most this many 64-key tiles) take the persistent
// form of the unmasked bf16 kernel: with few key tiles per query tile, the
// per-tile pipeline fill, drain and epilogue are a large share of a CTA's
// time, and the persistent CTA overlaps them with the next tile's work.
constexpr int64_t kDefaultPersistKeyTiles = 32;
std::atomic<int64_t> g_persist_key_tiles{kDefaultPersistKeyTiles};

// The unmasked, unsplit dQ and dK kernels run as CTA pairs (cta_group::2)
// when this is set.  Off by default: on B200 the pairs measured 4-5 % slower
// than single CTAs for both kernels.
std::atomic<int> g_bwd_pairs{0};

template <bool kSplit, int MASK, bool kPersist = false>
cudaError_t set_fwd_smem() {
    return cudaFuncSetAttribute(ajvp::sm100::attn_jvp_fwd_kernel<kSplit, MASK, kPersist>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)(kPersist ? ajvp::sm100::SMEM_BYTES_P : ajvp::sm100::SMEM_BYTES));
}

template <int VAR, int MASK>
cudaError_t set_bwd_smem_one() {
    return cudaFuncSetAttribute(ajvp::bwd::attn_jvp_bwd_kernel<VAR, MASK>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ajvp::bwd::Var<VAR>::SMEM_BYTES);
}

// every mask instantiation (none, causal, packed, both) of one variant, and
// the pair form of the dQ / dK variants
template <int VAR>
cudaError_t set_bwd_smem() {
    cudaError_t e = set_bwd_smem_one<VAR, 0>();
    if constexpr (VAR != ajvp::bwd::V_V) {
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(ajvp::bwd::attn_jvp_bwd_kernel_pair<VAR>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)ajvp::bwd::Var<VAR, true>::SMEM_BYTES);
    }
    if (e == cudaSuccess) e = set_bwd_smem_one<VAR, 1>();
    if (e == cudaSuccess) e = set_bwd_smem_one<VAR, 2>();
    if (e == cudaSuccess) e = set_bwd_smem_one<VAR, 3>();
    if constexpr (VAR != ajvp::bwd::V_Q) {  // the key-side variants' split form
        if (e == cudaSuccess) e = set_bwd_smem_one<VAR, ajvp::bwd::MASK_SPLIT>();
    }
    return e;
}

int device_setup(int *dev_out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail_cuda(e);
    if (dev < 0 || dev >= kMaxDevices) return AJVP_ERR_UNSUPPORTED_DEVICE;
    DeviceState &st = g_dev[dev];
    std::call_once(st.once, [&]() {
        int major = 0, minor = 0;
        cudaError_t e1 = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaError_t e2 = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        if (e1 != cudaSuccess || e2 != cudaSuccess) {
            st.status = AJVP_ERR_CUDA;
            st.cuda_error = (int)(e1 != cudaSuccess ? e1 : e2);
            return;
        }
        if (major != 10 || minor != 0) {
            st.status = AJVP_ERR_UNSUPPORTED_DEVICE;
            return;
        }
        cudaError_t e0 = cudaDeviceGetAttribute(&st.sm_count, cudaDevAttrMultiProcessorCount, dev);
        if (e0 != cudaSuccess || st.sm_count < 1) {
            st.status = AJVP_ERR_CUDA;
            st.cuda_error = (int)e0;
            return;
        }
        cudaError_t e3 = cudaFuncSetAttribute(ajvp::sm100::attn_jvp_fwd_kernel<false>,
                                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              (int)ajvp::sm100::SMEM_BYTES);
        if (e3 == cudaSuccess)
            e3 = cudaFuncSetAttribute(ajvp::sm100::attn_jvp_fwd_kernel<true>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ajvp::sm100::SMEM_BYTES);
        if (e3 == cudaSuccess) e3 = set_fwd_smem<false, 0, true>();
        if (e3 == cudaSuccess) e3 = set_fwd_smem<false, 1>();
        if (e3 == cudaSuccess) e3 = set_fwd_smem<false, 2>();
        if (e3 == cudaSuccess) e3 = set_fwd_smem<false, 3>();
        if (e3 == cudaSuccess) e3 = set_fwd_smem<true, 1>();
        if (e3 == cudaSuccess) e3 = set_fwd_smem<true, 2>();
        if (e3 == cudaSuccess) e3 = set_fwd_smem<true, 3>();
        if (e3 == cudaSuccess) e3 = set_bwd_smem<ajvp::bwd::V_Q>();
        if (e3 == cudaSuccess) e3 = set_bwd_smem<ajvp::bwd::V_K>();
        if (e3 == cudaSuccess) e3 = set_bwd_smem<ajvp::bwd::V_V>();
        cudaError_t e4 = cudaFuncSetAttribute(ajvp::f32::attn_jvp_fwd_f32_kernel,
                                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              (int)ajvp::f32::smem_bytes(ajvp::f32::DMAX));
        if (e3 != cudaSuccess || e4 != cudaSuccess) {
            st.status = AJVP_ERR_CUDA;
            st.cuda_error = (int)(e3 != cudaSuccess ? e3 : e4);
        }
    });
    if (st.status == AJVP_ERR_CUDA) t_last_cuda_error = st.cuda_error;
    *dev_out = dev;
    return st.status;
}

int get_encoder() {
    std::call_once(g_encode_once, []() {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    });
    return g_encode ? AJVP_OK : AJVP_ERR_CUDA;
}

// [BH][L][d] bf16 tensor, boxes of 64 columns x box_rows rows, 128-byte swizzle
int encode_3d(CUtensorMap *m, const void *ptr, int64_t d, int64_t L, int64_t BH, uint32_t box_rows) {
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)L, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)(d * 2), (cuuint64_t)(L * d * 2)};
    cuuint32_t box[3] = {64u, box_rows, 1u};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        t_last_cuda_error = (int)r;
        return AJVP_ERR_CUDA;
    }
    return AJVP_OK;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Checks shared by both entry points; sets *noop when there is nothing to do.
int check_common(const void *q, const void *k, const void *v, const void *tq, const void *tk, const void *tv,
                 const void *o, const void *to, int64_t B, int64_t H, int64_t Lq, int64_t Lk, int64_t d,
                 float scale, bool *noop) {
    *noop = false;
    if (B < 0 || H < 0 || Lq < 0 || Lk < 1 || d < 1) return AJVP_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return AJVP_ERR_INVALID_ARG;
    if (B == 0 || H == 0 || Lq == 0) {
        *noop = true;
        return AJVP_OK;
    }
    if (!q || !k || !v || !tq || !tk || !tv || !o || !to) return AJVP_ERR_INVALID_ARG;
    if (Lq >= (int64_t(1) << 31) || Lk >= (int64_t(1) << 31) || B * H >= (int64_t(1) << 31))
        return AJVP_ERR_TOO_LARGE;
    return AJVP_OK;
}

// Shared host path of the tensor-core forward entry points (kSplit: fp32
// outputs, split-bf16 probability operands; MASK: causal and/or packed
// sequences -- packed calls pass B = 1, H, the total row counts as Lq, Lk and
// the sequence offsets).
template <bool kSplit, int MASK = 0>
int launch_sm100(const void *q, const void *k, const void *v, const void *tq, const void *tk, const void *tv,
                 void *o, void *to, float *lse, int64_t B, int64_t H, int64_t Lq, int64_t Lk, int64_t d,
                 float scale, void *stream, float *mu = nullptr, const int *cu_q = nullptr,
                 const int *cu_k = nullptr, int64_t n_seq = 0, int64_t max_qtiles = 0) {
    constexpr bool kPacked = (MASK & ajvp::sm100::MASK_PACKED) != 0;
    bool noop = false;
    int rc = check_common(q, k, v, tq, tk, tv, o, to, B, H, Lq, Lk, d, scale, &noop);
    if (rc != AJVP_OK || noop) return rc;
    if (d != ajvp::sm100::HD) return AJVP_ERR_UNSUPPORTED_DIM;
    const void *ptrs[10] = {q, k, v, tq, tk, tv, o, to, lse, mu};
    for (int i = 0; i < 10; ++i)
        if (ptrs[i] && !aligned(ptrs[i], 16)) return AJVP_ERR_MISALIGNED;
    const int64_t BH = B * H;
    const int64_t n_qtiles = kPacked ? max_qtiles : (Lq + ajvp::sm100::BR - 1) / ajvp::sm100::BR;
    const int64_t n_cta = n_qtiles * BH * (kPacked ? n_seq : 1);
    if (n_cta >= (int64_t(1) << 31)) return AJVP_ERR_TOO_LARGE;
    if (n_cta == 0) return AJVP_OK;

    int dev = 0;
    rc = device_setup(&dev);
    if (rc != AJVP_OK) return rc;

    rc = get_encoder();
    if (rc != AJVP_OK) return rc;

    ajvp::sm100::Params p;
    std::memset(&p, 0, sizeof(p));
    if ((rc = encode_3d(&p.tm_q, q, d, Lq, BH, 128)) != AJVP_OK) return rc;
    if ((rc = encode_3d(&p.tm_tq, tq, d, Lq, BH, 128)) != AJVP_OK) return rc;
    if ((rc = encode_3d(&p.tm_k, k, d, Lk, BH, 64)) != AJVP_OK) return rc;
    if ((rc = encode_3d(&p.tm_tk, tk, d, Lk, BH, 64)) != AJVP_OK) return rc;
    if ((rc = encode_3d(&p.tm_v, v, d, Lk, BH, 64)) != AJVP_OK) return rc;
    if ((rc = encode_3d(&p.tm_tv, tv, d, Lk, BH, 64)) != AJVP_OK) return rc;
    if (kSplit) {
        p.o_f32 = static_cast<float *>(o);
        p.to_f32 = static_cast<float *>(to);
    } else {
        if ((rc = encode_3d(&p.tm_o, o, d, Lq, BH, 128)) != AJVP_OK) return rc;
        if ((rc = encode_3d(&p.tm_to, to, d, Lq, BH, 128)) != AJVP_OK) return rc;
    }
    p.lse = lse;
    p.mu = mu;
    if (!kSplit) {
        p.o_bf = static_cast<__nv_bfloat16 *>(o);
        p.to_bf = static_cast<__nv_bfloat16 *>(to);
    }
    p.cu_q = cu_q;
    p.cu_k = cu_k;
    p.n_seq = (int)n_seq;
    p.BH = (int)BH;
    p.Lq = (int)Lq;
    p.Lk = (int)Lk;
    p.n_qtiles = (int)n_qtiles;
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.bound_ns = g_bound_ns.load();
    p.n_units = (int)n_cta;

    const int sm_count = g_dev[dev].sm_count;
    const int64_t nk = (Lk + ajvp::sm100::BC - 1) / ajvp::sm100::BC;
    if (!kSplit && MASK == 0 && nk >= 3 && nk <= g_persist_key_tiles.load() && n_cta > sm_count) {
        // one CTA per SM walks the query tiles (its V-side ring keeps the next tile's first
        // V tile clear of the staged outputs for units of at least three key tiles)
        ajvp::sm100::attn_jvp_fwd_kernel<false, 0, true><<<(unsigned)sm_count, ajvp::sm100::NTHREADS,
                                                          ajvp::sm100::SMEM_BYTES_P, (cudaStream_t)stream>>>(p);
    } else {
        ajvp::sm100::attn_jvp_fwd_kernel<kSplit, MASK><<<(unsigned)n_cta, ajvp::sm100::NTHREADS,
                                                         ajvp::sm100::SMEM_BYTES, (cudaStream_t)stream>>>(p);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail_cuda(e);
    return AJVP_OK;
}

// ---------------------------------------------------------------- backward
// Row statistics {lse log2(e), mu, a, D} per query row, plus BN rows of
// padding that the streamed statistics copies of the last tile may read.
uint64_t bwd_stats_bytes(int64_t BH, int64_t Lq) {
    return ((uint64_t)(BH * Lq + ajvp::bwd::BN) * 16u + 255u) / 256u * 256u;
}

// Packed sequences of a backward call (MASK_PACKED): device offsets of the
// query and key rows of each sequence, and the longest sequences (grid size).
struct BwdPack {
    const int *cu_q = nullptr, *cu_k = nullptr;
    int64_t n_seq = 0, max_q = 0, max_k = 0;
};

// Parts of the streamed range for the unmasked key-side kernels.  When their
// 128-key tiles alone give fewer than four CTAs per SM (short key sequences,
// as in cross-attention to a few hundred text tokens), the 64-query tiles are
// cut into s parts (1 <= s <= 16), one CTA each, with s minimising a wave
// model of the run time: ceil(ctas * s / SMs) waves, each as long as one
// part's query tiles plus a fixed cost of about eight tiles per CTA (resident
// loads, pipeline fill and drain, epilogue), times 1 + s / 100 for the
// partial sums' traffic and their reduction.  On B200, over key sides of 96
// to 640 CTAs and s = 1 .. 16, the model's choice was the fastest measured or
// within 1 % of it.  For a given part length the smallest s wins, so no part
// is ever empty (the kernels still handle one).
int64_t bwd_key_split(int64_t BH, int64_t Lq, int64_t Lk, int sm_count) {
    const int64_t ctas = (Lk + ajvp::bwd::BM - 1) / ajvp::bwd::BM * BH;
    const int64_t tiles = (Lq + ajvp::bwd::BN - 1) / ajvp::bwd::BN;
    if (ctas <= 0 || tiles <= 1 || sm_count <= 0 || ctas >= 4 * (int64_t)sm_count) return 1;
    int64_t best = 1;
    double best_t = 0.0;
    for (int64_t s = 1; s <= 16 && s <= tiles; ++s) {
        const int64_t chunk = (tiles + s - 1) / s;
        const int64_t waves = (ctas * s + sm_count - 1) / sm_count;
        const double t = (double)waves * (double)(chunk + 8) * (1.0 + 0.01 * (double)s);
        if (s == 1 || t < best_t) {
            best = s;
            best_t = t;
        }
    }
    return best;
}

// fp32 partial sums of one split key-side kernel: [parts][B*H][Lk][2][128]
// (the dK/dtK and dV/dtV kernels each get a region of this size, after the
// row statistics, so that the two steps stay independent of each other)
uint64_t bwd_partial_bytes(int64_t BH, int64_t Lk, int64_t parts) {
    if (parts <= 1) return 0;
    return ((uint64_t)parts * (uint64_t)(BH * Lk) * 2u * ajvp::bwd::HD * 4u + 255u) / 256u * 256u;
}

// One backward variant: resident tensors r (row side, Lrow rows), streamed
// tensors l (the long ring) and sh (the short stage), Lcol rows; outputs
// out[] (Lrow rows) scaled by sc[]; MASK: causal and/or packed (cu_row /
// cu_col the row-side / streamed offsets, max_row the longest row-side run).
template <int VAR, int MASK>
int launch_bwd_var(std::initializer_list<const void *> r, std::initializer_list<const void *> l,
                   std::initializer_list<const void *> sh, std::initializer_list<void *> out,
                   std::initializer_list<float> sc, const void *stats, int64_t BH, int64_t Lrow, int64_t Lcol,
                   int64_t Lq, int64_t d, float scale, cudaStream_t stream, const int *cu_row, const int *cu_col,
                   int64_t n_seq, int64_t max_row, int64_t n_split = 1, float *partial = nullptr) {
    using namespace ajvp::bwd;
    constexpr bool kPacked = (MASK & MASK_PACKED) != 0;
    // CTA pairs: the unmasked dQ / dK kernels, an even number of row tiles per head
    const bool pair = MASK == 0 && VAR != V_V && g_bwd_pairs.load() != 0;
    int64_t n_rtiles = ((kPacked ? max_row : Lrow) + BM - 1) / BM;
    if (pair) n_rtiles = (n_rtiles + 1) / 2 * 2;
    const int64_t n_cta = n_rtiles * BH * (kPacked ? n_seq : 1) * n_split;
    if (n_cta >= (int64_t(1) << 31)) return AJVP_ERR_TOO_LARGE;
    if (n_cta == 0) return AJVP_OK;
    int rc;
    Params p;
    std::memset(&p, 0, sizeof(p));
    int i = 0;
    for (const void *x : r)
        if ((rc = encode_3d(&p.tm_r[i++], x, d, Lrow, BH, 128)) != AJVP_OK) return rc;
    i = 0;
    for (const void *x : l)
        if ((rc = encode_3d(&p.tm_l[i++], x, d, Lcol, BH, 64)) != AJVP_OK) return rc;
    i = 0;
    for (const void *x : sh)
        if ((rc = encode_3d(&p.tm_s[i++], x, d, Lcol, BH, 64)) != AJVP_OK) return rc;
    i = 0;
    for (void *x : out)
        if ((rc = encode_3d(&p.tm_out[i++], x, d, Lrow, BH, 128)) != AJVP_OK) return rc;
    if (pair) {  // the first streamed tensor of each ring in boxes of 32 rows
        if ((rc = encode_3d(&p.tm_l32, *l.begin(), d, Lcol, BH, 32)) != AJVP_OK) return rc;
        if ((rc = encode_3d(&p.tm_s32, *sh.begin(), d, Lcol, BH, 32)) != AJVP_OK) return rc;
    }
    i = 0;
    for (void *x : out) p.out[i++] = static_cast<__nv_bfloat16 *>(x);
    i = 0;
    for (float f : sc) p.out_scale[i++] = f;
    p.BH = (int)BH;
    p.n_seq = (int)n_seq;
    p.cu_row = cu_row;
    p.cu_col = cu_col;
    p.n_split = (int)n_split;
    p.partial = partial;
    p.stats = static_cast<const float4 *>(stats);
    p.Lrow = (int)Lrow;
    p.Lcol = (int)Lcol;
    p.Lq = (int)Lq;
    p.n_rtiles = (int)n_rtiles;
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.bound_ns = g_bound_ns.load();
    if constexpr (MASK == 0 && VAR != V_V) {
        if (pair)
            attn_jvp_bwd_kernel_pair<VAR><<<(unsigned)n_cta, NTHREADS, Var<VAR, true>::SMEM_BYTES, stream>>>(p);
        else
            attn_jvp_bwd_kernel<VAR, MASK><<<(unsigned)n_cta, NTHREADS, Var<VAR>::SMEM_BYTES, stream>>>(p);
    } else {
        attn_jvp_bwd_kernel<VAR, MASK><<<(unsigned)n_cta, NTHREADS, Var<VAR>::SMEM_BYTES, stream>>>(p);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail_cuda(e);
    return AJVP_OK;
}

// launch_bwd_var with the mask chosen at run time
template <int VAR>
int launch_bwd_mask(int mask, std::initializer_list<const void *> r, std::initializer_list<const void *> l,
                    std::initializer_list<const void *> sh, std::initializer_list<void *> out,
                    std::initializer_list<float> sc, const void *stats, int64_t BH, int64_t Lrow, int64_t Lcol,
                    int64_t Lq, int64_t d, float scale, cudaStream_t stream, const int *cu_row, const int *cu_col,
                    int64_t n_seq, int64_t max_row) {
    switch (mask) {
        case 0: return launch_bwd_var<VAR, 0>(r, l, sh, out, sc, stats, BH, Lrow, Lcol, Lq, d, scale, stream,
                                              cu_row, cu_col, n_seq, max_row);
        case 1: return launch_bwd_var<VAR, 1>(r, l, sh, out, sc, stats, BH, Lrow, Lcol, Lq, d, scale, stream,
                                              cu_row, cu_col, n_seq, max_row);
        case 2: return launch_bwd_var<VAR, 2>(r, l, sh, out, sc, stats, BH, Lrow, Lcol, Lq, d, scale, stream,
                                              cu_row, cu_col, n_seq, max_row);
        default: return launch_bwd_var<VAR, 3>(r, l, sh, out, sc, stats, BH, Lrow, Lcol, Lq, d, scale, stream,
                                               cu_row, cu_col, n_seq, max_row);
    }
}

// An unmasked key-side variant with its streamed range cut into n_split parts:
// the kernel writes fp32 partial sums, the reduction adds them up (in part
// order) into the two bf16 outputs.
template <int VAR>
int launch_bwd_split(std::initializer_list<const void *> r, std::initializer_list<const void *> l,
                     std::initializer_list<const void *> sh, void *out0, void *out1, float s0, float s1,
                     const void *stats, int64_t BH, int64_t Lrow, int64_t Lcol, int64_t Lq, int64_t d, float scale,
                     cudaStream_t stream, int64_t n_split, float *partial) {
    int rc = launch_bwd_var<VAR, ajvp::bwd::MASK_SPLIT>(r, l, sh, {out0, out1}, {s0, s1}, stats, BH, Lrow, Lcol, Lq,
                                                        d, scale, stream, nullptr, nullptr, 0, 0, n_split, partial);
    if (rc != AJVP_OK) return rc;
    const long long rows = (long long)(BH * Lrow);
    const long long n4 = rows * 2 * (ajvp::bwd::HD / 4);
    const unsigned grid = (unsigned)std::min<long long>((n4 + 255) / 256, 148LL * 16);
    ajvp::bwd::bwd_split_reduce_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const float4 *>(partial),
                                                                  (int)n_split, rows,
                                                                  static_cast<__nv_bfloat16 *>(out0),
                                                                  static_cast<__nv_bfloat16 *>(out1), s0, s1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail_cuda(e);
    return AJVP_OK;
}

// ---------------------------------------------------------- host pipeline
// One staging buffer holds, for `nh` (batch, head) slabs, the six bf16 inputs,
// the two bf16 outputs and lse, each array 256-byte aligned.
constexpr uint64_t kStageAlign = 256;
uint64_t round_up(uint64_t x) { return (x + kStageAlign - 1) / kStageAlign * kStageAlign; }

struct StageLayout {
    uint64_t q, tq, k, v, tk, tv, o, to, lse, bytes;  // offsets inside one buffer
};

StageLayout stage_layout(int64_t Lq, int64_t Lk, int64_t d, int64_t nh) {
    StageLayout s;
    const uint64_t qb = round_up((uint64_t)(nh * Lq * d * 2)), kb = round_up((uint64_t)(nh * Lk * d * 2));
    const uint64_t lb = round_up((uint64_t)(nh * Lq * 4));
    s.q = 0;
    s.tq = s.q + qb;
    s.k = s.tq + qb;
    s.v = s.k + kb;
    s.tk = s.v + kb;
    s.tv = s.tk + kb;
    s.o = s.tv + kb;
    s.to = s.o + qb;
    s.lse = s.to + qb;
    s.bytes = s.lse + lb;
    return s;
}

// The backward's staging buffer for `nh` slabs: its twelve inputs (q, tq, o,
// to, dout, dtout with Lq rows; k, v, tk, tv with Lk rows; lse, mu), its six
// gradients (dq, dtq; dk, dv, dtk, dtv) and the row-statistics workspace.
struct BwdStageLayout {
    uint64_t in[12], out[6], stats, stats_bytes, bytes;
};

BwdStageLayout bwd_stage_layout(int64_t Lq, int64_t Lk, int64_t d, int64_t nh) {
    BwdStageLayout s;
    const uint64_t qb = round_up((uint64_t)(nh * Lq * d * 2)), kb = round_up((uint64_t)(nh * Lk * d * 2));
    const uint64_t lb = round_up((uint64_t)(nh * Lq * 4));
    uint64_t off = 0;
    for (int t = 0; t < 12; ++t) {
        s.in[t] = off;
        off += t < 6 ? qb : (t < 10 ? kb : lb);
    }
    for (int t = 0; t < 6; ++t) {
        s.out[t] = off;
        off += t < 2 ? qb : kb;
    }
    s.stats = off;
    s.stats_bytes = bwd_stats_bytes(nh, Lq);
    s.bytes = round_up(off + s.stats_bytes);
    return s;
}

// Streams and events of the host-buffer pipeline.
// Chunk c uses staging buffer c % kBuffers and compute stream 1 + c % 2, so
// consecutive chunk kernels may overlap (the next one fills the SMs the
// previous one's last wave leaves idle).
constexpr int kBuffers = 3;
struct PipeObjects {
    cudaStream_t st[4] = {nullptr, nullptr, nullptr, nullptr};  // copy in, compute x2, copy out
    cudaEvent_t ev[1 + 3 * kBuffers] = {};                      // start, then in / comp / out per buffer
    cudaEvent_t &start() { return ev[0]; }
    cudaEvent_t &in(int b) { return ev[1 + b]; }
    cudaEvent_t &comp(int b) { return ev[1 + kBuffers + b]; }
    cudaEvent_t &out(int b) { return ev[1 + 2 * kBuffers + b]; }
    cudaError_t create() {
        cudaError_t e = cudaSuccess;
        for (int i = 0; i < 4 && e == cudaSuccess; ++i) e = cudaStreamCreateWithFlags(&st[i], cudaStreamNonBlocking);
        for (int i = 0; i < 1 + 3 * kBuffers && e == cudaSuccess; ++i)
            e = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming);
        return e;
    }
    // after a failed enqueue: wait until the chunks already issued are done, so
    // that no copy or kernel of this call still touches the staging memory
    // when the error is returned
    void drain() {
        for (cudaStream_t s : st)
            if (s) cudaStreamSynchronize(s);
    }
};
// one call's pipeline, released on scope exit (the driver defers the release
// of objects with work still pending)
struct HostPipe : PipeObjects {
    ~HostPipe() {
        for (cudaStream_t s : st)
            if (s) cudaStreamDestroy(s);
        for (cudaEvent_t x : ev)
            if (x) cudaEventDestroy(x);
    }
};

// packed sequences, bf16 or fp32 outputs (kSplit), optionally causal and saving mu
template <bool kSplit>
int launch_varlen(const void *q, const void *k, const void *v, const void *tq, const void *tk, const void *tv,
                  void *o, void *to, float *lse, float *mu, const int32_t *cu_seqlens_q,
                  const int32_t *cu_seqlens_k, int64_t n_seq, int64_t H, int64_t total_q, int64_t total_k,
                  int64_t max_seqlen_q, int64_t d, float scale, int causal, void *stream) {
    if (n_seq < 0 || max_seqlen_q < 0) return AJVP_ERR_INVALID_ARG;
    if (n_seq == 0 || max_seqlen_q == 0) {
        // nothing to compute; the size checks still apply
        if (H < 0 || total_q < 0 || total_k < 1 || d < 1 || !std::isfinite(scale)) return AJVP_ERR_INVALID_ARG;
        return AJVP_OK;
    }
    if (!cu_seqlens_q || !cu_seqlens_k) return AJVP_ERR_INVALID_ARG;
    if (!aligned(cu_seqlens_q, 4) || !aligned(cu_seqlens_k, 4)) return AJVP_ERR_MISALIGNED;
    if (n_seq >= (int64_t(1) << 31) || max_seqlen_q > total_q) return AJVP_ERR_INVALID_ARG;
    const int64_t max_qtiles = (max_seqlen_q + ajvp::sm100::BR - 1) / ajvp::sm100::BR;
    if (causal)
        return launch_sm100<kSplit, ajvp::sm100::MASK_PACKED | ajvp::sm100::MASK_CAUSAL>(
            q, k, v, tq, tk, tv, o, to, lse, 1, H, total_q, total_k, d, scale, stream, mu, cu_seqlens_q,
            cu_seqlens_k, n_seq, max_qtiles);
    return launch_sm100<kSplit, ajvp::sm100::MASK_PACKED>(q, k, v, tq, tk, tv, o, to, lse, 1, H, total_q, total_k, d,
                                                           scale, stream, mu, cu_seqlens_q, cu_seqlens_k, n_seq,
                                                           max_qtiles);
}

// The forward's host-buffer pipeline on `pipe`'s streams and events: chunks of
// nh (batch, head) slabs staged through kBuffers buffers of layout L at
// `workspace`, ordered after the caller's stream and before its continuation.
// On an error the chunks already issued are waited for before returning.
int fwd_host_enqueue(PipeObjects &pipe, const void *q, const void *k, const void *v, const void *tq, const void *tk,
                     const void *tv, void *o, void *to, float *lse, int64_t BH, int64_t Lq, int64_t Lk, int64_t d,
                     float scale, int64_t nh, const StageLayout &L, uint8_t *workspace, cudaStream_t caller) {
    auto bail = [&](int status) {
        pipe.drain();
        return status;
    };
    cudaError_t e = cudaEventRecord(pipe.start(), caller);
    if (e != cudaSuccess) return fail_cuda(e);
    for (cudaStream_t s : pipe.st)
        if ((e = cudaStreamWaitEvent(s, pipe.start(), 0)) != cudaSuccess) return bail(fail_cuda(e));

    const uint64_t qrow = (uint64_t)(Lq * d * 2), krow = (uint64_t)(Lk * d * 2);  // bytes per (b, h) slab
    const int64_t nchunks = (BH + nh - 1) / nh;
    const void *src[6] = {q, tq, k, v, tk, tv};
    const uint64_t dst_off[6] = {L.q, L.tq, L.k, L.v, L.tk, L.tv};
    for (int64_t c = 0; c < nchunks; ++c) {
        const int b = (int)(c % kBuffers);
        const int64_t h0 = c * nh, n = std::min<int64_t>(nh, BH - h0);
        uint8_t *buf = workspace + (uint64_t)b * L.bytes;
        // copy in, once the chunk that last used this buffer has been copied out
        if (c >= kBuffers && (e = cudaStreamWaitEvent(pipe.st[0], pipe.out(b), 0)) != cudaSuccess)
            return bail(fail_cuda(e));
        for (int t = 0; t < 6; ++t) {
            const uint64_t row = t < 2 ? qrow : krow;
            e = cudaMemcpyAsync(buf + dst_off[t], static_cast<const uint8_t *>(src[t]) + (uint64_t)h0 * row,
                                (uint64_t)n * row, cudaMemcpyHostToDevice, pipe.st[0]);
            if (e != cudaSuccess) return bail(fail_cuda(e));
        }
        if ((e = cudaEventRecord(pipe.in(b), pipe.st[0])) != cudaSuccess) return bail(fail_cuda(e));
        // compute
        const cudaStream_t cs = pipe.st[1 + (c & 1)];
        if ((e = cudaStreamWaitEvent(cs, pipe.in(b), 0)) != cudaSuccess) return bail(fail_cuda(e));
        const int rc = launch_sm100<false>(buf + L.q, buf + L.k, buf + L.v, buf + L.tq, buf + L.tk, buf + L.tv,
                                           buf + L.o, buf + L.to,
                                           lse ? reinterpret_cast<float *>(buf + L.lse) : nullptr, 1, n, Lq, Lk, d,
                                           scale, cs);
        if (rc != AJVP_OK) return bail(rc);
        if ((e = cudaEventRecord(pipe.comp(b), cs)) != cudaSuccess) return bail(fail_cuda(e));
        // copy out (in chunk order on one stream)
        if ((e = cudaStreamWaitEvent(pipe.st[3], pipe.comp(b), 0)) != cudaSuccess) return bail(fail_cuda(e));
        e = cudaMemcpyAsync(static_cast<uint8_t *>(o) + (uint64_t)h0 * qrow, buf + L.o, (uint64_t)n * qrow,
                            cudaMemcpyDeviceToHost, pipe.st[3]);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(static_cast<uint8_t *>(to) + (uint64_t)h0 * qrow, buf + L.to, (uint64_t)n * qrow,
                                cudaMemcpyDeviceToHost, pipe.st[3]);
        if (e == cudaSuccess && lse)
            e = cudaMemcpyAsync(lse + h0 * Lq, buf + L.lse, (uint64_t)(n * Lq * 4), cudaMemcpyDeviceToHost,
                                pipe.st[3]);
        if (e != cudaSuccess) return bail(fail_cuda(e));
        if ((e = cudaEventRecord(pipe.out(b), pipe.st[3])) != cudaSuccess) return bail(fail_cuda(e));
    }
    // the caller's stream continues once the last chunk (and so every chunk) is copied out
    if ((e = cudaStreamWaitEvent(caller, pipe.out((int)((nchunks - 1) % kBuffers)), 0)) != cudaSuccess)
        return bail(fail_cuda(e));
    return AJVP_OK;
}

// heads per chunk of the forward's host pipeline: as many as `workspace_bytes`
// holds in kBuffers buffers, at most a quarter of B*H (0 if one does not fit)
int64_t fwd_host_heads_per_chunk(int64_t BH, int64_t Lq, int64_t Lk, int64_t d, uint64_t workspace_bytes) {
    const uint64_t one = stage_layout(Lq, Lk, d, 1).bytes;
    if (workspace_bytes < kBuffers * one) return 0;
    int64_t nh = std::min<int64_t>((int64_t)(workspace_bytes / (kBuffers * one)), (BH + 3) / 4);
    while (nh > 1 && kBuffers * stage_layout(Lq, Lk, d, nh).bytes > workspace_bytes) --nh;
    return std::max<int64_t>(nh, 1);
}

}  // namespace

extern "C" {

int attn_jvp_fwd(const void *q, const void *k, const void *v, const void *tq, const void *tk, const void *tv,
                 void *o, void *to, float *lse, int64_t B, int64_t H, int64_t Lq, int64_t Lk, int64_t d,
                 float scale, void *stream) {
    return launch_sm100<false>(q, k, v, tq, tk, tv, o, to, lse, B, H, Lq, Lk, d, scale, stream);
}

int attn_jvp_fwd_f32out(const void *q, const void *k, const void *v, const void *tq, const void *tk,
                        const void *tv, float *o, float *to, float *lse, int64_t B, int64_t H, int64_t Lq,
                        int64_t Lk, int64_t d, float scale, void *stream) {
    return launch_sm100<true>(q, k, v, tq, tk, tv, o, to, lse, B, H, Lq, Lk, d, scale, stream);
}

int attn_jvp_fwd_causal(const void *q, const void *k, const void *v, const void *tq, const void *tk, const void *tv,
                        void *o, void *to, float *lse, int64_t B, int64_t H, int64_t Lq, int64_t Lk, int64_t d,
                        float scale, void *stream) {
    return launch_sm100<false, ajvp::sm100::MASK_CAUSAL>(q, k, v, tq, tk, tv, o, to, lse, B, H, Lq, Lk, d, scale,
                                                          stream);
}

int attn_jvp_fwd_varlen(const void *q, const void *k, const void *v, const void *tq, const void *tk, const void *tv,
                        void *o, void *to, float *lse, const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                        int64_t n_seq, int64_t H, int64_t total_q, int64_t total_k, int64_t max_seqlen_q, int64_t d,
                        float scale, int causal, void *stream) {
    return launch_varlen<false>(q, k, v, tq, tk, tv, o, to, lse, nullptr, cu_seqlens_q, cu_seqlens_k, n_seq, H,
                                total_q, total_k, max_seqlen_q, d, scale, causal, stream);
}

int attn_jvp_fwd_f32out_causal(const void *q, const void *k, const void *v, const void *tq, const void *tk,
                               const void *tv, float *o, float *to, float *lse, int64_t B, int64_t H, int64_t Lq,
                               int64_t Lk, int64_t d, float scale, void *stream) {
    return launch_sm100<true, ajvp::sm100::MASK_CAUSAL>(q, k, v, tq, tk, tv, o, to, lse, B, H, Lq, Lk, d, scale,
                                                         stream);
}

int attn_jvp_fwd_f32out_varlen(const void *q, const void *k, const void *v, const void *tq, const void *tk,
                               const void *tv, float *o, float *to, float *lse, const int32_t *cu_seqlens_q,
                               const int32_t *cu_seqlens_k, int64_t n_seq, int64_t H, int64_t total_q,
                               int64_t total_k, int64_t max_seqlen_q, int64_t d, float scale, int causal,
                               void *stream) {
    return launch_varlen<true>(q, k, v, tq, tk, tv, o, to, lse, nullptr, cu_seqlens_q, cu_seqlens_k, n_seq, H,
                               total_q, total_k, max_seqlen_q, d, scale, causal, stream);
}

int attn_jvp_fwd_stats(const void *q, const void *k, const void *v, const void *tq, const void *tk, const void *tv,
                       void *o, void *to, float *lse, float *mu, int64_t B, int64_t H, int64_t Lq, int64_t Lk,
                       int64_t d, float scale, void *stream) {
    if (B > 0 && H > 0 && Lq > 0 && (!lse || !mu)) return AJVP_ERR_INVALID_ARG;
    return launch_sm100<false>(q, k, v, tq, tk, tv, o, to, lse, B, H, Lq, Lk, d, scale, stream, mu);
}

uint64_t attn_jvp_bwd_workspace_bytes(int64_t B, int64_t H, int64_t Lq) {
    if (B < 0 || H < 0 || Lq < 0) return 0;
    return bwd_stats_bytes(B * H, Lq);
}

int64_t attn_jvp_bwd_key_split_parts(int64_t B, int64_t H, int64_t Lq, int64_t Lk, int64_t sm_count) {
    if (B < 0 || H < 0 || Lq < 0 || Lk < 0 || sm_count < 1 || sm_count > (int64_t(1) << 20)) return 0;
    if (B > 0 && H > (int64_t(1) << 40) / B) return 0;
    return bwd_key_split(B * H, Lq, Lk, (int)sm_count);
}

uint64_t attn_jvp_bwd_workspace_bytes_split(int64_t B, int64_t H, int64_t Lq, int64_t Lk) {
    if (B < 0 || H < 0 || Lq < 0 || Lk < 0) return 0;
    const uint64_t base = bwd_stats_bytes(B * H, Lq);
    int dev = 0;
    if (device_setup(&dev) != AJVP_OK) return base;  // no usable device: the minimum
    return base + 2u * bwd_partial_bytes(B * H, Lk, bwd_key_split(B * H, Lq, Lk, g_dev[dev].sm_count));
}

}  // extern "C"

namespace {
// Kernels first..last of the backward (0 row statistics, 1 dQ and dtQ, 2 dK
// and dtK, 3 dV and dtV) after the full argument check; mask: causal and/or
// packed (pk: the sequences of a packed call).
int bwd_steps(int first, int last, int mask, const BwdPack &pk, const void *q, const void *k, const void *v,
              const void *tq, const void *tk, const void *tv, const void *o, const void *to, const float *lse,
              const float *mu, const void *dout,
              const void *dtout, void *dq, void *dk, void *dv, void *dtq, void *dtk, void *dtv, int64_t B, int64_t H,
              int64_t Lq, int64_t Lk, int64_t d, float scale, void *workspace, uint64_t workspace_bytes,
              void *stream) {
    bool noop = false;
    int rc = check_common(q, k, v, tq, tk, tv, o, to, B, H, Lq, Lk, d, scale, &noop);
    if (rc != AJVP_OK) return rc;
    const int64_t BH = B * H;
    const cudaStream_t st = (cudaStream_t)stream;
    if (noop) {
        // no query rows: the key-side gradients are zero; nothing else to write
        if (BH == 0) return AJVP_OK;
        if (!dk || !dv || !dtk || !dtv) return AJVP_ERR_INVALID_ARG;
        if (BH * Lk >= (int64_t(1) << 31)) return AJVP_ERR_TOO_LARGE;
        const size_t bytes = (size_t)(BH * Lk * d) * 2u;
        // the steps that would write them: dk and dtk 2, dv and dtv 3
        void *zero[4] = {dk, dtk, dv, dtv};
        const int kern[4] = {2, 2, 3, 3};
        for (int i = 0; i < 4; ++i) {
            if (first > kern[i] || last < kern[i]) continue;
            cudaError_t e = cudaMemsetAsync(zero[i], 0, bytes, st);
            if (e != cudaSuccess) return fail_cuda(e);
        }
        return AJVP_OK;
    }
    if (d != ajvp::bwd::HD) return AJVP_ERR_UNSUPPORTED_DIM;
    const void *ptrs[18] = {q, k, v, tq, tk, tv, o, to, lse, mu, dout, dtout, dq, dk, dv, dtq, dtk, dtv};
    for (int i = 0; i < 18; ++i) {
        if (!ptrs[i]) return AJVP_ERR_INVALID_ARG;
        if (!aligned(ptrs[i], 16)) return AJVP_ERR_MISALIGNED;
    }
    if (((Lq + 127) / 128) * BH >= (int64_t(1) << 31) || ((Lk + 127) / 128) * BH >= (int64_t(1) << 31) ||
        BH * Lq + ajvp::bwd::BN >= (int64_t(1) << 40))
        return AJVP_ERR_TOO_LARGE;
    // the masked kernels form row + (Lk - Lq) sums in 32 bits
    if (mask != 0 && (Lq >= (int64_t(1) << 30) || Lk >= (int64_t(1) << 30))) return AJVP_ERR_TOO_LARGE;
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < bwd_stats_bytes(BH, Lq))
        return AJVP_ERR_WORKSPACE;
    int dev = 0;
    if ((rc = device_setup(&dev)) != AJVP_OK) return rc;
    if ((rc = get_encoder()) != AJVP_OK) return rc;
    // unmasked key side: cut the query range into parts when the key tiles alone
    // cannot fill the GPU and the workspace holds the partial sums
    int64_t n_split = mask == 0 ? bwd_key_split(BH, Lq, Lk, g_dev[dev].sm_count) : 1;
    const uint64_t part_bytes = bwd_partial_bytes(BH, Lk, n_split);
    if (n_split > 1 && workspace_bytes < bwd_stats_bytes(BH, Lq) + 2u * part_bytes) n_split = 1;
    uint8_t *const part_base = static_cast<uint8_t *>(workspace) + bwd_stats_bytes(BH, Lq);
    float *const partial_k = reinterpret_cast<float *>(part_base);
    float *const partial_v = reinterpret_cast<float *>(part_base + part_bytes);

    using namespace ajvp::bwd;
    if (first <= 0 && last >= 0) {
        const long long rows = (long long)(BH * Lq);
        const unsigned grid = (unsigned)std::min<long long>((rows + 7) / 8, 148LL * 16);
        bwd_rowstats_kernel<<<grid, 256, 0, st>>>(
            static_cast<const __nv_bfloat16 *>(o), static_cast<const __nv_bfloat16 *>(to),
            static_cast<const __nv_bfloat16 *>(dout), static_cast<const __nv_bfloat16 *>(dtout), lse, mu,
            static_cast<float4 *>(workspace), rows);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return fail_cuda(e);
    }
    auto want = [&](int k) { return first <= k && last >= k; };
    const float s1 = scale;
    // rows = queries, streamed keys: dq, dtq
    if (want(1) && (rc = launch_bwd_mask<V_Q>(mask, {q, tq, dtout, dout}, {k, tk}, {v, tv}, {dq, dtq}, {s1, s1},
                                              workspace, BH, Lq, Lk, Lq, d, scale, st, pk.cu_q, pk.cu_k, pk.n_seq,
                                              pk.max_q)) != AJVP_OK)
        return rc;
    // rows = keys, streamed queries: dk, dtk; dv, dtv (split: each kernel with its
    // own partial-sum region, reduced on the stream before the step returns)
    if (want(2)) {
        rc = n_split > 1 ? launch_bwd_split<V_K>({k, tk, v, tv}, {q, tq}, {dtout, dout}, dk, dtk, s1, s1, workspace,
                                                 BH, Lk, Lq, Lq, d, scale, st, n_split, partial_k)
                         : launch_bwd_mask<V_K>(mask, {k, tk, v, tv}, {q, tq}, {dtout, dout}, {dk, dtk}, {s1, s1},
                                                workspace, BH, Lk, Lq, Lq, d, scale, st, pk.cu_k, pk.cu_q, pk.n_seq,
                                                pk.max_k);
        if (rc != AJVP_OK) return rc;
    }
    if (want(3)) {
        rc = n_split > 1 ? launch_bwd_split<V_V>({k, tk}, {dout, dtout}, {q, tq}, dv, dtv, 1.0f, 1.0f, workspace, BH,
                                                 Lk, Lq, Lq, d, scale, st, n_split, partial_v)
                         : launch_bwd_mask<V_V>(mask, {k, tk}, {dout, dtout}, {q, tq}, {dv, dtv}, {1.0f, 1.0f},
                                                workspace, BH, Lk, Lq, Lq, d, scale, st, pk.cu_k, pk.cu_q, pk.n_seq,
                                                pk.max_k);
        if (rc != AJVP_OK) return rc;
    }
    return AJVP_OK;
}
}  // namespace

extern "C" {

int attn_jvp_bwd(const void *q, const void *k, const void *v, const void *tq, const void *tk, const void *tv,
                 const void *o, const void *to, const float *lse, const float *mu, const void *dout,
                 const void *dtout, void *dq, void *dk, void *dv, void *dtq, void *dtk, void *dtv, int64_t B,
                 int64_t H, int64_t Lq, int64_t Lk, int64_t d, float scale, void *workspace,
                 uint64_t workspace_bytes, void *stream) {
    return bwd_steps(0, 3, 0, BwdPack(), q, k, v, tq, tk, tv, o, to, lse, mu, dout, dtout, dq, dk, dv, dtq, dtk,
                     dtv, B, H, Lq, Lk, d, scale, workspace, workspace_bytes, stream);
}

int attn_jvp_fwd_causal_stats(const void *q, const void *k, const void *v, const void *tq, const void *tk,
                              const void *tv, void *o, void *to, float *lse, float *mu, int64_t B, int64_t H,
                              int64_t Lq, int64_t Lk, int64_t d, float scale, void *stream) {
    if (B > 0 && H > 0 && Lq > 0 && (!lse || !mu)) return AJVP_ERR_INVALID_ARG;
    return launch_sm100<false, ajvp::sm100::MASK_CAUSAL>(q, k, v, tq, tk, tv, o, to, lse, B, H, Lq, Lk, d, scale,
                                                          stream, mu);
}

int attn_jvp_bwd_causal(const void *q, const void *k, const void *v, const void *tq, const void *tk,
                        const void *tv, const void *o, const void *to, const float *lse, const float *mu,
                        const void *dout, const void *dtout, void *dq, void *dk, void *dv, void *dtq, void *dtk,
                        void *dtv, int64_t B, int64_t H, int64_t Lq, int64_t Lk, int64_t d, float scale,
                        void *workspace, uint64_t workspace_bytes, void *stream) {
    return bwd_steps(0, 3, ajvp::bwd::MASK_CAUSAL, BwdPack(), q, k, v, tq, tk, tv, o, to, lse, mu, dout, dtout, dq,
                     dk, dv, dtq, dtk, dtv, B, H, Lq, Lk, d, scale, workspace, workspace_bytes, stream);
}

int attn_jvp_fwd_varlen_stats(const void *q, const void *k, const void *v, const void *tq, const void *tk,
                              const void *tv, void *o, void *to, float *lse, float *mu,
                              const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k, int64_t n_seq, int64_t H,
                              int64_t total_q, int64_t total_k, int64_t max_seqlen_q, int64_t d, float scale,
                              int causal, void *stream) {
    if (n_seq > 0 && max_seqlen_q > 0 && H > 0 && total_q > 0 && (!lse || !mu)) return AJVP_ERR_INVALID_ARG;
    return launch_varlen<false>(q, k, v, tq, tk, tv, o, to, lse, mu, cu_seqlens_q, cu_seqlens_k, n_seq, H, total_q,
                                total_k, max_seqlen_q, d, scale, causal, stream);
}

int attn_jvp_bwd_varlen(const void *q, const void *k, const void *v, const void *tq, const void *tk,
                        const void *tv, const void *o, const void *to, const float *lse, const float *mu,
                        const void *dout, const void *dtout, void *dq, void *dk, void *dv, void *dtq, void *dtk,
                        void *dtv, const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k, int64_t n_seq,
                        int64_t H, int64_t total_q, int64_t total_k, int64_t max_seqlen_q, int64_t max_seqlen_k,
                        int64_t d, float scale, int causal, void *workspace, uint64_t workspace_bytes,
                        void *stream) {
    if (n_seq < 0 || max_seqlen_q < 0 || max_seqlen_k < 0) return AJVP_ERR_INVALID_ARG;
    if (max_seqlen_q > total_q || max_seqlen_k > total_k || n_seq >= (int64_t(1) << 31))
        return AJVP_ERR_INVALID_ARG;
    BwdPack pk;
    pk.cu_q = cu_seqlens_q;
    pk.cu_k = cu_seqlens_k;
    pk.n_seq = n_seq;
    pk.max_q = max_seqlen_q;
    pk.max_k = max_seqlen_k;
    if (n_seq > 0 && total_q > 0) {
        if (!cu_seqlens_q || !cu_seqlens_k) return AJVP_ERR_INVALID_ARG;
        if (!aligned(cu_seqlens_q, 4) || !aligned(cu_seqlens_k, 4)) return AJVP_ERR_MISALIGNED;
    }
    const int mask = ajvp::bwd::MASK_PACKED | (causal ? ajvp::bwd::MASK_CAUSAL : 0);
    return bwd_steps(0, 3, mask, pk, q, k, v, tq, tk, tv, o, to, lse, mu, dout, dtout, dq, dk, dv, dtq, dtk, dtv, 1,
                     H, total_q, total_k, d, scale, workspace, workspace_bytes, stream);
}

int attn_jvp_bwd_step(int step, const void *q, const void *k, const void *v, const void *tq, const void *tk,
                      const void *tv, const void *o, const void *to, const float *lse, const float *mu,
                      const void *dout, const void *dtout, void *dq, void *dk, void *dv, void *dtq, void *dtk,
                      void *dtv, int64_t B, int64_t H, int64_t Lq, int64_t Lk, int64_t d, float scale,
                      void *workspace, uint64_t workspace_bytes, void *stream) {
    if (step < 0 || step > 3) return AJVP_ERR_INVALID_ARG;
    return bwd_steps(step, step, 0, BwdPack(), q, k, v, tq, tk, tv, o, to, lse, mu, dout, dtout, dq, dk, dv, dtq, dtk,
                     dtv, B, H, Lq, Lk, d, scale, workspace, workspace_bytes, stream);
}

uint64_t attn_jvp_host_workspace_bytes(int64_t Lq, int64_t Lk, int64_t d, int64_t heads_per_chunk) {
    if (Lq < 1 || Lk < 1 || d < 1 || heads_per_chunk < 1) return 0;
    return kBuffers * stage_layout(Lq, Lk, d, heads_per_chunk).bytes;
}

int attn_jvp_fwd_host(const void *q, const void *k, const void *v, const void *tq, const void *tk, const void *tv,
                      void *o, void *to, float *lse, int64_t B, int64_t H, int64_t Lq, int64_t Lk, int64_t d,
                      float scale, void *workspace, uint64_t workspace_bytes, void *stream) {
    bool noop = false;
    int rc = check_common(q, k, v, tq, tk, tv, o, to, B, H, Lq, Lk, d, scale, &noop);
    if (rc != AJVP_OK || noop) return rc;
    if (d != ajvp::sm100::HD) return AJVP_ERR_UNSUPPORTED_DIM;
    const int64_t BH = B * H;
    const int64_t nh = fwd_host_heads_per_chunk(BH, Lq, Lk, d, workspace_bytes);
    if (!workspace || !aligned(workspace, kStageAlign) || nh < 1) return AJVP_ERR_WORKSPACE;
    const StageLayout L = stage_layout(Lq, Lk, d, nh);
    int dev = 0;
    if ((rc = device_setup(&dev)) != AJVP_OK) return rc;

    HostPipe pipe;
    const cudaError_t e = pipe.create();
    if (e != cudaSuccess) return fail_cuda(e);
    return fwd_host_enqueue(pipe, q, k, v, tq, tk, tv, o, to, lse, BH, Lq, Lk, d, scale, nh, L,
                            static_cast<uint8_t *>(workspace), (cudaStream_t)stream);
}

uint64_t attn_jvp_bwd_host_workspace_bytes(int64_t Lq, int64_t Lk, int64_t d, int64_t heads_per_chunk) {
    if (Lq < 1 || Lk < 1 || d < 1 || heads_per_chunk < 1) return 0;
    return kBuffers * bwd_stage_layout(Lq, Lk, d, heads_per_chunk).bytes;
}

int attn_jvp_bwd_host(const void *q, const void *k, const void *v, const void *tq, const void *tk, const void *tv,
                      const void *o, const void *to, const float *lse, const float *mu, const void *dout,
                      const void *dtout, void *dq, void *dk, void *dv, void *dtq, void *dtk, void *dtv, int64_t B,
                      int64_t H, int64_t Lq, int64_t Lk, int64_t d, float scale, void *workspace,
                      uint64_t workspace_bytes, void *stream) {
    bool noop = false;
    int rc = check_common(q, k, v, tq, tk, tv, o, to, B, H, Lq, Lk, d, scale, &noop);
    if (rc != AJVP_OK) return rc;
    const int64_t BH = B * H;
    if (noop) {
        // no query rows: the key-side gradients are zero (written once the caller's
        // stream has reached this call, like the device entry's memsets)
        if (BH == 0) return AJVP_OK;
        if (!dk || !dv || !dtk || !dtv) return AJVP_ERR_INVALID_ARG;
        cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
        if (e != cudaSuccess) return fail_cuda(e);
        const size_t bytes = (size_t)(BH * Lk * d) * 2u;
        for (void *g : {dk, dv, dtk, dtv}) std::memset(g, 0, bytes);
        return AJVP_OK;
    }
    if (d != ajvp::bwd::HD) return AJVP_ERR_UNSUPPORTED_DIM;
    const void *ptrs[18] = {q, k, v, tq, tk, tv, o, to, lse, mu, dout, dtout, dq, dk, dv, dtq, dtk, dtv};
    for (int i = 0; i < 18; ++i)
        if (!ptrs[i]) return AJVP_ERR_INVALID_ARG;
    const uint64_t one = bwd_stage_layout(Lq, Lk, d, 1).bytes;
    if (!workspace || !aligned(workspace, kStageAlign) || workspace_bytes < kBuffers * one) return AJVP_ERR_WORKSPACE;
    // heads per chunk: as many as the workspace holds, at most a quarter of B*H
    int64_t nh = std::min<int64_t>((int64_t)(workspace_bytes / (kBuffers * one)), (BH + 3) / 4);
    while (nh > 1 && kBuffers * bwd_stage_layout(Lq, Lk, d, nh).bytes > workspace_bytes) --nh;
    nh = std::max<int64_t>(nh, 1);
    const BwdStageLayout L = bwd_stage_layout(Lq, Lk, d, nh);
    int dev = 0;
    if ((rc = device_setup(&dev)) != AJVP_OK) return rc;

    HostPipe pipe;
    cudaError_t e = pipe.create();
    if (e != cudaSuccess) return fail_cuda(e);
    // after the start event: on an error, wait for the chunks already issued
    auto bail = [&](int status) {
        pipe.drain();
        return status;
    };
    const cudaStream_t caller = (cudaStream_t)stream;
    if ((e = cudaEventRecord(pipe.start(), caller)) != cudaSuccess) return fail_cuda(e);
    for (cudaStream_t s : pipe.st)
        if ((e = cudaStreamWaitEvent(s, pipe.start(), 0)) != cudaSuccess) return bail(fail_cuda(e));

    // bytes per (b, h) slab of each array, in the layout's order
    const uint64_t qrow = (uint64_t)(Lq * d * 2), krow = (uint64_t)(Lk * d * 2), srow = (uint64_t)(Lq * 4);
    const void *src[12] = {q, tq, o, to, dout, dtout, k, v, tk, tv, lse, mu};
    const uint64_t in_row[12] = {qrow, qrow, qrow, qrow, qrow, qrow, krow, krow, krow, krow, srow, srow};
    void *dst[6] = {dq, dtq, dk, dv, dtk, dtv};
    const uint64_t out_row[6] = {qrow, qrow, krow, krow, krow, krow};
    const int64_t nchunks = (BH + nh - 1) / nh;
    for (int64_t c = 0; c < nchunks; ++c) {
        const int b = (int)(c % kBuffers);
        const int64_t h0 = c * nh, n = std::min<int64_t>(nh, BH - h0);
        uint8_t *buf = static_cast<uint8_t *>(workspace) + (uint64_t)b * L.bytes;
        // copy in, once the chunk that last used this buffer has been copied out
        if (c >= kBuffers && (e = cudaStreamWaitEvent(pipe.st[0], pipe.out(b), 0)) != cudaSuccess)
            return bail(fail_cuda(e));
        for (int t = 0; t < 12; ++t) {
            e = cudaMemcpyAsync(buf + L.in[t], static_cast<const uint8_t *>(src[t]) + (uint64_t)h0 * in_row[t],
                                (uint64_t)n * in_row[t], cudaMemcpyHostToDevice, pipe.st[0]);
            if (e != cudaSuccess) return bail(fail_cuda(e));
        }
        if ((e = cudaEventRecord(pipe.in(b), pipe.st[0])) != cudaSuccess) return bail(fail_cuda(e));
        // compute: the four backward kernels on the chunk's n (batch, head) slabs
        const cudaStream_t cs = pipe.st[1 + (c & 1)];
        if ((e = cudaStreamWaitEvent(cs, pipe.in(b), 0)) != cudaSuccess) return bail(fail_cuda(e));
        rc = bwd_steps(0, 3, 0, BwdPack(), buf + L.in[0], buf + L.in[6], buf + L.in[7], buf + L.in[1], buf + L.in[8],
                       buf + L.in[9], buf + L.in[2], buf + L.in[3], reinterpret_cast<const float *>(buf + L.in[10]),
                       reinterpret_cast<const float *>(buf + L.in[11]), buf + L.in[4], buf + L.in[5],
                       buf + L.out[0], buf + L.out[2], buf + L.out[3], buf + L.out[1], buf + L.out[4],
                       buf + L.out[5], 1, n, Lq, Lk, d, scale, buf + L.stats, L.stats_bytes, cs);
        if (rc != AJVP_OK) return bail(rc);
        if ((e = cudaEventRecord(pipe.comp(b), cs)) != cudaSuccess) return bail(fail_cuda(e));
        // copy out (in chunk order on one stream)
        if ((e = cudaStreamWaitEvent(pipe.st[3], pipe.comp(b), 0)) != cudaSuccess) return bail(fail_cuda(e));
        for (int t = 0; t < 6; ++t) {
            e = cudaMemcpyAsync(static_cast<uint8_t *>(dst[t]) + (uint64_t)h0 * out_row[t], buf + L.out[t],
                                (uint64_t)n * out_row[t], cudaMemcpyDeviceToHost, pipe.st[3]);
            if (e != cudaSuccess) return bail(fail_cuda(e));
        }
        if ((e = cudaEventRecord(pipe.out(b), pipe.st[3])) != cudaSuccess) return bail(fail_cuda(e));
    }
    if ((e = cudaStreamWaitEvent(caller, pipe.out((int)((nchunks - 1) % kBuffers)), 0)) != cudaSuccess)
        return bail(fail_cuda(e));
    return AJVP_OK;
}

int attn_jvp_fwd_f32(const float *q, const float *k, const float *v, const float *tq, const float *tk,
                     const float *tv, float *o, float *to, float *lse, int64_t B, int64_t H, int64_t Lq, int64_t Lk,
                     int64_t d, float scale, void *stream) {
    bool noop = false;
    int rc = check_common(q, k, v, tq, tk, tv, o, to, B, H, Lq, Lk, d, scale, &noop);
    if (rc != AJVP_OK || noop) return rc;
    if (d > ajvp::f32::DMAX) return AJVP_ERR_UNSUPPORTED_DIM;
    const void *ptrs[9] = {q, k, v, tq, tk, tv, o, to, lse};
    for (int i = 0; i < 9; ++i)
        if (ptrs[i] && !aligned(ptrs[i], 4)) return AJVP_ERR_MISALIGNED;
    const int64_t BH = B * H;
    const int64_t n_qtiles = (Lq + ajvp::f32::BR - 1) / ajvp::f32::BR;
    if (n_qtiles * BH >= (int64_t(1) << 31)) return AJVP_ERR_TOO_LARGE;

    int dev = 0;
    rc = device_setup(&dev);
    if (rc != AJVP_OK) return rc;
    ajvp::f32::attn_jvp_fwd_f32_kernel<<<(unsigned)(n_qtiles * BH), ajvp::f32::WARPS * 32,
                                         ajvp::f32::smem_bytes((int)d), (cudaStream_t)stream>>>(
        q, k, v, tq, tk, tv, o, to, lse, (int)Lq, (int)Lk, (int)d, (int)n_qtiles, scale);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail_cuda(e);
    return AJVP_OK;
}

const char *attn_jvp_strerror(int status) {
    switch (status) {
        case AJVP_OK: return "success";
        case AJVP_ERR_INVALID_ARG: return "invalid argument (null pointer, negative size, Lk < 1 or non-finite scale)";
        case AJVP_ERR_UNSUPPORTED_DIM: return "unsupported head dimension for this entry point";
        case AJVP_ERR_MISALIGNED: return "pointer not aligned as the entry point requires";
        case AJVP_ERR_UNSUPPORTED_DEVICE: return "current device is not compute capability 10.0 (B200)";
        case AJVP_ERR_TIMEOUT: return "a kernel wait ran past its bound";
        case AJVP_ERR_CUDA: return "CUDA runtime or driver error";
        case AJVP_ERR_TOO_LARGE: return "a size exceeds the supported maximum";
        case AJVP_ERR_WORKSPACE: return "device workspace missing, not 256-byte aligned or too small";
        case AJVP_ERR_DEVICE_LAYOUT: return "a kernel found its shared memory misaligned and did nothing";
        default: return "unknown status";
    }
}

int attn_jvp_last_cuda_error(void) { return t_last_cuda_error; }

int attn_jvp_check_device_status(void *stream) {
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return fail_cuda(e);
    int word = 0;
    e = cudaMemcpyFromSymbol(&word, ajvp::g_status_word, sizeof(int));
    if (e != cudaSuccess) return fail_cuda(e);
    if (word != 0) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(ajvp::g_status_word, &zero, sizeof(int));
        if (e != cudaSuccess) return fail_cuda(e);
        return (word & 2) ? AJVP_ERR_DEVICE_LAYOUT : AJVP_ERR_TIMEOUT;
    }
    return AJVP_OK;
}

int attn_jvp_set_wait_bound_ns(uint64_t ns) {
    g_bound_ns.store(ns == 0 ? kDefaultBoundNs : ns);
    return AJVP_OK;
}

int attn_jvp_set_persistent_key_tiles(int64_t max_key_tiles) {
    if (max_key_tiles < 0) return AJVP_ERR_INVALID_ARG;
    g_persist_key_tiles.store(max_key_tiles);
    return AJVP_OK;
}

int attn_jvp_set_bwd_pairs(int on) {
    g_bwd_pairs.store(on != 0 ? 1 : 0);
    return AJVP_OK;
}

int attn_jvp_version(void) { return kVersion; }

}  // extern "C"

// ------------------------------------------------------- failure self test
namespace {
__global__ void selftest_wait_kernel(unsigned long long bound_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    const uint32_t b = ajvp::smem_u32(&bar);
    if (threadIdx.x == 0) {
        ajvp::mbar_init(b, 1);
        abort_flag = 0;
        ajvp::fence_barrier_init();
    }
    __syncwarp();
    // nothing ever arrives on `bar`: the bounded wait must give up
    bool ok = ajvp::mbar_wait(b, 0, reinterpret_cast<volatile int *>(&abort_flag), bound_ns);
    ok = __all_sync(0xffffffffu, ok);
    (void)ok;
}
}  // namespace

extern "C" int attn_jvp_selftest_wait_timeout(uint64_t bound_ns, void *stream) {
    int dev = 0;
    int rc = device_setup(&dev);
    if (rc != AJVP_OK) return rc;
    if (bound_ns == 0 || bound_ns > 10000000000ull) return AJVP_ERR_INVALID_ARG;
    selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((unsigned long long)bound_ns);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail_cuda(e);
    return AJVP_OK;
}

// ------------------------------------------- host entry on static scratch
// attn_jvp_fwd_host_noalloc stages its chunks in this file-scope device
// array instead of a caller-supplied workspace.  On the entry point's first
// call on a device (that device current) it looks up the array's device
// address there and creates the pipeline's streams and events, which every
// later call on the device reuses, so that a call itself creates and frees
// nothing.  Nothing in the array needs to start at zero: every byte a kernel
// reads is first written by the same call's copies.
namespace {
constexpr uint64_t kNoallocScratchBytes = 64ull << 20;  // 64 MiB per device
struct NoallocState {
    std::once_flag once;
    std::mutex enqueue;  // one call at a time enqueues on the shared streams and events
    void *ptr = nullptr;
    PipeObjects pipe;    // kept until the process exits
    int cuda_error = 0;
};
NoallocState g_noalloc[kMaxDevices];
}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

extern "C" int attn_jvp_fwd_host_noalloc(const void *q, const void *k, const void *v, const void *tq,
                                         const void *tk, const void *tv, void *o, void *to, float *lse, int64_t B,
                                         int64_t H, int64_t Lq, int64_t Lk, int64_t d, float scale, void *stream) {
    bool noop = false;
    int rc = check_common(q, k, v, tq, tk, tv, o, to, B, H, Lq, Lk, d, scale, &noop);
    if (rc != AJVP_OK || noop) return rc;
    if (d != ajvp::sm100::HD) return AJVP_ERR_UNSUPPORTED_DIM;
    // one (batch, head) slab, three staging buffers, must fit the scratch
    const int64_t nh = fwd_host_heads_per_chunk(B * H, Lq, Lk, d, kNoallocScratchBytes);
    if (nh < 1) return AJVP_ERR_TOO_LARGE;
    int dev = 0;
    if ((rc = device_setup(&dev)) != AJVP_OK) return rc;
    NoallocState &st = g_noalloc[dev];
    std::call_once(st.once, [&]() {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e == cudaSuccess) e = st.pipe.create();
        if (e == cudaSuccess)
            st.ptr = p;
        else
            st.cuda_error = (int)e;
    });
    if (!st.ptr) {
        t_last_cuda_error = st.cuda_error;
        return AJVP_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(st.enqueue);
    return fwd_host_enqueue(st.pipe, q, k, v, tq, tk, tv, o, to, lse, B * H, Lq, Lk, d, scale, nh,
                            stage_layout(Lq, Lk, d, nh), static_cast<uint8_t *>(st.ptr), (cudaStream_t)stream);
}
