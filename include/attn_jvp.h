/*
 * attn_jvp.h -- C ABI of the fused attention + Jacobian-vector-product
 * forward pass for NVIDIA B200 (sm_100a).
 *
 * The operation (rCM, "Large-scale diffusion distillation via
 * score-regularized continuous-time consistency", §3.2 / App. C, as the
 * anthology record LIT-783 summarises it: FlashAttention-2 and its JVP in one
 * tiled pass, for self- and cross-attention; the model card "rCM Consistency
 * Distillation Diffusion Model", Research Highlights, names the open-source
 * FlashAttention-2 JVP kernel).  For every batch b, head h and query row i:
 *
 *   S   = s * Q K^T                   P  = row-softmax(S)
 *   dS  = s * (tQ K^T + Q tK^T)       mu = rowsum(P .* dS)
 *   O   = P V
 *   tO  = (P .* (dS - mu)) V + P tV   (the derivative of O along (tQ, tK, tV))
 *   lse = ln sum_j exp(S_ij)          (natural log, fp32)
 *
 * computed in one pass over the keys with an online softmax: P and dS are
 * never written to memory.  No dropout; Lq may differ from Lk
 * (cross-attention); attn_jvp_fwd_causal and attn_jvp_fwd_varlen add a
 * causal mask and packed variable-length sequences, attn_jvp_bwd the
 * backward pass (attn_jvp_bwd_causal and attn_jvp_bwd_varlen those of the
 * masked forwards).  s is a constant (no derivative with respect to it).
 *
 * Layout: every tensor is a contiguous row-major [B][H][L][d] array (the
 * layout of a PyTorch [B, H, L, d] tensor); the tangents tQ, tK, tV share the
 * layout of Q, K, V (the anthology record notes that context parallelism
 * distributes the QKV tangents like QKV).  lse is [B][H][Lq] fp32.
 *
 * Ownership and execution: all pointers are DEVICE pointers owned by the
 * caller (except the data pointers of attn_jvp_fwd_host and
 * attn_jvp_fwd_host_noalloc, which are host pointers).  The library
 * allocates no device memory per call and keeps no per-call state.  Calls
 * are stream-ordered and asynchronous: they return
 * after enqueueing work on `stream` (a cudaStream_t; NULL = legacy default
 * stream) and do not synchronise.  The device-buffer calls enqueue kernels
 * only (attn_jvp_bwd with Lq == 0: memsets), so after one eager call on a
 * device (which does its one-time set-up) they can be captured into a CUDA
 * graph.  Calls are thread-safe.  Inputs must not alias outputs.  Non-finite
 * inputs give unspecified (but memory-safe) results.
 *
 * Errors: argument checks run on the host before any launch and return a
 * negative ajvp_status; nothing is enqueued then.  A failed launch returns
 * AJVP_ERR_CUDA and the cudaError_t is kept per thread
 * (attn_jvp_last_cuda_error).  Every wait inside the kernels is bounded: if a
 * pipeline wait ever exceeds the wait bound, the kernel records
 * AJVP_ERR_TIMEOUT in a device status word, releases what it holds and
 * returns; attn_jvp_check_device_status reads (and clears) that word.
 */
#ifndef ATTN_JVP_H
#define ATTN_JVP_H

#include <stdint.h>

#if defined(__GNUC__)
#define AJVP_API __attribute__((visibility("default")))
#else
#define AJVP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    AJVP_OK = 0,
    AJVP_ERR_INVALID_ARG = -1,        /* null pointer, negative size, Lk == 0, non-finite scale */
    AJVP_ERR_UNSUPPORTED_DIM = -2,    /* head dimension d not supported by this entry point */
    AJVP_ERR_MISALIGNED = -3,         /* a pointer breaks the alignment rule of the entry point */
    AJVP_ERR_UNSUPPORTED_DEVICE = -4, /* current device is not compute capability 10.0 */
    AJVP_ERR_TIMEOUT = -5,            /* a kernel wait ran past its bound (device status word) */
    AJVP_ERR_CUDA = -6,               /* a CUDA runtime/driver call failed */
    AJVP_ERR_TOO_LARGE = -7,          /* a size exceeds the documented maximum */
    AJVP_ERR_WORKSPACE = -8,          /* workspace missing, misaligned or too small */
    AJVP_ERR_DEVICE_LAYOUT = -9       /* a kernel found its shared memory misaligned (device status word) */
} ajvp_status;

/*
 * attn_jvp_fwd -- bf16 I/O, fp32 accumulation, tcgen05 tensor-core kernel.
 *
 *   q, tq      : const __nv_bfloat16 [B][H][Lq][d]
 *   k, v, tk, tv: const __nv_bfloat16 [B][H][Lk][d]
 *   o, to      : __nv_bfloat16 [B][H][Lq][d]   (outputs, round-to-nearest-even)
 *   lse        : float [B][H][Lq], or NULL to skip it
 *   scale      : the softmax scale s (finite)
 *   stream     : cudaStream_t, or NULL
 *
 * Supported: d == 128; B, H, Lq >= 0; Lk >= 1; Lq, Lk < 2^31;
 * B*H*ceil(Lq/128) < 2^31.  B*H == 0 or Lq == 0 is a no-op returning AJVP_OK.
 * Every pointer must be 16-byte aligned (tensor-memory-accelerator rule).
 * The current device must be compute capability 10.0 (B200).
 * Returns AJVP_OK once the kernel is enqueued.
 */
AJVP_API int attn_jvp_fwd(const void *q, const void *k, const void *v,
                 const void *tq, const void *tk, const void *tv,
                 void *o, void *to, float *lse,
                 int64_t B, int64_t H, int64_t Lq, int64_t Lk, int64_t d,
                 float scale, void *stream);

/*
 * attn_jvp_fwd_f32out -- bf16 inputs, fp32 outputs, for when the tangent must
 * be accurate beyond bf16 (the anthology record LIT-783, takeaway on §3.3 and
 * Fig. 11: BF16 JVP error is much larger than BF16 output error).  Same
 * tcgen05 kernel as attn_jvp_fwd, but the probabilities P and the tangent
 * weights P.*s dS' are each carried as two bf16 parts (hi + lo, ~16
 * significant bits) into the P.V products, and O, tO are written in fp32
 * (1.5x the tensor-core work of attn_jvp_fwd).
 *
 *   q, k, v, tq, tk, tv : const __nv_bfloat16, layouts as attn_jvp_fwd
 *   o, to               : float [B][H][Lq][d]
 *   lse                 : float [B][H][Lq], or NULL
 *
 * Same sizes, alignment (16 bytes), device and error rules as attn_jvp_fwd.
 */
AJVP_API int attn_jvp_fwd_f32out(const void *q, const void *k, const void *v,
                        const void *tq, const void *tk, const void *tv,
                        float *o, float *to, float *lse,
                        int64_t B, int64_t H, int64_t Lq, int64_t Lk, int64_t d,
                        float scale, void *stream);

/*
 * attn_jvp_fwd_causal -- attn_jvp_fwd with a causal mask: key j is visible to
 * query row i iff j <= i + (Lk - Lq), i.e. the lower-triangular mask when
 * Lq == Lk and bottom-right aligned otherwise.  Rows that see no key (only
 * when Lq > Lk) get O = tO = 0 and lse = -infinity.  The pages do not
 * describe masks; the arguments, layout and rules are those of
 * attn_jvp_fwd.
 */
AJVP_API int attn_jvp_fwd_causal(const void *q, const void *k, const void *v,
                        const void *tq, const void *tk, const void *tv,
                        void *o, void *to, float *lse,
                        int64_t B, int64_t H, int64_t Lq, int64_t Lk, int64_t d,
                        float scale, void *stream);

/*
 * attn_jvp_fwd_f32out_causal -- attn_jvp_fwd_f32out with the causal mask of
 * attn_jvp_fwd_causal (rows that see no key: O = tO = 0, lse = -infinity);
 * arguments and rules as attn_jvp_fwd_f32out.  The pages describe neither
 * masks nor this variant; it is the masked definition with the tangent
 * carried as attn_jvp_fwd_f32out carries it.
 */
AJVP_API int attn_jvp_fwd_f32out_causal(const void *q, const void *k, const void *v,
                        const void *tq, const void *tk, const void *tv,
                        float *o, float *to, float *lse,
                        int64_t B, int64_t H, int64_t Lq, int64_t Lk, int64_t d,
                        float scale, void *stream);

/*
 * attn_jvp_fwd_varlen -- packed variable-length sequences (for example text
 * conditions of different lengths in one batch), optionally causal.
 *
 *   q, tq, o, to        : __nv_bfloat16 [H][total_q][d]
 *   k, v, tk, tv        : __nv_bfloat16 [H][total_k][d]
 *   lse                 : float [H][total_q], or NULL
 *   cu_seqlens_q / _k   : DEVICE int32 arrays of n_seq + 1 non-decreasing
 *                         offsets, first 0, last total_q / total_k: sequence
 *                         b is query rows cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1
 *                         and keys cu_seqlens_k[b] .. cu_seqlens_k[b+1]-1 of
 *                         every head
 *   max_seqlen_q        : at least the longest query sequence (sets the grid;
 *                         rows of longer sequences would not be computed)
 *   causal              : 0, or the causal rule of attn_jvp_fwd_causal inside
 *                         each sequence
 *
 * Attention never crosses sequences.  A sequence with no keys (or a causal
 * row with none visible) gives O = tO = 0 and lse = -infinity.  Offsets
 * outside [0, total] are clamped in the kernel (memory-safe; the results of
 * such a call are unspecified).  Supported: d == 128, total_k >= 1, the
 * tensors 16-byte and the offset arrays 4-byte aligned; other rules as
 * attn_jvp_fwd.  n_seq == 0, max_seqlen_q == 0 or total_q == 0 is a no-op.
 */
AJVP_API int attn_jvp_fwd_varlen(const void *q, const void *k, const void *v,
                        const void *tq, const void *tk, const void *tv,
                        void *o, void *to, float *lse,
                        const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                        int64_t n_seq, int64_t H, int64_t total_q, int64_t total_k,
                        int64_t max_seqlen_q, int64_t d, float scale, int causal,
                        void *stream);

/*
 * attn_jvp_fwd_f32out_varlen -- attn_jvp_fwd_varlen with fp32 outputs
 * o, to (float [H][total_q][d]), as attn_jvp_fwd_f32out computes them;
 * other arguments and rules as attn_jvp_fwd_varlen (rows past a sequence's
 * end are never written, empty rows give zeros and lse = -infinity).
 */
AJVP_API int attn_jvp_fwd_f32out_varlen(const void *q, const void *k, const void *v,
                        const void *tq, const void *tk, const void *tv,
                        float *o, float *to, float *lse,
                        const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                        int64_t n_seq, int64_t H, int64_t total_q, int64_t total_k,
                        int64_t max_seqlen_q, int64_t d, float scale, int causal,
                        void *stream);

/*
 * attn_jvp_fwd_stats -- attn_jvp_fwd that also saves, per query row, the
 * statistic mu_i = sum_j P_ij dS_ij (fp32 [B][H][Lq]) that attn_jvp_bwd needs
 * beside lse.  lse and mu are required (non-NULL, 16-byte aligned); all
 * other arguments and rules as attn_jvp_fwd.
 */
AJVP_API int attn_jvp_fwd_stats(const void *q, const void *k, const void *v,
                       const void *tq, const void *tk, const void *tv,
                       void *o, void *to, float *lse, float *mu,
                       int64_t B, int64_t H, int64_t Lq, int64_t Lk, int64_t d,
                       float scale, void *stream);

/*
 * attn_jvp_bwd -- backward pass of attn_jvp_fwd: the gradients of
 *
 *     L = sum <dout, O> + sum <dtout, tO>
 *
 * with respect to q, k, v and the tangents tq, tk, tv (rCM trains through
 * its fused attention + JVP kernel; the pages describe its forward pass
 * only, and this is the gradient of that forward definition).
 *
 *   q, k, v, tq, tk, tv : the forward's bf16 inputs (layouts as attn_jvp_fwd)
 *   o, to               : the forward's bf16 outputs [B][H][Lq][d]
 *   lse, mu             : the forward's float row statistics [B][H][Lq]
 *                         (attn_jvp_fwd_stats)
 *   dout, dtout         : bf16 cotangents of O and tO, [B][H][Lq][d]
 *   dq, dtq             : bf16 [B][H][Lq][d] (written)
 *   dk, dv, dtk, dtv    : bf16 [B][H][Lk][d] (written)
 *   workspace           : DEVICE memory owned by the caller, 256-byte aligned,
 *                         at least attn_jvp_bwd_workspace_bytes(B, H, Lq)
 *                         bytes; nothing in it needs to start at zero
 *
 * Four kernels on `stream`: per-row statistics into the workspace, then
 * three gradient kernels (tcgen05: dq and dtq; dk and dtk; dv and dtv), each
 * owning its outputs (no atomics: results are deterministic).  With a
 * workspace of attn_jvp_bwd_workspace_bytes_split bytes the dk/dtk and
 * dv/dtv kernels may split short key sequences over several CTAs, each
 * followed by an ordered reduction kernel (six kernels in all).  Gradients are
 * accumulated in fp32 and rounded to bf16 (round-to-nearest-even).
 * Supported: d == 128, every pointer non-NULL and 16-byte aligned, sizes as
 * attn_jvp_fwd.  B*H == 0 is a no-op; Lq == 0 writes zeros to dk, dv, dtk,
 * dtv.  Outputs must not alias inputs.  Errors as attn_jvp_fwd plus
 * AJVP_ERR_WORKSPACE.
 */
AJVP_API int attn_jvp_bwd(const void *q, const void *k, const void *v,
                 const void *tq, const void *tk, const void *tv,
                 const void *o, const void *to, const float *lse, const float *mu,
                 const void *dout, const void *dtout,
                 void *dq, void *dk, void *dv, void *dtq, void *dtk, void *dtv,
                 int64_t B, int64_t H, int64_t Lq, int64_t Lk, int64_t d,
                 float scale, void *workspace, uint64_t workspace_bytes, void *stream);

/*
 * attn_jvp_bwd_step -- one of attn_jvp_bwd's four kernels, for callers that
 * schedule them (or time them) separately: step 0 writes the row
 * statistics into the workspace, step 1 dq and dtq, step 2 dk and dtk,
 * step 3 dv and dtv.  Steps 1-3 read the workspace step 0 wrote (same
 * inputs, same workspace, ordered after it); they are independent of each
 * other.  Arguments, checks and errors as attn_jvp_bwd (every pointer is
 * checked, even those a step does not touch); AJVP_ERR_INVALID_ARG for a
 * step outside 0..3.
 */
AJVP_API int attn_jvp_bwd_step(int step, const void *q, const void *k, const void *v,
                      const void *tq, const void *tk, const void *tv,
                      const void *o, const void *to, const float *lse, const float *mu,
                      const void *dout, const void *dtout,
                      void *dq, void *dk, void *dv, void *dtq, void *dtk, void *dtv,
                      int64_t B, int64_t H, int64_t Lq, int64_t Lk, int64_t d,
                      float scale, void *workspace, uint64_t workspace_bytes, void *stream);

/*
 * attn_jvp_fwd_causal_stats -- attn_jvp_fwd_causal that also saves mu (as
 * attn_jvp_fwd_stats does for the unmasked forward): the statistics
 * attn_jvp_bwd_causal needs.  Rows that see no key get lse = -infinity and
 * mu = 0.  lse and mu are required; other arguments and rules as
 * attn_jvp_fwd_causal.
 */
AJVP_API int attn_jvp_fwd_causal_stats(const void *q, const void *k, const void *v,
                       const void *tq, const void *tk, const void *tv,
                       void *o, void *to, float *lse, float *mu,
                       int64_t B, int64_t H, int64_t Lq, int64_t Lk, int64_t d,
                       float scale, void *stream);

/*
 * attn_jvp_bwd_causal -- backward pass of attn_jvp_fwd_causal: the gradients
 * of L = sum <dout, O> + sum <dtout, tO> where O, tO are the causal forward's
 * outputs (key j visible to query row i iff j <= i + (Lk - Lq)).  The pages
 * describe neither masks nor the backward; this is the gradient of the
 * masked forward definition, with every sum over keys taken over the keys a
 * row sees.  o, to, lse, mu come from attn_jvp_fwd_causal_stats.  Each
 * gradient kernel streams only the tiles some row of its own tile sees
 * (about half the work of attn_jvp_bwd when Lq == Lk); gradients of rows
 * that see no key, and of keys no row sees, are zero.  Arguments, layouts,
 * workspace, checks and errors as attn_jvp_bwd, plus AJVP_ERR_TOO_LARGE for
 * Lq or Lk >= 2^30.
 */
AJVP_API int attn_jvp_bwd_causal(const void *q, const void *k, const void *v,
                 const void *tq, const void *tk, const void *tv,
                 const void *o, const void *to, const float *lse, const float *mu,
                 const void *dout, const void *dtout,
                 void *dq, void *dk, void *dv, void *dtq, void *dtk, void *dtv,
                 int64_t B, int64_t H, int64_t Lq, int64_t Lk, int64_t d,
                 float scale, void *workspace, uint64_t workspace_bytes, void *stream);

/*
 * attn_jvp_fwd_varlen_stats -- attn_jvp_fwd_varlen that also saves mu
 * (float [H][total_q]), the statistics attn_jvp_bwd_varlen needs beside lse.
 * Rows that see no key get lse = -infinity and mu = 0.  lse and mu are
 * required; other arguments and rules as attn_jvp_fwd_varlen.
 */
AJVP_API int attn_jvp_fwd_varlen_stats(const void *q, const void *k, const void *v,
                       const void *tq, const void *tk, const void *tv,
                       void *o, void *to, float *lse, float *mu,
                       const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                       int64_t n_seq, int64_t H, int64_t total_q, int64_t total_k,
                       int64_t max_seqlen_q, int64_t d, float scale, int causal,
                       void *stream);

/*
 * attn_jvp_bwd_varlen -- backward pass of attn_jvp_fwd_varlen (packed
 * variable-length sequences, optionally causal inside each sequence): the
 * gradients of L = sum <dout, O> + sum <dtout, tO>.  The pages describe
 * neither packed batches nor the backward; this is the gradient of the
 * packed forward definition, attention never crossing sequences.
 *
 *   q, tq, o, to, dout, dtout, dq, dtq : __nv_bfloat16 [H][total_q][d]
 *   k, v, tk, tv, dk, dv, dtk, dtv     : __nv_bfloat16 [H][total_k][d]
 *   lse, mu             : float [H][total_q] (attn_jvp_fwd_varlen_stats)
 *   cu_seqlens_q / _k, n_seq, causal   : as attn_jvp_fwd_varlen
 *   max_seqlen_q / _k   : at least the longest query / key sequence (they
 *                         set the grids; rows of longer sequences would not
 *                         be computed)
 *   workspace           : DEVICE memory, 256-byte aligned, at least
 *                         attn_jvp_bwd_workspace_bytes(1, H, total_q) bytes
 *
 * Gradients of rows that see no key, and of keys that no row sees (a
 * sequence without queries), are zero; rows outside every sequence are not
 * written.  Offsets outside [0, total] are clamped in the kernels
 * (memory-safe; such a call's results are unspecified).  total_q == 0 writes
 * zeros to dk, dv, dtk, dtv.  Supported: d == 128, total_k >= 1, tensors
 * 16-byte and offset arrays 4-byte aligned; workspace, checks and errors as
 * attn_jvp_bwd, plus AJVP_ERR_TOO_LARGE for total_q or total_k >= 2^30.
 */
AJVP_API int attn_jvp_bwd_varlen(const void *q, const void *k, const void *v,
                 const void *tq, const void *tk, const void *tv,
                 const void *o, const void *to, const float *lse, const float *mu,
                 const void *dout, const void *dtout,
                 void *dq, void *dk, void *dv, void *dtq, void *dtk, void *dtv,
                 const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                 int64_t n_seq, int64_t H, int64_t total_q, int64_t total_k,
                 int64_t max_seqlen_q, int64_t max_seqlen_k, int64_t d,
                 float scale, int causal, void *workspace, uint64_t workspace_bytes,
                 void *stream);

/* Device workspace, in bytes, that attn_jvp_bwd needs (0 for invalid sizes). */
AJVP_API uint64_t attn_jvp_bwd_workspace_bytes(int64_t B, int64_t H, int64_t Lq);

/*
 * attn_jvp_bwd_workspace_bytes_split -- the workspace with which
 * attn_jvp_bwd (and attn_jvp_bwd_step) may split the query range of its two
 * key-side kernels (dk, dtk and dv, dtv) over several CTAs per 128-key tile:
 * when the key tiles alone cannot fill the current device (short key
 * sequences, such as cross-attention to a few hundred text tokens), each
 * part writes fp32 partial sums to the workspace (one region for dk/dtk,
 * one for dv/dtv, so that attn_jvp_bwd_step's steps 2 and 3 stay
 * independent) and a reduction adds them up in part order (the result stays
 * deterministic, though not bit-identical to the unsplit kernels).  At least attn_jvp_bwd_workspace_bytes; equal to
 * it when no split applies.  Reads the current device's SM count (the
 * minimum is returned when no usable device is current).  A call whose
 * workspace is smaller than this runs the unsplit kernels.
 */
AJVP_API uint64_t attn_jvp_bwd_workspace_bytes_split(int64_t B, int64_t H, int64_t Lq, int64_t Lk);

/*
 * attn_jvp_bwd_key_split_parts -- the number of parts (1 = no split) into
 * which attn_jvp_bwd, given the split workspace, cuts the query range of
 * its key-side kernels on a device with `sm_count` SMs.  Pure host
 * arithmetic (no CUDA call).  Splits only when the 128-key tiles give
 * fewer than four CTAs per SM; the count (at most 16, at most the number
 * of 64-query tiles) minimises a wave model of the run time:
 * ceil(key CTAs x parts / SMs) waves, each as long as one part's query
 * tiles plus about eight tiles of fixed cost per CTA, times 1 + parts / 100;
 * ties go to fewer parts, so no part is empty.  Returns 0 for negative
 * sizes or an sm_count outside 1 .. 2^20.
 */
AJVP_API int64_t attn_jvp_bwd_key_split_parts(int64_t B, int64_t H, int64_t Lq, int64_t Lk, int64_t sm_count);

/*
 * attn_jvp_bwd_host -- attn_jvp_bwd on HOST buffers: every tensor argument
 * (the twelve inputs, lse and mu included, and the six gradients) is host
 * memory in the layouts of attn_jvp_bwd; pinned memory gives overlapped
 * transfers, pageable memory works but copies synchronously.  (batch, head)
 * slabs are processed in chunks through `workspace`, DEVICE memory owned by
 * the caller, 256-byte aligned, at least
 * attn_jvp_bwd_host_workspace_bytes(Lq, Lk, d, 1) bytes (a larger one allows
 * chunks of several heads, at most a quarter of B*H): each chunk is copied in
 * on one internal stream, its four backward kernels run on one of two
 * others, and its gradients are copied back on a fourth, so copies overlap
 * the kernels of neighbouring chunks.  Results are identical to attn_jvp_bwd
 * on the same data with a workspace of attn_jvp_bwd_workspace_bytes (the
 * chunks' key-side kernels never split).  Stream-ordered with respect to `stream` (the call
 * returns once everything is enqueued; the host buffers must stay valid and
 * unchanged until `stream` reaches that point).  Lq == 0 writes zeros to dk,
 * dv, dtk, dtv on the host after synchronising `stream`.  Errors as
 * attn_jvp_bwd; AJVP_ERR_WORKSPACE for a missing, misaligned or too small
 * workspace.  On an error after work was enqueued, the call waits for that
 * work to finish before returning.
 */
AJVP_API int attn_jvp_bwd_host(const void *q, const void *k, const void *v,
                      const void *tq, const void *tk, const void *tv,
                      const void *o, const void *to, const float *lse, const float *mu,
                      const void *dout, const void *dtout,
                      void *dq, void *dk, void *dv, void *dtq, void *dtk, void *dtv,
                      int64_t B, int64_t H, int64_t Lq, int64_t Lk, int64_t d,
                      float scale, void *workspace, uint64_t workspace_bytes, void *stream);

/* Device workspace, in bytes, for attn_jvp_bwd_host with chunks of
 * `heads_per_chunk` (batch, head) slabs (0 for invalid sizes). */
AJVP_API uint64_t attn_jvp_bwd_host_workspace_bytes(int64_t Lq, int64_t Lk, int64_t d, int64_t heads_per_chunk);

/*
 * attn_jvp_fwd_f32 -- fp32 I/O, fp32 arithmetic (CUDA-core kernel), for the
 * accuracy-critical configuration.  Same math, layout and error rules as
 * attn_jvp_fwd, with float tensors.  Supported: 1 <= d <= 256; pointers
 * 4-byte aligned.  Any compute capability 10.0 device.
 */
AJVP_API int attn_jvp_fwd_f32(const float *q, const float *k, const float *v,
                     const float *tq, const float *tk, const float *tv,
                     float *o, float *to, float *lse,
                     int64_t B, int64_t H, int64_t Lq, int64_t Lk, int64_t d,
                     float scale, void *stream);

/*
 * attn_jvp_fwd_host -- the attn_jvp_fwd computation on HOST buffers.
 *
 *   q, k, v, tq, tk, tv : host __nv_bfloat16 arrays, layouts as attn_jvp_fwd
 *   o, to               : host __nv_bfloat16 [B][H][Lq][d] (written)
 *   lse                 : host float [B][H][Lq], or NULL
 *   workspace           : DEVICE memory owned by the caller, 256-byte aligned,
 *                         at least attn_jvp_host_workspace_bytes(Lq, Lk, d, 1)
 *   workspace_bytes     : its size
 *
 * The (batch, head) slabs are processed in chunks of consecutive heads: while
 * the kernel runs on one chunk, the next chunk's inputs are copied in and the
 * previous chunk's outputs copied out (three staging buffers in the
 * workspace used in turn; four internal streams: copy in, two compute
 * streams taken in turn so that consecutive chunk kernels may overlap, copy
 * out).  Chunk size: as many heads as three buffers in the workspace hold, at
 * most a quarter of B*H (rounded up).
 * Host buffers should be page-locked; pageable memory works but copies then
 * do not overlap.  Stream-ordered on `stream` like attn_jvp_fwd: the work
 * starts after what is already queued on `stream`, and work queued on
 * `stream` afterwards (e.g. a synchronisation) sees the host outputs written.
 * The internal streams and events are created and released per call, so the
 * call must not be made while `stream` is being captured into a CUDA graph.
 * On an error after work was enqueued, the call waits for that work to
 * finish before returning, so nothing of it still touches the workspace.
 * Same size, device and error rules as attn_jvp_fwd, plus AJVP_ERR_WORKSPACE.
 */
AJVP_API int attn_jvp_fwd_host(const void *q, const void *k, const void *v,
                      const void *tq, const void *tk, const void *tv,
                      void *o, void *to, float *lse,
                      int64_t B, int64_t H, int64_t Lq, int64_t Lk, int64_t d,
                      float scale, void *workspace, uint64_t workspace_bytes,
                      void *stream);

/*
 * Device workspace, in bytes, that attn_jvp_fwd_host needs to stage chunks
 * of `heads_per_chunk` (batch, head) slabs (three staging buffers, every
 * array 256-byte aligned).  Returns 0 for invalid sizes.
 */
AJVP_API uint64_t attn_jvp_host_workspace_bytes(int64_t Lq, int64_t Lk, int64_t d,
                                       int64_t heads_per_chunk);

/*
 * attn_jvp_fwd_host_noalloc -- attn_jvp_fwd_host without a caller-supplied
 * workspace: the chunks are staged in a static device array of the library
 * (64 MiB per device, reserved when the library's device code is loaded on
 * that device).  The pages have no counterpart: it exists for callers that
 * cannot hand the library device memory (see attn_jvp_fwd_host for the
 * computation, layouts and the host-buffer contract).
 *
 *   q, k, v, tq, tk, tv : host __nv_bfloat16 arrays, layouts as attn_jvp_fwd
 *   o, to               : host __nv_bfloat16 [B][H][Lq][d] (written)
 *   lse                 : host float [B][H][Lq], or NULL
 *
 * Maximum size: one (batch, head) slab in three staging buffers must fit the
 * 64 MiB, i.e. attn_jvp_host_workspace_bytes(Lq, Lk, d, 1) <= 67108864
 * (for d = 128 about Lq + Lk <= 21800); larger sizes return
 * AJVP_ERR_TOO_LARGE before anything is enqueued.  Chunks hold as many heads
 * as fit, at most a quarter of B*H.
 * A call allocates nothing: no cudaMalloc, cudaFree or allocating library
 * call, and no stream or event is created or destroyed.  The first call on a
 * device does a one-time set-up there, with that device current: it looks up
 * the array's device address (cudaGetSymbolAddress) and creates the
 * pipeline's four internal streams and ten events, which every later call on
 * the device reuses and which are kept until the process exits; make that
 * first call before any stream capture begins.  If the set-up fails, that
 * call and every later one on the device return AJVP_ERR_CUDA.  Nothing in
 * the array needs to start at zero.  The array is shared by every call on
 * the device: calls on one stream are ordered and safe, but calls on
 * different streams whose executions overlap race on it and give undefined
 * results; serialise them.  Calls from several host threads enqueue their
 * work one at a time.  On an error after work was enqueued, the call waits
 * for that work to finish before returning.  Other rules as
 * attn_jvp_fwd_host.
 */
AJVP_API int attn_jvp_fwd_host_noalloc(const void *q, const void *k, const void *v,
                              const void *tq, const void *tk, const void *tv,
                              void *o, void *to, float *lse,
                              int64_t B, int64_t H, int64_t Lq, int64_t Lk, int64_t d,
                              float scale, void *stream);

/* Static, human-readable description of an ajvp_status value. */
AJVP_API const char *attn_jvp_strerror(int status);

/* cudaError_t behind the calling thread's last AJVP_ERR_CUDA (0 if none). */
AJVP_API int attn_jvp_last_cuda_error(void);

/*
 * Synchronise `stream`, then read and clear the device status word of the
 * current device.  Returns AJVP_OK, AJVP_ERR_TIMEOUT (some kernel wait ran
 * past its bound since the last check), AJVP_ERR_DEVICE_LAYOUT (a backward
 * kernel or the persistent forward found its dynamic shared memory not
 * 1024-byte aligned and returned without work) or AJVP_ERR_CUDA.
 */
AJVP_API int attn_jvp_check_device_status(void *stream);

/*
 * Bound, in nanoseconds, on any single pipeline wait inside the kernels
 * (default 2e9, i.e. 2 s; 0 restores the default).  Applies to launches made
 * after the call, process-wide.
 */
AJVP_API int attn_jvp_set_wait_bound_ns(uint64_t ns);

/*
 * Scheduling of the bf16 forward entry points without masks (attn_jvp_fwd,
 * attn_jvp_fwd_stats, the host entries): when the keys span at least 3 and
 * at most `max_key_tiles` tiles of 64 and there are more 128-row query tiles
 * than SMs, one persistent CTA per SM walks the query tiles and overlaps each
 * tile's epilogue with the next tile's loads and score products (short key
 * sequences, e.g. cross-attention to a few hundred text tokens).  Results are
 * bit-identical either way.  Default 32; 0 turns the persistent form off;
 * negative values are rejected (AJVP_ERR_INVALID_ARG).  Applies to launches
 * made after the call, process-wide.
 */
AJVP_API int attn_jvp_set_persistent_key_tiles(int64_t max_key_tiles);

/*
 * Scheduling of the backward's unmasked dQ/dtQ and dK/dtK kernels (steps 1
 * and 2 of attn_jvp_bwd, attn_jvp_bwd_step and attn_jvp_bwd_host, without a
 * split key side): with `on` != 0 two CTAs on two SMs of a cluster share
 * each tensor-core product (cta_group::2, 256 rows per product), each
 * holding its own 128 rows and half of each streamed operand; with 0 (the
 * default) every CTA works alone.  The pairs read half the shared-memory B
 * operand per product, which on B200 bought no time (both kernels 4-5 %
 * slower: the tensor pipe is not bound by the operand reads there, and the
 * pairs tie each tile to two SMs).  The two forms add the same products in
 * a different order within a tile, so results agree to rounding, not bit
 * for bit.
 * Applies to launches made after the call, process-wide.  Returns AJVP_OK.
 * A scheduling choice with no counterpart in the method.
 */
AJVP_API int attn_jvp_set_bwd_pairs(int on);

/*
 * Failure-detection self test: enqueue a one-warp kernel that waits, through
 * the same bounded-wait routine the attention kernel uses, on a barrier that
 * nothing ever completes, with a bound of `bound_ns`.  The kernel gives up,
 * records AJVP_ERR_TIMEOUT in the device status word and returns; the GPU
 * context stays usable.  Returns AJVP_OK once enqueued.
 */
AJVP_API int attn_jvp_selftest_wait_timeout(uint64_t bound_ns, void *stream);

/* Library version, major * 10000 + minor * 100 + patch. */
AJVP_API int attn_jvp_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_JVP_H */
