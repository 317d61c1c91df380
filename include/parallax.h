/*
 * parallax.h -- C ABI of the Parallax attention library (B200, sm_100a).
 *
 * Parallax keeps exact softmax attention and subtracts the softmax-weighted
 * key/value covariance projected by a learned probe rho_i = W_R x_i
 * (zubnet.ai news item on Parallax, paragraph 2; encorp.ai blog "Integraciones
 * de IA personalizadas tras la atencion Parallax", section "Por que eliminar el
 * solucionador de gradiente conjugado..."):
 *
 *   z_ij = q_i . k_j / sqrt(d),  s_ij = softmax_j(z_ij) over the visible keys
 *   o_i  = sum_j s_ij v_j,  a_ij = k_j . rho_i,  abar_i = sum_j s_ij a_ij,
 *   m_i  = sum_j s_ij a_ij v_j
 *   y_i  = o_i - C_i rho_i = o_i - (m_i - o_i abar_i)
 *
 * With rho = 0 (W_R = 0) the result is plain softmax attention exactly (same
 * passages, and the encorp.ai FAQ on converting a pretrained Transformer).
 *
 * Conventions for every call:
 *   - Tensors are caller-owned, contiguous, row-major DEVICE memory unless a
 *     parameter says otherwise.  The library never frees or keeps them.
 *   - Every device pointer must be 16-byte aligned (TMA and 128-bit loads).
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls only
 *     enqueue work on it and return; results are ready when the stream is.
 *   - A host-detectable error (null pointer, bad size, misalignment, an
 *     unsupported dtype pair) returns a nonzero parallax_status_t and enqueues
 *     nothing.  A failed launch returns PARALLAX_ERR_CUDA.  The library never
 *     prints, never aborts and never falls back to another implementation.
 *   - Device-side waits are bounded.  A wait that gives up records
 *     PARALLAX_ERR_DEVICE_TIMEOUT in a per-device error word and the kernel
 *     returns; an out-of-range page id met by the paged decode records
 *     PARALLAX_ERR_DEVICE_INDEX there, and a non-finite prefill output
 *     PARALLAX_ERR_DEVICE_RANGE.  Read (and clear) it with
 *     parallax_last_device_error().
 *   - Scratch.  A call that needs scratch device memory (parallax_fwd and its
 *     variants on the tensor-core path: a work counter and a block-scaled fp16
 *     copy of V; parallax_decode, parallax_softmax_decode and
 *     parallax_decode_paged: the split partials; parallax_bwd: its work
 *     counters and per-row statistics) takes it
 *     for that call alone from a library-owned, per-device stream-ordered
 *     memory pool
 *     (cudaMallocFromPoolAsync on `stream`) and returns it with cudaFreeAsync
 *     on `stream` once its kernels are enqueued.  Calls may therefore run
 *     concurrently on different streams and be made from several host threads
 *     at once: no two calls share scratch, and nothing is freed while a kernel
 *     may still use it.  The pool keeps returned memory for later calls.
 *     parallax_decode_ex (caller's workspace) and parallax_decode_noalloc
 *     (static array) do not use the pool.
 */
#ifndef PARALLAX_H
#define PARALLAX_H

#include <stddef.h>

#if defined(__GNUC__)
#define PARALLAX_API __attribute__((visibility("default")))
#else
#define PARALLAX_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef void *parallax_stream_t; /* a cudaStream_t */

typedef enum {
    PARALLAX_F32 = 0,  /* IEEE binary32 */
    PARALLAX_BF16 = 1  /* bfloat16 */
} parallax_dtype_t;

typedef enum {
    PARALLAX_OK = 0,
    PARALLAX_ERR_NULL = 1,           /* a required pointer is NULL */
    PARALLAX_ERR_SHAPE = 2,          /* a size is out of range */
    PARALLAX_ERR_ALIGN = 3,          /* a pointer is not 16-byte aligned */
    PARALLAX_ERR_DTYPE = 4,          /* unsupported dtype or dtype pair */
    PARALLAX_ERR_UNSUPPORTED = 5,    /* valid request this build does not serve */
    PARALLAX_ERR_CUDA = 6,           /* a CUDA runtime/driver call failed */
    PARALLAX_ERR_DEVICE_TIMEOUT = 7, /* a device-side wait gave up */
    PARALLAX_ERR_DEVICE_INDEX = 8,   /* a device-side index (a page id) was out of range */
    PARALLAX_ERR_DEVICE_RANGE = 9    /* a result was not finite: an input outside the kernel's range */
} parallax_status_t;

/*
 * parallax_fwd -- prefill / forward over whole sequences.
 *
 * Passage: zubnet.ai news item on Parallax, paragraph 2 (output = softmax
 * attention minus the probe-projected KV covariance; both branches reuse one
 * KV stream); encorp.ai blog, section "Como cambia Parallax la historia del
 * hardware en GPU Hopper" (same KV streaming structure as FlashAttention).
 *
 *   q, k, v, rho : [B, H, T, d] of in_dtype.  rho == NULL selects the
 *                  softmax-only instantiation of the same kernel (y = o); with
 *                  rho all zeros the result is bitwise equal to that.
 *   y            : [B, H, T, d] of out_dtype (written).
 *   lse          : [B, H, T] fp32, natural-log log-sum-exp of the scaled scores
 *                  z_ij of each row (written); may be NULL.
 *   B, H >= 1; T >= 1; d in {64, 128}.
 *   causal       : nonzero -> query i sees keys 0..i; zero -> all T keys.
 *   in_dtype/out_dtype:
 *     F32  -> F32   fp32 CUDA-core kernel (fp32 arithmetic throughout)
 *     BF16 -> F32   tensor-core kernel (tcgen05), fp32 accumulation
 *     BF16 -> BF16  same kernel, y rounded to bf16 on store
 *   Tensor-core path: d in {64, 128}.  The P.V products run on fp16 operands:
 *   V is converted to fp16 with a power-of-two scale per block of 64 keys,
 *   which keeps fp16 precision for |v| from about 1e-5 (smaller values lose
 *   precision gradually) up to |v| < 2^23; the correction weights
 *   P o (k_j . rho_i) / 256 are staged in fp16, so |k_j . rho_i| < 65504
 *   (divided by 2^e in a block where V needed a scale 2^-e, e <= 7).  A
 *   non-finite output (an input outside these ranges, or a non-finite input)
 *   sets PARALLAX_ERR_DEVICE_RANGE in the device error word.  Scratch: 2 bytes
 *   per V element plus a few bytes (see the conventions above).
 */
PARALLAX_API int parallax_fwd(const void *q, const void *k, const void *v, const void *rho,
                 void *y, float *lse, int B, int H, int T, int d, int causal,
                 int in_dtype, int out_dtype, parallax_stream_t stream);

/*
 * parallax_fwd_fused -- parallax_fwd with the probe computed inside the kernel.
 *
 * Passage: encorp.ai blog, section "Por que eliminar el solucionador de
 * gradiente conjugado..." (the probe comes from a learned projector W_R of the
 * layer input), zubnet.ai news item on Parallax, paragraph 2 (rho_i = W_R x_i).
 * Instead of reading rho from memory, each 128-row query tile of a head
 * computes its probe tile rho = x[b, rows, :] W_R[:, h*d:(h+1)*d] on the tensor
 * cores (fp32 accumulation over d_model, rounded to bf16 as parallax_rho_proj
 * rounds it) and keeps it on chip; rho never goes to HBM.
 *
 *   q, k, v : [B, H, T, d] bf16;  x : [B, T, d_model] bf16 (the layer input);
 *   W_R     : [d_model, H*d] bf16 row-major (column block h is head h).
 *   y, lse, causal, out_dtype: as parallax_fwd.
 *   d == 128 (PARALLAX_ERR_UNSUPPORTED otherwise); d_model a multiple of 64.
 *   in_dtype must be BF16.  Scratch as parallax_fwd.
 * With W_R = 0 the result is bitwise the softmax-only result of parallax_fwd.
 */
PARALLAX_API int parallax_fwd_fused(const void *q, const void *k, const void *v, const void *x, const void *W_R,
                                    void *y, float *lse, int B, int H, int T, int d, int d_model, int causal,
                                    int in_dtype, int out_dtype, parallax_stream_t stream);

/*
 * parallax_fwd_train -- parallax_fwd that also keeps what the backward needs.
 *
 * Same operator and tensor-core kernel as parallax_fwd (bf16 inputs, fp32 y),
 * and also writes, per row, the softmax attention output o_i = sum_j s_ij v_j
 * and abar_i = sum_j s_ij a_ij.
 *   q, k, v, rho : [B, H, T, d] bf16 (rho required).
 *   y, o         : [B, H, T, d] fp32 (written);  lse, abar : [B, H, T] fp32 (written).
 *   d in {64, 128}; in_dtype must be BF16.  Scratch as parallax_fwd.
 */
PARALLAX_API int parallax_fwd_train(const void *q, const void *k, const void *v, const void *rho, float *y,
                                    float *lse, float *o, float *abar, int B, int H, int T, int d, int causal,
                                    int in_dtype, parallax_stream_t stream);

/*
 * parallax_bwd -- gradients of the prefill with respect to q, k, v and rho.
 *
 * The pages train with this operator (encorp.ai blog, section "Las ganancias
 * de preentrenamiento..."; zubnet.ai news item on Parallax, paragraph 1); the
 * gradients are the chain rule through the definitions above, for a loss L
 * with dL/dy = dy.  Chain to W_R through rho = x W_R with the caller's GEMMs.
 *   q, k, v, rho, dy : [B, H, T, d] bf16.
 *   y, o, abar, lse  : the outputs of parallax_fwd_train on the same inputs.
 *   dq, dk, dv, drho : [B, H, T, d] fp32 (written, not accumulated).
 *   d in {64, 128}; B * H <= 65535; in_dtype must be BF16.
 * tcgen05 tensor-core kernels: one over 128-query tiles for dq and drho, one
 * over 128-key tiles for dk and dv, both recomputing the scores, so no gradient
 * is accumulated with atomics and the result is deterministic.
 * Scratch (see the conventions above): 256 bytes of work counters, 8 bytes per
 * row (g.o and delta), and 16 bytes per row of packed per-query statistics with
 * T rounded up to a multiple of 64 per head.
 */
PARALLAX_API int parallax_bwd(const void *q, const void *k, const void *v, const void *rho, const float *y,
                              const float *o, const float *abar, const float *lse, const void *dy, float *dq,
                              float *dk, float *dv, float *drho, int B, int H, int T, int d, int causal,
                              int in_dtype, parallax_stream_t stream);

/*
 * parallax_decode -- one new query token per sequence against a KV cache.
 *
 * Passage: zubnet.ai news item on Parallax, paragraph 2 (the KV cache is still
 * required for decoding; the decode kernel reuses one KV stream for both
 * branches, which doubles the arithmetic intensity).
 *
 *   q, rho         : [B, H, d] bf16 (the current token's query and probe).
 *   kcache, vcache : [B, H, Tcap, d] bf16; rows 0..seqlens[b]-1 are valid and
 *                    already include the current token's key and value.
 *   seqlens        : DEVICE int32 [B], 0 <= seqlens[b] <= Tcap (not read on the
 *                    host; an empty sequence yields y = 0, lse = -inf).
 *   y              : [B, H, d] of out_dtype (F32 or BF16).
 *   lse            : [B, H] fp32, may be NULL.
 *   B, H >= 1; Tcap >= 1; d in {64, 128}; in_dtype must be BF16.
 * Split partials use per-call scratch from the library's pool (see the
 * conventions above); calls on different streams may overlap.  See
 * parallax_decode_ex for caller-provided scratch.
 */
PARALLAX_API int parallax_decode(const void *q, const void *rho, const void *kcache, const void *vcache,
                    const int *seqlens, void *y, float *lse, int B, int H, int Tcap, int d,
                    int in_dtype, int out_dtype, parallax_stream_t stream);

/*
 * parallax_softmax_decode -- plain softmax attention decode, the reference the
 * pages compare the Parallax decode with.
 *
 * Passage: encorp.ai blog, section "Como cambia Parallax la historia del
 * hardware en GPU Hopper", and zubnet.ai news item on Parallax, paragraph 2
 * (decode against FlashAttention 2/3, "compute-matched" and "I/O-matched").
 * The same split kernel as parallax_decode with the probe branch removed:
 * y = sum_j s_j v_j.  Head dims 64, 128 and 256: at the same d it reads the
 * same KV bytes as parallax_decode (I/O-matched); at 2d it does the same
 * arithmetic per cached token (compute-matched).
 *   q : [B, H, d] bf16;  kcache, vcache : [B, H, Tcap, d] bf16;
 *   seqlens, y, lse, dtypes and scratch as parallax_decode.
 */
PARALLAX_API int parallax_softmax_decode(const void *q, const void *kcache, const void *vcache, const int *seqlens,
                                         void *y, float *lse, int B, int H, int Tcap, int d, int in_dtype,
                                         int out_dtype, parallax_stream_t stream);

/* Bytes of scratch parallax_decode_ex needs for this shape on the current
 * device (0 if it needs none, or on a bad shape or CUDA error). */
PARALLAX_API size_t parallax_decode_workspace_bytes(int B, int H, int Tcap, int d);

/*
 * parallax_decode_ex -- parallax_decode with caller-provided scratch.
 *   workspace : device memory of at least parallax_decode_workspace_bytes(...)
 *               bytes, 256-byte aligned, not used concurrently by another call.
 *   Other arguments as parallax_decode.
 */
PARALLAX_API int parallax_decode_ex(const void *q, const void *rho, const void *kcache, const void *vcache,
                       const int *seqlens, void *y, float *lse, int B, int H, int Tcap, int d,
                       int in_dtype, int out_dtype, void *workspace, size_t workspace_bytes,
                       parallax_stream_t stream);

/*
 * parallax_decode_paged -- parallax_decode over a paged KV cache with grouped
 * query heads.
 *
 * The operator per query head is the one of parallax_decode (zubnet.ai news
 * item on Parallax, paragraph 2).  The pages describe neither paging nor
 * grouped heads; these are the layouts serving engines keep their caches in:
 * the cache is a pool of fixed-size pages that a per-sequence table maps, and
 * G = Hq / Hkv consecutive query heads share one key/value head (query head h
 * reads KV head h / G).
 *
 *   q, rho         : [B, Hq, d] bf16.
 *   kpages, vpages : [num_pages, Hkv, page_size, d] bf16.
 *   block_table    : DEVICE int32 [B, max_pages]; token t of sequence b is row
 *                    t % page_size of page block_table[b * max_pages + t / page_size].
 *                    Entries a sequence does not reach are not read.  An entry
 *                    outside [0, num_pages) that is reached is not followed: its
 *                    rows read as zero and the device error word is set to
 *                    PARALLAX_ERR_DEVICE_INDEX (see parallax_last_device_error).
 *   seqlens        : DEVICE int32 [B], 0 <= seqlens[b] <= max_pages * page_size.
 *   y              : [B, Hq, d] of out_dtype (F32 or BF16); lse [B, Hq] fp32 or NULL.
 *   B, Hkv >= 1; Hq a multiple of Hkv; page_size a power of two in [16, 4096];
 *   max_pages, num_pages >= 1; d in {64, 128}; in_dtype BF16.
 * Split partials use per-call scratch from the library's pool (see the
 * conventions above); calls on different streams may overlap.
 */
PARALLAX_API int parallax_decode_paged(const void *q, const void *rho, const void *kpages, const void *vpages,
                                       const int *block_table, const int *seqlens, void *y, float *lse, int B,
                                       int Hq, int Hkv, int page_size, int max_pages, int num_pages, int d,
                                       int in_dtype, int out_dtype, parallax_stream_t stream);

/*
 * parallax_decode_noalloc -- parallax_decode that never allocates device memory.
 *
 * The pages have no counterpart to this call.  It is for callers that must not
 * have a library allocate on their behalf: serving engines that reserve the
 * device's memory through their own pool at start-up and run under a fixed
 * budget, decode loops where a cudaMalloc, or the device-wide synchronization
 * of a cudaFree, would stall every stream, and plugin interfaces whose execute
 * callbacks forbid allocation.
 *
 * Same arguments, results and errors as parallax_decode.  The split partials
 * live in a static device array of PARALLAX_DECODE_NOALLOC_SCRATCH_BYTES
 * (16 MiB) compiled into the library; every GPU that loads the library holds
 * it until the process exits.  A shape whose partials need more than that
 * (parallax_decode_workspace_bytes tells) returns PARALLAX_ERR_SHAPE and
 * enqueues nothing.  The first call on a device looks up the array's device
 * address (cudaGetSymbolAddress) with that device current; make that first
 * call before any stream capture.  All calls on a device share the array and
 * it keeps the last call's contents (nothing in it needs clearing between
 * calls), so calls that overlap on the GPU, e.g. on two streams at once, race:
 * the caller must serialize them.
 */
#define PARALLAX_DECODE_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
PARALLAX_API int parallax_decode_noalloc(const void *q, const void *rho, const void *kcache,
                                         const void *vcache, const int *seqlens, void *y, float *lse,
                                         int B, int H, int Tcap, int d, int in_dtype, int out_dtype,
                                         parallax_stream_t stream);

/*
 * parallax_rho_proj -- the learned probe rho = x W_R, split per head.
 *
 * Passage: encorp.ai blog, section "Por que eliminar el solucionador de
 * gradiente conjugado..." (a learned projector W_R acting on the layer input
 * replaces the per-query solve); zubnet.ai, paragraph 2 (rho_i = W_R x_i).
 *
 *   x   : [B, T, d_model] bf16 (the layer input).
 *   W_R : [d_model, H*d] bf16 row-major (column block h*d..h*d+d-1 is head h).
 *   rho : [B, H, T, d] bf16 (written): rho[b,h,t,:] = x[b,t,:] @ W_R[:, h*d:(h+1)*d],
 *         fp32 accumulation, rounded to bf16 on store.  No bias.
 *   d_model % 64 == 0; (H*d) % 256 == 0; d in {64, 128}; dtype must be BF16.
 */
PARALLAX_API int parallax_rho_proj(const void *x, const void *W_R, void *rho, int B, int T, int d_model,
                      int H, int d, int dtype, parallax_stream_t stream);

/* Static English text for a status code (never NULL). */
PARALLAX_API const char *parallax_strerror(int status);

/*
 * Synchronizes `stream`, then returns and clears the device error word of the
 * current device: PARALLAX_OK, or PARALLAX_ERR_DEVICE_TIMEOUT when a kernel
 * gave up on a bounded wait since the last read.  Returns PARALLAX_ERR_CUDA if
 * the synchronization itself fails.
 */
PARALLAX_API int parallax_last_device_error(parallax_stream_t stream);

/* Number of SMs the library sizes its persistent grids for on the current device (0 on error). */
PARALLAX_API int parallax_device_sm_count(void);

#ifdef __cplusplus
}
#endif

#endif /* PARALLAX_H */
