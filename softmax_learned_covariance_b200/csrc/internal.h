// internal.h -- launch entry points shared between the host API and the kernels.
#pragma once
#include <atomic>
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "decode_plan.h"
#include "parallax.h"

namespace plx {

// Raises kernel `f`'s dynamic shared-memory limit to `bytes` once per device
// (function attributes belong to a device's context; `done` remembers the
// devices already set, for device ordinals below 64).
template <typename F> cudaError_t ensure_smem_limit(F f, int bytes, std::atomic<unsigned long long> &done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = dev < 64 ? 1ull << dev : 0ull;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_release);
    return e;
}

// Per-launch wait policy: absolute %globaltimer deadline is computed in-kernel
// from this budget (nanoseconds).
struct DeviceCtl {
    int *err;                       // device error word
    unsigned long long wait_ns;     // bound for every device-side wait
    unsigned int debug_flags;       // test hooks (see DEBUG_*), 0 in normal use
};
constexpr unsigned DEBUG_FWD_SKIP_FIRST_K_LOAD = 1u;   // fwd: never load the first K tile

// fp32 / bf16 CUDA-core forward (one warp per query row)
cudaError_t launch_fwd_simt(const void *q, const void *k, const void *v, const void *rho, void *y, float *lse,
                            int B, int H, int T, int d, int causal, int in_dtype, int out_dtype, cudaStream_t s);

// split-KV decode + combine (the split plan is in decode_plan.h)
cudaError_t launch_decode(const void *q, const void *rho, const void *kc, const void *vc, const int *seqlens,
                          void *y, float *lse, int B, int H, int Tcap, int d, int out_dtype, const DecodePlan &p,
                          float *partials, int sm_count, const DeviceCtl &ctl, cudaStream_t s);

// Plain softmax attention decode (no probe) with the same split kernel, d in
// {64, 128, 256}: the reference point the pages compare the decode with.
cudaError_t launch_softmax_decode(const void *q, const void *kc, const void *vc, const int *seqlens, void *y,
                                  float *lse, int B, int H, int Tcap, int d, int out_dtype, const DecodePlan &p,
                                  float *partials, cudaStream_t s);

// Paged KV layout for the decode: pages [num_pages, Hkv, 1 << pshift, d];
// query head h reads KV head h / group.
struct PagedKV {
    const int *table;   // [B, max_pages] page ids (device)
    int max_pages, num_pages, pshift, Hkv, group;
};
// Tensor-core split kernel of the paged decode (any Hq / Hkv); writes the same
// partials (or y when nsplit == 1) as the split decode kernel.
cudaError_t launch_decode_gqa_split(const void *q, const void *rho, const void *kpages, const void *vpages,
                                    const PagedKV &pg, const int *seqlens, void *y, float *lse, int B, int Hq, int d,
                                    int out_dtype, const DecodePlan &p, float *partials, int *err, cudaStream_t s);
cudaError_t launch_decode_paged(const void *q, const void *rho, const void *kpages, const void *vpages,
                                const PagedKV &pg, const int *seqlens, void *y, float *lse, int B, int Hq, int d,
                                int out_dtype, const DecodePlan &p, float *partials, const DeviceCtl &ctl,
                                cudaStream_t s);

// Wait policy and test hooks from the environment (PARALLAX_WAIT_TIMEOUT_MS,
// PARALLAX_DEBUG_FLAGS) around the given device error word.  No allocation.
DeviceCtl ctl_from_env(int *err);

// Device error word of the no-allocation decode entry point on the current
// device, or nullptr if that entry point has not been set up there.
int *noalloc_error_word();

// tcgen05 GEMM for rho = x W_R, scattered per head
cudaError_t launch_rho_proj(const CUtensorMap &tm_x, const CUtensorMap &tm_w, void *rho, int B, int T, int d_model,
                            int H, int d, int sm_count, const DeviceCtl &ctl, cudaStream_t s);

// V [B*H, T, d] bf16 -> fp16 in 64-key blocks, block b of head bh scaled by
// 2^-vexp[bh * v16_blocks(T) + b] (the forward kernel's P.V operand).
int v16_blocks(int T);
cudaError_t launch_v_to_f16_blocks(const void *v, void *v16, signed char *vexp, int BH, int T, int d,
                                   cudaStream_t s);

// tcgen05 causal/full prefill forward: bf16 q, k, rho, fp16 block-scaled V
// (tensor map `v` over the output of launch_v_to_f16_blocks, exponents in
// `vexp`), fp32 accumulation, d in {64, 128}.  work_counter: one device int,
// reset by the launch (stream-ordered), the persistent grid's item counter.
// x, w: the fused probe's operands (x [B*T, d_model] and W_R [d_model, H*d],
// 2-D, 128-byte swizzle, boxes 64 x 128 and 64 x 64); unused otherwise.
struct FwdTensorMaps {
    CUtensorMap q, k, r, v, x, w;
};
// o_out [B,H,T,d] fp32 and abar_out [B,H,T] fp32 (nullable): the softmax
// attention output o and abar of each row, kept for the backward.
cudaError_t launch_fwd_sm100(const FwdTensorMaps &tm, bool with_rho, void *y, float *lse, float *o_out,
                             float *abar_out, const signed char *vexp, int B, int H, int T, int d, int causal,
                             int out_dtype, int sm_count, int *work_counter, const DeviceCtl &ctl, cudaStream_t s);
// The same forward with rho computed inside the kernel from x and W_R (d = 128).
cudaError_t launch_fwd_fused_sm100(const FwdTensorMaps &tm, void *y, float *lse, const signed char *vexp, int B,
                                   int H, int T, int d_model, int causal, int out_dtype, int sm_count,
                                   int *work_counter, const DeviceCtl &ctl, cudaStream_t s);

// Tensor maps of the tensor-core gradient kernels: q, rho, dY, k and v, each
// [B*H rows of T x d] bf16 seen as {d, T, B*H}, 128-byte swizzled boxes of 64
// columns x 128 rows (the dq / drho kernel) or x 64 rows for q, rho, dY (the
// dk / dv kernel).
struct BwdTensorMaps {
    CUtensorMap q, r, g, k, v;
};
// dq and drho (fp32, [B,H,T,d]) from lse, abar (training forward) and go, delta
// (k_bwd_rowstats) on tcgen05 (bwd_sm100.cu); work_counter: one int of scratch.
cudaError_t launch_bwd_dq_sm100(const BwdTensorMaps &tm, const float *lse, const float *abar, const float *go,
                                const float *delta, float *dq, float *drho, int B, int H, int T, int d, int causal,
                                int sm_count, int *work_counter, const DeviceCtl &ctl, cudaStream_t s);
// Rows of the packed per-query statistics of the backward per head: T rounded up to 64.
inline int bwd_tpad(int T) { return (T + 63) / 64 * 64; }
// dk and dv (fp32, [B,H,T,d]) on tcgen05 (bwd_dkdv_sm100.cu); stats: per head
// and 64-query block the 64 values of lse log2 e, abar, go and delta in turn
// (B*H*Tpad*4 floats), padding queries (+inf, 0, 0, 0); tm: q, rho, dY with
// 64-row boxes, k and v with 128-row boxes.
cudaError_t launch_bwd_dkdv_sm100(const BwdTensorMaps &tm, const void *stats, float *dk, float *dv, int B, int H, int T,
                                  int d, int causal, int sm_count, int *work_counter, const DeviceCtl &ctl,
                                  cudaStream_t s);
// Gradients of the prefill: go, delta are [B*H*T] fp32 scratch, st4 is
// [B*H*bwd_tpad(T)*4] fp32 scratch (the packed statistics), counters two ints of scratch; tm_dq and
// tm_dkdv the tensor maps of the two gradient kernels.
cudaError_t launch_bwd(const void *dy, const float *y, const float *o, const float *abar, const float *lse, float *go,
                       float *delta, void *st4, float *dq, float *dk, float *dv, float *drho, int B, int H, int T, int d,
                       int causal, const BwdTensorMaps &tm_dq, const BwdTensorMaps &tm_dkdv, int sm_count,
                       int *counters, const DeviceCtl &ctl, cudaStream_t s);

}  // namespace plx
