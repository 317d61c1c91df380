// fwd_simt.cu -- CUDA-core forward (fp32 arithmetic throughout).
//
// One warp per query row; each lane owns d/32 of the head dimensions.  For every
// visible key the warp forms z = q.k/sqrt(d) and a = k.rho with shuffle
// reductions and updates the running (max, l, abar, O, M) state with an exact
// rescale, so the result is the one-pass form y = o - (m - o abar) of the
// operator (zubnet.ai news item on Parallax, paragraph 2), in fp32.
// This is the fp32-input path; bf16 inputs run on the tensor cores.
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"

namespace plx {
namespace {

__device__ __forceinline__ float ld_as_f32(const float *p) { return __ldg(p); }

template <typename Tin, typename Tout, int D, bool WITH_RHO>
__global__ void __launch_bounds__(128) k_fwd_simt(const Tin *__restrict__ q, const Tin *__restrict__ k,
                                                  const Tin *__restrict__ v, const Tin *__restrict__ rho,
                                                  Tout *__restrict__ y, float *__restrict__ lse, int BH, int T,
                                                  int causal) {
    constexpr int E = D / 32;
    const int lane = threadIdx.x & 31;
    const long row = (long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    if (row >= (long)BH * T) return;
    const long bh = row / T;
    const int i = (int)(row % T);
    const size_t head = (size_t)bh * T * D;

    float qv[E], rv[E], O[E], Mv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        qv[e] = ld_as_f32(q + head + (size_t)i * D + lane + 32 * e);
        rv[e] = WITH_RHO ? ld_as_f32(rho + head + (size_t)i * D + lane + 32 * e) : 0.f;
        O[e] = 0.f;
        Mv[e] = 0.f;
    }
    const float scale = 1.0f / sqrtf((float)D);
    float mx = -INFINITY, l = 0.f, abar = 0.f;
    const int n = causal ? i + 1 : T;
    for (int j = 0; j < n; ++j) {
        const Tin *kj = k + head + (size_t)j * D;
        const Tin *vj = v + head + (size_t)j * D;
        float dz = 0.f, da = 0.f, kv[E], vv[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
            kv[e] = ld_as_f32(kj + lane + 32 * e);
            vv[e] = ld_as_f32(vj + lane + 32 * e);
            dz = fmaf(qv[e], kv[e], dz);
            if (WITH_RHO) da = fmaf(rv[e], kv[e], da);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            dz += __shfl_xor_sync(0xffffffffu, dz, off);
            if (WITH_RHO) da += __shfl_xor_sync(0xffffffffu, da, off);
        }
        const float z = dz * scale;
        const float mnew = fmaxf(mx, z);
        const float alpha = expf(mx - mnew);   // 0 on the first key (mx = -inf)
        const float p = expf(z - mnew);
        l = l * alpha + p;
        if (WITH_RHO) abar = abar * alpha + p * da;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            O[e] = O[e] * alpha + p * vv[e];
            if (WITH_RHO) Mv[e] = Mv[e] * alpha + (p * da) * vv[e];
        }
        mx = mnew;
    }
    const float inv_l = 1.0f / l;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const float o = O[e] * inv_l;
        float out = o;
        if (WITH_RHO) out = o - (Mv[e] * inv_l - o * (abar * inv_l));
        if constexpr (sizeof(Tout) == 4)
            y[head + (size_t)i * D + lane + 32 * e] = out;
        else
            y[head + (size_t)i * D + lane + 32 * e] = __float2bfloat16_rn(out);
    }
    if (lse != nullptr && lane == 0) lse[row] = mx + logf(l);
}

template <typename Tin, typename Tout, int D>
cudaError_t launch_t(const void *q, const void *k, const void *v, const void *rho, void *y, float *lse, int BH,
                     int T, int causal, cudaStream_t s) {
    const long rows = (long)BH * T;
    const unsigned blocks = (unsigned)((rows + 3) / 4);
    if (rho)
        k_fwd_simt<Tin, Tout, D, true><<<blocks, 128, 0, s>>>(
            (const Tin *)q, (const Tin *)k, (const Tin *)v, (const Tin *)rho, (Tout *)y, lse, BH, T, causal);
    else
        k_fwd_simt<Tin, Tout, D, false><<<blocks, 128, 0, s>>>(
            (const Tin *)q, (const Tin *)k, (const Tin *)v, nullptr, (Tout *)y, lse, BH, T, causal);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_simt(const void *q, const void *k, const void *v, const void *rho, void *y, float *lse,
                            int B, int H, int T, int d, int causal, int in_dtype, int out_dtype, cudaStream_t s) {
    if (in_dtype != PARALLAX_F32 || out_dtype != PARALLAX_F32) return cudaErrorInvalidValue;
    const int BH = B * H;
    if (d == 64) return launch_t<float, float, 64>(q, k, v, rho, y, lse, BH, T, causal, s);
    return launch_t<float, float, 128>(q, k, v, rho, y, lse, BH, T, causal, s);
}

}  // namespace plx
