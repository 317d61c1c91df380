// bwd.cu -- gradients of the Parallax prefill: dq, dk, dv, drho.
//
// The pages train their models with this operator (encorp.ai blog
// "Integraciones de IA personalizadas tras la atencion Parallax", section "Las
// ganancias de preentrenamiento..."; zubnet.ai news item on Parallax,
// paragraph 1) but print no backward; what follows is the chain rule through
// the forward's definitions.  Per row i (query) and key j, with g_i = dY_i:
//   s_ij = exp(z_ij - lse_i),  a_ij = k_j . rho_i,  G_ij = g_i . v_j
//   go_i = g_i . o_i,          delta_i = g_i . y_i + abar_i go_i
//   W_ij  = s_ij (1 + abar_i - a_ij)                    (dv_j   = sum_i W_ij g_i)
//   dZ_ij = s_ij (W_ij/s_ij G_ij + a_ij go_i - delta_i)  (dq_i   = sum_j dZ_ij k_j / sqrt(d),
//                                                          dk_j  += sum_i dZ_ij q_i / sqrt(d))
//   dA_ij = s_ij (go_i - G_ij)                           (drho_i = sum_j dA_ij k_j,
//                                                          dk_j  += sum_i dA_ij rho_i)
// lse_i, abar_i and o_i come from the training forward (parallax_fwd_train).
//
// Three kernels: k_bwd_rowstats here (go, delta per row, and the packed
// per-query statistics), then the two tensor-core kernels that recompute S, A
// and G from q, k, rho, v and dY: the query-stationary dq / drho kernel
// (bwd_sm100.cu) and the key-stationary dk / dv kernel (bwd_dkdv_sm100.cu).
// Every gradient accumulates in TMEM over the tiles of one CTA, so nothing
// needs atomics and the result is deterministic.  W, dZ and dA are rounded to
// bf16 as tensor-core operands (relative error 2^-9 per weight).
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"

namespace plx {
namespace {

constexpr float LOG2E = 1.4426950408889634f;

// ------------------------------------------------------------ row stats --
// go_i = dY_i . o_i and delta_i = dY_i . y_i + abar_i go_i, one warp per row,
// for rows padded to Tpad per head: go and delta go to [B*H*T] arrays (real
// rows only) and (lse_i log2 e, abar_i, go_i, delta_i) to the packed
// statistics: per head and 64-row block, the 64 values of each of the four in
// turn (1 KB per block); padding rows get (+inf, 0, 0, 0), i.e. zero weights.
template <int D>
__global__ void __launch_bounds__(256) k_bwd_rowstats(const __nv_bfloat16 *__restrict__ dy, const float *__restrict__ o,
                                                     const float *__restrict__ y, const float *__restrict__ abar,
                                                     const float *__restrict__ lse, float *__restrict__ go,
                                                     float *__restrict__ delta, float *__restrict__ st, int T,
                                                     int Tpad, long prows) {
    const long prow = (long)blockIdx.x * 8 + threadIdx.x / 32;
    const int lane = threadIdx.x & 31;
    if (prow >= prows) return;
    const long bh = prow / Tpad;
    const int t = (int)(prow % Tpad);
    float *blk = st + (prow - (t & 63)) * 4 + (t & 63);   // this row's slot in its block
    if (t >= T) {
        if (lane == 0) {
            blk[0] = INFINITY;
            blk[64] = blk[128] = blk[192] = 0.f;
        }
        return;
    }
    const long row = bh * T + t;
    float so = 0.f, sy = 0.f;
#pragma unroll
    for (int e = lane; e < D; e += 32) {
        const float g = __bfloat162float(dy[row * D + e]);
        so = fmaf(g, o[row * D + e], so);
        sy = fmaf(g, y[row * D + e], sy);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        so += __shfl_xor_sync(0xffffffffu, so, off);
        sy += __shfl_xor_sync(0xffffffffu, sy, off);
    }
    if (lane == 0) {
        const float ab = abar[row], dl = sy + ab * so;
        go[row] = so;
        delta[row] = dl;
        blk[0] = lse[row] * LOG2E;
        blk[64] = ab;
        blk[128] = so;
        blk[192] = dl;
    }
}

template <int D>
cudaError_t launch_t(const void *dy, const float *y, const float *o, const float *abar, const float *lse, float *go,
                     float *delta, void *st4, float *dq, float *dk, float *dv, float *drho, int B, int H, int T,
                     int causal, const BwdTensorMaps &tm_dq, const BwdTensorMaps &tm_dkdv, int sm_count,
                     int *counters, const DeviceCtl &ctl, cudaStream_t s) {
    const int Tpad = bwd_tpad(T);
    const long prows = (long)B * H * Tpad;
    k_bwd_rowstats<D><<<(unsigned)((prows + 7) / 8), 256, 0, s>>>((const __nv_bfloat16 *)dy, o, y, abar, lse, go, delta,
                                                                   static_cast<float *>(st4), T, Tpad, prows);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if ((e = launch_bwd_dq_sm100(tm_dq, lse, abar, go, delta, dq, drho, B, H, T, D, causal, sm_count, counters, ctl, s)))
        return e;
    return launch_bwd_dkdv_sm100(tm_dkdv, st4, dk, dv, B, H, T, D, causal, sm_count, counters + 1, ctl, s);
}

}  // namespace

cudaError_t launch_bwd(const void *dy, const float *y, const float *o, const float *abar, const float *lse, float *go,
                       float *delta, void *st4, float *dq, float *dk, float *dv, float *drho, int B, int H, int T, int d,
                       int causal, const BwdTensorMaps &tm_dq, const BwdTensorMaps &tm_dkdv, int sm_count,
                       int *counters, const DeviceCtl &ctl, cudaStream_t s) {
    if (d == 64)
        return launch_t<64>(dy, y, o, abar, lse, go, delta, st4, dq, dk, dv, drho, B, H, T, causal, tm_dq, tm_dkdv,
                            sm_count, counters, ctl, s);
    return launch_t<128>(dy, y, o, abar, lse, go, delta, st4, dq, dk, dv, drho, B, H, T, causal, tm_dq, tm_dkdv,
                         sm_count, counters, ctl, s);
}

}  // namespace plx
