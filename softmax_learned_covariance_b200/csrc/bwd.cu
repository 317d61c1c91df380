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
// Three kernels: k_bwd_rowstats (go, delta per row), the tensor-core dq / drho
// kernel of bwd_sm100.cu (query tiles of 128 rows, looping over the keys) and
// k_bwd_dkdv here (key blocks of 64, looping over the queries: dk and dv
// accumulate in registers).  Both main kernels recompute S, A and G from q, k,
// rho, v and dY, so no gradient needs atomics and the result is deterministic.
// k_bwd_dkdv runs on warp-level mma.sync (m16n8k16, bf16 operands, fp32
// accumulation): W, dZ and dA are rounded to bf16 as operands (relative error
// 2^-9 per weight), as in the dq kernel.  Operand tiles are staged in shared
// memory with 16-byte chunks XOR-swizzled by row, loaded with cp.async
// (double-buffered) and read with ldmatrix.
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"

namespace plx {
namespace {

constexpr int BR = 64;          // rows a CTA owns (4 warps x 16)
constexpr int BC = 32;          // columns per step
constexpr int NT = 128;
constexpr float LOG2E = 1.4426950408889634f;

// Byte offset of 16-byte chunk c of row r in a tile of D-element bf16 rows.
template <int D> __device__ __forceinline__ uint32_t swz(int r, int c) {
    return (uint32_t)(r * (D * 2) + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src, bool valid) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(valid ? 4 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// rows [0, rows) x D of a row-major bf16 matrix into a swizzled tile; rows at
// or past `valid` are zero-filled (no global read).
template <int D>
__device__ __forceinline__ void load_tile(uint32_t sdst, const __nv_bfloat16 *src, int rows, int valid) {
    constexpr int CH = D / 8;
    for (int idx = threadIdx.x; idx < rows * CH; idx += NT) {
        const int r = idx / CH, c = idx % CH;
        const bool ok = r < valid;
        cp_async16(sdst + swz<D>(r, c), ok ? (const void *)(src + (size_t)r * D + c * 8) : (const void *)src, ok);
    }
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
// c += a (16x16, row) * b (16x8, col), bf16 operands, fp32 accumulators.
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// A fragment (16 rows x 16 k) of this warp's rows [16 w, 16 w + 16) at k-step kk
// from a swizzled tile whose rows are the mma rows.
template <int D> __device__ __forceinline__ void lda(uint32_t tile, int row0, int kk, uint32_t (&a)[4]) {
    const int lane = threadIdx.x & 31;
    ldsm_x4(tile + swz<D>(row0 + (lane & 15), 2 * kk + (lane >> 4)), a);
}
// B fragments of two n8 tiles (rows n0..n0+15 of a tile stored [n][k]) at k-step kk.
template <int D> __device__ __forceinline__ void ldb(uint32_t tile, int n0, int kk, uint32_t (&b)[4]) {
    const int lane = threadIdx.x & 31, mi = lane >> 3;
    ldsm_x4(tile + swz<D>(n0 + ((mi >> 1) << 3) + (lane & 7), 2 * kk + (mi & 1)), b);
}
// B fragments of two n8 tiles (columns n 16 nd .. 16 nd + 15) at k-step m from a
// tile stored [k][n] (rows are the k index).
template <int D> __device__ __forceinline__ void ldb_t(uint32_t tile, int m, int nd, uint32_t (&b)[4]) {
    const int lane = threadIdx.x & 31, mi = lane >> 3;
    ldsm_x4_t(tile + swz<D>(16 * m + ((mi & 1) << 3) + (lane & 7), 2 * nd + (mi >> 1)), b);
}

// ------------------------------------------------------------ row stats --
// go_i = dY_i . o_i and delta_i = dY_i . y_i + abar_i go_i, one warp per row.
template <int D>
__global__ void __launch_bounds__(256) k_bwd_rowstats(const __nv_bfloat16 *__restrict__ dy, const float *__restrict__ o,
                                                     const float *__restrict__ y, const float *__restrict__ abar,
                                                     float *__restrict__ go, float *__restrict__ delta, long rows) {
    const long row = (long)blockIdx.x * 8 + threadIdx.x / 32;
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
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
        go[row] = so;
        delta[row] = sy + abar[row] * so;
    }
}

// --------------------------------------------------- dk, dv per key block --
template <int D>
__global__ void __launch_bounds__(NT, 2)
    k_bwd_dkdv(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
               const __nv_bfloat16 *__restrict__ v, const __nv_bfloat16 *__restrict__ rho,
               const __nv_bfloat16 *__restrict__ dy, const float *__restrict__ lse, const float *__restrict__ abar,
               const float *__restrict__ go, const float *__restrict__ delta, float *__restrict__ dk,
               float *__restrict__ dv, int T, int causal) {
    constexpr int ROWB = BR * D * 2, COLB = BC * D * 2, ND = D / 8;
    constexpr int STATB = 4 * BC * 4;            // lse, abar, go, delta of BC queries
    extern __shared__ __align__(128) uint8_t sm[];
    const uint32_t sK = (uint32_t)__cvta_generic_to_shared(sm), sV = sK + ROWB;
    const uint32_t sC0 = sV + ROWB;              // per buffer: Q, R, dY tiles, then the statistics
    constexpr uint32_t BUFB = 3 * COLB + STATB;
    const int warp = threadIdx.x / 32, lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
    const long bh = blockIdx.y;
    const int key0 = blockIdx.x * BR;
    const size_t hb = (size_t)bh * T;
    const float sc = LOG2E / sqrtf((float)D), inv_sqrt = 1.0f / sqrtf((float)D);

    load_tile<D>(sK, k + (hb + key0) * D, BR, T - key0);
    load_tile<D>(sV, v + (hb + key0) * D, BR, T - key0);
    const int qbeg = causal ? key0 : 0;           // queries before the block's first key see none of it
    const int nsteps = (T - qbeg + BC - 1) / BC;
    auto load_cols = [&](int st) {
        const uint32_t b = sC0 + (st & 1) * BUFB;
        const int i0 = qbeg + st * BC;
        load_tile<D>(b, q + (hb + i0) * D, BC, T - i0);
        load_tile<D>(b + COLB, rho + (hb + i0) * D, BC, T - i0);
        load_tile<D>(b + 2 * COLB, dy + (hb + i0) * D, BC, T - i0);
        const int sidx = threadIdx.x;            // 4 statistics x BC queries = 128 words
        const int which = sidx / BC, qi = sidx % BC;
        const float *src = which == 0 ? lse : which == 1 ? abar : which == 2 ? go : delta;
        const bool ok = i0 + qi < T;
        cp_async4(b + 3 * COLB + sidx * 4, ok ? (const void *)(src + hb + i0 + qi) : (const void *)src, ok);
    };
    load_cols(0);
    cp_async_commit();

    const int kr[2] = {key0 + 16 * warp + gq, key0 + 16 * warp + gq + 8};
    float ak[ND][4], av_[ND][4];
#pragma unroll
    for (int t = 0; t < ND; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) ak[t][e] = av_[t][e] = 0.f;

    for (int st = 0; st < nsteps; ++st) {
        if (st + 1 < nsteps) load_cols(st + 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        const uint32_t b = sC0 + (st & 1) * BUFB, sQ = b, sR = b + COLB, sG = b + 2 * COLB;
        const float *stat = reinterpret_cast<const float *>(sm + (b + 3 * COLB - (uint32_t)__cvta_generic_to_shared(sm)));
        const int i0 = qbeg + st * BC;
        // S^T = K Q^T, A^T = K R^T, G^T = V dY^T for 16 keys x 32 queries
        float s4[4][4], a4[4][4], g4[4][4];
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) s4[t][e] = a4[t][e] = g4[t][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            uint32_t fk[4], fv[4];
            lda<D>(sK, 16 * warp, kk, fk);
            lda<D>(sV, 16 * warp, kk, fv);
#pragma unroll
            for (int nb = 0; nb < 2; ++nb) {
                uint32_t bq[4], br[4], bg[4];
                ldb<D>(sQ, 16 * nb, kk, bq);
                ldb<D>(sR, 16 * nb, kk, br);
                ldb<D>(sG, 16 * nb, kk, bg);
                mma16816(s4[2 * nb], fk, bq[0], bq[1]);
                mma16816(s4[2 * nb + 1], fk, bq[2], bq[3]);
                mma16816(a4[2 * nb], fk, br[0], br[1]);
                mma16816(a4[2 * nb + 1], fk, br[2], br[3]);
                mma16816(g4[2 * nb], fv, bg[0], bg[1]);
                mma16816(g4[2 * nb + 1], fv, bg[2], bg[3]);
            }
        }
        // W, dZ / sqrt(d), dA as bf16 A fragments, k = the 32 queries
        uint32_t fw[2][4], fz[2][4], fa[2][4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            float w[4], z[4], a[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int h = e >> 1;
                const int qc = 8 * t + 2 * tq + (e & 1);      // query within the step
                const int qi = i0 + qc;
                const bool ok = qi < T && kr[h] < T && (!causal || kr[h] <= qi);
                const float l2 = stat[qc] * LOG2E, abq = stat[BC + qc], goq = stat[2 * BC + qc],
                            dlq = stat[3 * BC + qc];
                const float s = ok ? exp2f(fmaf(s4[t][e], sc, -l2)) : 0.f;
                const float avv = a4[t][e], gv = g4[t][e];
                const float f1 = 1.f + abq - avv;
                w[e] = s * f1;
                z[e] = s * (fmaf(f1, gv, avv * goq) - dlq) * inv_sqrt;
                a[e] = s * (goq - gv);
            }
            fw[t >> 1][(t & 1) * 2 + 0] = pack_bf16(w[0], w[1]);
            fw[t >> 1][(t & 1) * 2 + 1] = pack_bf16(w[2], w[3]);
            fz[t >> 1][(t & 1) * 2 + 0] = pack_bf16(z[0], z[1]);
            fz[t >> 1][(t & 1) * 2 + 1] = pack_bf16(z[2], z[3]);
            fa[t >> 1][(t & 1) * 2 + 0] = pack_bf16(a[0], a[1]);
            fa[t >> 1][(t & 1) * 2 + 1] = pack_bf16(a[2], a[3]);
        }
        // dv += W dY, dk += dZ Q / sqrt(d) + dA R
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int nd = 0; nd < D / 16; ++nd) {
                uint32_t bg[4], bq[4], br[4];
                ldb_t<D>(sG, m, nd, bg);
                ldb_t<D>(sQ, m, nd, bq);
                ldb_t<D>(sR, m, nd, br);
                mma16816(av_[2 * nd], fw[m], bg[0], bg[1]);
                mma16816(av_[2 * nd + 1], fw[m], bg[2], bg[3]);
                mma16816(ak[2 * nd], fz[m], bq[0], bq[1]);
                mma16816(ak[2 * nd + 1], fz[m], bq[2], bq[3]);
                mma16816(ak[2 * nd], fa[m], br[0], br[1]);
                mma16816(ak[2 * nd + 1], fa[m], br[2], br[3]);
            }
        __syncthreads();
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        if (kr[h] >= T) continue;
        float *pk = dk + (hb + kr[h]) * D, *pv = dv + (hb + kr[h]) * D;
#pragma unroll
        for (int t = 0; t < ND; ++t) {
            *reinterpret_cast<float2 *>(pk + 8 * t + 2 * tq) = make_float2(ak[t][2 * h], ak[t][2 * h + 1]);
            *reinterpret_cast<float2 *>(pv + 8 * t + 2 * tq) = make_float2(av_[t][2 * h], av_[t][2 * h + 1]);
        }
    }
}

template <int D>
cudaError_t launch_t(const void *q, const void *k, const void *v, const void *rho, const void *dy, const float *y,
                     const float *o, const float *abar, const float *lse, float *go, float *delta, float *dq,
                     float *dk, float *dv, float *drho, int B, int H, int T, int causal, const BwdTensorMaps &tm,
                     int sm_count, int *work_counter, const DeviceCtl &ctl, cudaStream_t s) {
    const int BH = B * H;
    using bf = __nv_bfloat16;
    const long rows = (long)BH * T;
    k_bwd_rowstats<D><<<(unsigned)((rows + 7) / 8), 256, 0, s>>>((const bf *)dy, o, y, abar, go, delta, rows);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    constexpr int ROWB = BR * D * 2, COLB = BC * D * 2;
    constexpr int SM_DK = 2 * ROWB + 2 * (3 * COLB + 4 * BC * 4);
    static std::atomic<unsigned long long> set_dk{0};
    if ((e = ensure_smem_limit(k_bwd_dkdv<D>, SM_DK, set_dk))) return e;
    const dim3 grid((unsigned)((T + BR - 1) / BR), (unsigned)BH);
    if ((e = launch_bwd_dq_sm100(tm, lse, abar, go, delta, dq, drho, B, H, T, D, causal, sm_count, work_counter, ctl,
                                 s)))
        return e;
    k_bwd_dkdv<D><<<grid, NT, SM_DK, s>>>((const bf *)q, (const bf *)k, (const bf *)v, (const bf *)rho,
                                         (const bf *)dy, lse, abar, go, delta, dk, dv, T, causal);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd(const void *q, const void *k, const void *v, const void *rho, const void *dy, const float *y,
                       const float *o, const float *abar, const float *lse, float *go, float *delta, float *dq,
                       float *dk, float *dv, float *drho, int B, int H, int T, int d, int causal,
                       const BwdTensorMaps &tm, int sm_count, int *work_counter, const DeviceCtl &ctl, cudaStream_t s) {
    if (d == 64)
        return launch_t<64>(q, k, v, rho, dy, y, o, abar, lse, go, delta, dq, dk, dv, drho, B, H, T, causal, tm, sm_count,
                            work_counter, ctl, s);
    return launch_t<128>(q, k, v, rho, dy, y, o, abar, lse, go, delta, dq, dk, dv, drho, B, H, T, causal, tm, sm_count,
                         work_counter, ctl, s);
}

}  // namespace plx
