// rho_proj.cu -- rho = x W_R on the tensor cores (tcgen05), scattered per head.
//
// The probe of the covariance branch is a learned projection of the layer
// input (encorp.ai blog "Integraciones de IA personalizadas tras la atencion
// Parallax", section "Por que eliminar el solucionador de gradiente
// conjugado..."; zubnet.ai news item on Parallax, paragraph 2: rho_i = W_R x_i).
//
// GEMM [M = B*T, K = d_model] x [K, N = H*d] -> rho[b, h, t, :] in bf16.
// Persistent kernel, one CTA per SM, 128 x 256 output tiles walked n-fastest so
// a row block of x is reused from L2 across the column blocks.
//   warp 0      : TMA producer (x tile K-major, W_R tile MN-major, 128-B swizzle)
//   warp 1      : TMEM allocation + single-thread UMMA issue (M=128, N=256, K=16)
//   warps 4..7  : epilogue, TMEM -> registers -> bf16 -> global, one row per thread
// Two TMEM accumulators (2 x 256 columns) let the epilogue of one tile overlap
// the main loop of the next.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace plx {
namespace {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;            // 16 KB
constexpr int B_BYTES = BK * BN * 2;            // 32 KB (4 column groups of 64)
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // 48 KB
constexpr int NTHREADS = 256;
constexpr uint32_t IDESC = idesc_f16(/*a bf16*/ 1, /*b bf16*/ 1, /*a K-major*/ 0, /*b MN-major*/ 1, BM, BN);

struct __align__(8) Bars {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;               // the UMMA issuer's last commit (all its MMAs complete)
    uint32_t tmem_base;
    int abort_flag;
};
constexpr unsigned long long DRAIN_NS = 2000000ull;   // bound of the exit-time drain waits

constexpr size_t SMEM_BYTES = 1024 /*align slack*/ + (size_t)STAGES * STAGE_BYTES + sizeof(Bars);

__global__ void __launch_bounds__(NTHREADS, 1)
    k_rho_proj(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
               __nv_bfloat16 *__restrict__ rho, int M, int N, int K, int T, int H, int d, DeviceCtl ctl) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars *bars = reinterpret_cast<Bars *>(smem + (size_t)STAGES * STAGE_BYTES);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&bars->full[s]), 1);
            mbar_init(smem_u32(&bars->empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&bars->acc_full[b]), 1);
            mbar_init(smem_u32(&bars->acc_empty[b]), 128);
        }
        mbar_init(smem_u32(&bars->drain), 1);
        bars->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&bars->tmem_base), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    WaitCtl wc{ctl.err, &bars->abort_flag, ctl.wait_ns};
    const int m_tiles = (M + BM - 1) / BM;
    const int n_tiles = N / BN;
    const int tiles = m_tiles * n_tiles;
    const int k_blocks = K / BK;

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------ TMA producer --
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_w);
        uint32_t it = 0;
        int armed[STAGES];   // parity of each stage's last fill still to land, -1 if none
        for (int s = 0; s < STAGES; ++s) armed[s] = -1;
        bool ok = true;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
            const int m0 = (t / n_tiles) * BM, n0 = (t % n_tiles) * BN;
            for (int kb = 0; kb < k_blocks; ++kb, ++it) {
                const int s = it % STAGES;
                const uint32_t ph = (it / STAGES) & 1;
                if (!mbar_wait(smem_u32(&bars->empty[s]), ph ^ 1, wc)) { ok = false; break; }
                const uint32_t full = smem_u32(&bars->full[s]);
                armed[s] = (int)ph;
                mbar_arrive_expect_tx(full, STAGE_BYTES);
                const uint32_t sa = smem_u32(smem + (size_t)s * STAGE_BYTES);
                const uint32_t sb = sa + A_BYTES;
                tma_load_2d(sa, &tm_x, full, kb * BK, m0);
#pragma unroll
                for (int g = 0; g < BN / 64; ++g) tma_load_2d(sb + g * (BK * 128), &tm_w, full, n0 + g * 64, kb * BK);
            }
        }
        // no copy of this thread may still be landing when the CTA exits
        for (int s = 0; s < STAGES; ++s)
            if (armed[s] >= 0) mbar_wait_drain(smem_u32(&bars->full[s]), (uint32_t)armed[s], DRAIN_NS);
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------- UMMA issuer --
        uint32_t it = 0, local = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++local) {
            const uint32_t ab = local & 1;
            if (!mbar_wait(smem_u32(&bars->acc_empty[ab]), ((local >> 1) & 1) ^ 1, wc)) break;
            tc_fence_after();
            const uint32_t d_tmem = tmem + ab * BN;
            for (int kb = 0; kb < k_blocks; ++kb, ++it) {
                const int s = it % STAGES;
                const uint32_t ph = (it / STAGES) & 1;
                if (!mbar_wait(smem_u32(&bars->full[s]), ph, wc)) { ok = false; break; }
                tc_fence_after();
                const uint32_t sa = smem_u32(smem + (size_t)s * STAGE_BYTES);
                const uint32_t sb = sa + A_BYTES;
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
                    const uint64_t adesc = sdesc_sw128(sa + kk * 32, 16, 1024);
                    const uint64_t bdesc = sdesc_sw128(sb + kk * 16 * 128, BK * 128, 1024);
                    umma_ss(d_tmem, adesc, bdesc, IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(smem_u32(&bars->empty[s]));
            }
            if (ok) tc_commit(smem_u32(&bars->acc_full[ab]));
        }
        // every MMA this thread issued has completed before TMEM is released
        tc_commit(smem_u32(&bars->drain));
        mbar_wait_drain(smem_u32(&bars->drain), 0, DRAIN_NS);
    } else if (warp >= 4) {
        // ---------------------------------------------------- epilogue --
        const int quarter = warp & 3;
        const int row_in_tile = quarter * 32 + lane;
        uint32_t local = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++local) {
            const uint32_t ab = local & 1;
            // warp-uniform outcome: tcgen05.ld below is .sync.aligned
            if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->acc_full[ab]), (local >> 1) & 1, wc))) break;
            tc_fence_after();
            const int m0 = (t / n_tiles) * BM, n0 = (t % n_tiles) * BN;
            const int m = m0 + row_in_tile;
            const int b = m / T, tt = m % T;
            const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + ab * BN;
#pragma unroll 1
            for (int c = 0; c < BN; c += 32) {
                uint32_t r0[16], r1[16];
                tmem_ld16(taddr + c, r0);
                tmem_ld16(taddr + c + 16, r1);
                tmem_wait_ld();
                if (m < M) {
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        __nv_bfloat162 h0 = __floats2bfloat162_rn(__uint_as_float(r0[2 * i]), __uint_as_float(r0[2 * i + 1]));
                        __nv_bfloat162 h1 = __floats2bfloat162_rn(__uint_as_float(r1[2 * i]), __uint_as_float(r1[2 * i + 1]));
                        pk[i] = *reinterpret_cast<uint32_t *>(&h0);
                        pk[8 + i] = *reinterpret_cast<uint32_t *>(&h1);
                    }
                    const int n = n0 + c;
                    const int h = n / d, e = n % d;
                    uint4 *dst = reinterpret_cast<uint4 *>(rho + (((size_t)b * H + h) * T + tt) * d + e);
#pragma unroll
                    for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                }
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&bars->acc_empty[ab]));
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace

cudaError_t launch_rho_proj(const CUtensorMap &tm_x, const CUtensorMap &tm_w, void *rho, int B, int T, int d_model,
                            int H, int d, int sm_count, const DeviceCtl &ctl, cudaStream_t s) {
    static std::atomic<unsigned long long> limit_set{0};
    if (cudaError_t e = ensure_smem_limit(k_rho_proj, (int)SMEM_BYTES, limit_set)) return e;
    const int M = B * T, N = H * d;
    const int tiles = ((M + BM - 1) / BM) * (N / BN);
    const int grid = tiles < sm_count ? tiles : sm_count;
    k_rho_proj<<<grid, NTHREADS, SMEM_BYTES, s>>>(tm_x, tm_w, static_cast<__nv_bfloat16 *>(rho), M, N, d_model, T, H,
                                                  d, ctl);
    return cudaGetLastError();
}

}  // namespace plx
