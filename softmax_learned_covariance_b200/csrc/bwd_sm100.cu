// bwd_sm100.cu -- dq and drho of the Parallax prefill on the tensor cores
// (tcgen05 + TMA + TMEM).
//
// The chain rule through the forward's definitions (see bwd.cu for the
// derivation; zubnet.ai news item on Parallax, paragraph 2, for the operator):
// per query row i and key j, with g_i = dY_i,
//   s_ij  = exp(z_ij - lse_i),  a_ij = k_j . rho_i,  G_ij = g_i . v_j
//   dZ_ij = s_ij ((1 + abar_i - a_ij) G_ij + a_ij go_i - delta_i)
//   dA_ij = s_ij (go_i - G_ij)
//   dq_i  = sum_j dZ_ij k_j / sqrt(d),   drho_i = sum_j dA_ij k_j.
// One CTA per SM, persistent over (head, 128-row query tile) items, walks the
// key tiles of its rows.  Per 128-key tile three score products land one after
// another in a TMEM tile region (S = Q K^T, A = R K^T, G = dY V^T, bf16 in,
// fp32 out); the softmax warps read each once, form dZ / sqrt(d) and dA as
// bf16 over the G columns they have read, and the second issuing thread
// accumulates dq += dZ K and drho += dA K in TMEM (the K tile in shared memory
// read as the MN-major B operand).  lse, abar, go and delta of each row come
// from the training forward and k_bwd_rowstats, so no row max or row sum is
// taken here: the weights are final when formed.
//
// TMEM: tile regions X0, X1 (tile G uses X(G mod 2), so the next tile's S can
// land while this tile's products are still being read) and the accumulators
// dQ, dR.  Shared memory: Q, R and dY of the item, a 2-stage K ring, one V
// buffer (V of the next tile is loaded once G of this tile is done).
//
// Roles (640 threads, persistent, items longest-first from an atomic counter):
//   warp 0 lane 0   scheduler + TMA for Q, R, dY (per item), K and V (per tile)
//   warp 1          TMEM owner; lane 0 issues S, A and G
//   warps 2..17     four warpgroups; group g takes keys [32g, 32g + 32) of each
//                   tile for all 128 rows (one row per thread); then the
//                   item's epilogue (group g writes d/4 columns of dq, drho)
//   warp 18 lane 0  issues dq += dZ K, drho += dA K
// Every wait is bounded; a wait that gives up lets every role leave its loop.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include "internal.h"
#include "sm100.cuh"
#include "softmax_sm100.cuh"

namespace plx {
namespace {

constexpr int BM = 128;                   // query rows per tile
constexpr int BN = 128;                   // keys per tile
constexpr int NGRP = 4;                   // elementwise warpgroups
constexpr int GCOLS = BN / NGRP;          // keys per group
constexpr int KST = 2;                    // K ring stages
constexpr int SCHED = 4;                  // scheduler ring depth
constexpr int FIRST_SOFT_WARP = 2;
constexpr int NSOFT_WARPS = NGRP * 4;
constexpr int DQ_WARP = FIRST_SOFT_WARP + NSOFT_WARPS;   // dq / drho issuer
constexpr int NTHREADS = (DQ_WARP + 1) * 32;
constexpr float LOG2E = 1.4426950408889634f;
constexpr unsigned long long DRAIN_NS = 2000000ull;

template <int D> struct GeoB {
    static constexpr int HALVES = D / 64;                // 128-byte column blocks of a row
    static constexpr int T_BYTES = BM * D * 2;           // one 128-row bf16 tile
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_R = OFF_Q + T_BYTES;
    static constexpr int OFF_G = OFF_R + T_BYTES;        // dY
    static constexpr int OFF_K = OFF_G + T_BYTES;
    static constexpr int OFF_V = OFF_K + KST * T_BYTES;
    static constexpr int OFF_BARS = OFF_V + T_BYTES;
    static constexpr int OCOLS = D / NGRP;               // dq / drho columns each group writes
    static_assert(OCOLS % 16 == 0, "16-column TMEM loads");
};

// TMEM: tile regions X0, X1; accumulators dQ and dR on 128-column boundaries.
constexpr uint32_t COL_X0 = 0, COL_DQ = 256, COL_DR = 384;
__host__ __device__ constexpr uint32_t col_x(uint32_t G) { return COL_X0 + (G & 1) * BN; }
// Within a region, the bf16 dZ of keys [16c, 16c + 16) sits in columns
// [16c, 16c + 8) and their dA in the next 8: the G columns of those keys.
__host__ __device__ constexpr uint32_t col_dz(uint32_t kk) { return kk * 16; }
constexpr uint32_t DA_SHIFT = 8;

constexpr uint32_t IDESC_S = idesc_f16(1, 1, 0, 0, BM, BN);                       // bf16 K-major x bf16 K-major
template <int D> constexpr uint32_t idesc_dq() { return idesc_f16(1, 1, 0, 1, BM, D); }   // bf16 (TMEM) x bf16 K tile (MN-major)

struct __align__(8) BarsB {
    uint64_t qr_full, qr_empty;        // Q, R, dY of the item
    uint64_t k_full[KST], k_empty[KST];
    uint64_t v_full, v_empty;
    uint64_t s_full, a_full, g_full;   // score products of the current tile done
    uint64_t s_free, a_free;           // the elementwise warps have read S, A
    uint64_t p_full[2];                // per region: dZ, dA of its tile are in TMEM
    uint64_t pv_done[2];               // per region: dq / drho products of its tile done
    uint64_t om_free;                  // the epilogue has read dQ and dR
    uint64_t drain[2];
    uint64_t sched_full[SCHED], sched_empty[SCHED];
    int sched_item[SCHED];
    uint32_t tmem_base;
    int abort_flag;
};

template <int D> constexpr size_t smem_bytes_b() { return (size_t)GeoB<D>::OFF_BARS + sizeof(BarsB); }
static_assert(smem_bytes_b<128>() <= 232448, "shared memory budget");

struct ItemB {
    int bh, qt, nkv;
};

__device__ __forceinline__ ItemB item_of_b(int w, int BH, int nq, int T, int causal) {
    ItemB it;
    it.qt = nq - 1 - w / BH;   // longest rows first
    it.bh = w % BH;
    const int kend = causal ? min(T, (it.qt + 1) * BM) : T;
    it.nkv = (kend + BN - 1) / BN;
    return it;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

template <int D>
__global__ void __launch_bounds__(NTHREADS, 1)
    k_bwd_dq_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_r,
                const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const float *__restrict__ lse,
                const float *__restrict__ abar, const float *__restrict__ go, const float *__restrict__ delta,
                float *__restrict__ dq, float *__restrict__ drho, int BH, int T, int causal,
                int *__restrict__ work_counter, DeviceCtl ctl) {
    using Gm = GeoB<D>;
    extern __shared__ __align__(1024) uint8_t smem[];
    if (smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) atomicExch(ctl.err, PARALLAX_ERR_UNSUPPORTED);
        return;
    }
    BarsB *bars = reinterpret_cast<BarsB *>(smem + Gm::OFF_BARS);
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bars->qr_full), 1);
        mbar_init(smem_u32(&bars->qr_empty), 1);
        for (int s = 0; s < KST; ++s) {
            mbar_init(smem_u32(&bars->k_full[s]), 1);
            mbar_init(smem_u32(&bars->k_empty[s]), 1);
        }
        mbar_init(smem_u32(&bars->v_full), 1);
        mbar_init(smem_u32(&bars->v_empty), 1);
        mbar_init(smem_u32(&bars->s_full), 1);
        mbar_init(smem_u32(&bars->a_full), 1);
        mbar_init(smem_u32(&bars->g_full), 1);
        mbar_init(smem_u32(&bars->s_free), NSOFT_WARPS);
        mbar_init(smem_u32(&bars->a_free), NSOFT_WARPS);
        for (int x = 0; x < 2; ++x) {
            mbar_init(smem_u32(&bars->p_full[x]), NSOFT_WARPS);
            mbar_init(smem_u32(&bars->pv_done[x]), 1);
        }
        mbar_init(smem_u32(&bars->om_free), NSOFT_WARPS);
        mbar_init(smem_u32(&bars->drain[0]), 1);
        mbar_init(smem_u32(&bars->drain[1]), 1);
        for (int s = 0; s < SCHED; ++s) {
            mbar_init(smem_u32(&bars->sched_full[s]), 1);
            mbar_init(smem_u32(&bars->sched_empty[s]), 2 + NSOFT_WARPS);   // two UMMA threads, elementwise warps
        }
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
    const int nq = (T + BM - 1) / BM;
    const int items = nq * BH;

    if (warp == 0 && lane == 0) {
        // ===================================== scheduler + TMA producer ==
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_r);
        tma_prefetch_desc(&tm_g);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        uint32_t kc = 0, G = 0;
        int k_armed[KST], qr_armed = -1, v_armed = -1;
        for (int s = 0; s < KST; ++s) k_armed[s] = -1;
        bool ok = true;
        for (uint32_t ic = 0; ok; ++ic) {
            const uint32_t ss = ic % SCHED;
            if (!mbar_wait(smem_u32(&bars->sched_empty[ss]), ((ic / SCHED) & 1) ^ 1, wc)) break;
            const int w = ic == 0 ? (int)blockIdx.x : (int)gridDim.x + atomicAdd(work_counter, 1);
            bars->sched_item[ss] = w;
            mbar_arrive(smem_u32(&bars->sched_full[ss]));
            if (w >= items) break;
            const ItemB it = item_of_b(w, BH, nq, T, causal);
            const int q0 = it.qt * BM;
            if (!mbar_wait(smem_u32(&bars->qr_empty), (ic & 1) ^ 1, wc)) break;
            const uint32_t qf = smem_u32(&bars->qr_full);
            qr_armed = (int)(ic & 1);
            mbar_arrive_expect_tx(qf, 3 * Gm::T_BYTES);
#pragma unroll
            for (int h = 0; h < Gm::HALVES; ++h) {
                const uint32_t hoff = h * (Gm::T_BYTES / Gm::HALVES);
                tma_load_3d(sbase + Gm::OFF_Q + hoff, &tm_q, qf, h * 64, q0, it.bh);
                tma_load_3d(sbase + Gm::OFF_R + hoff, &tm_r, qf, h * 64, q0, it.bh);
                tma_load_3d(sbase + Gm::OFF_G + hoff, &tm_g, qf, h * 64, q0, it.bh);
            }
            for (int j = 0; j < it.nkv; ++j, ++kc, ++G) {
                const int s = kc % KST;
                if (!mbar_wait(smem_u32(&bars->k_empty[s]), ((kc / KST) & 1) ^ 1, wc)) { ok = false; break; }
                const uint32_t f = smem_u32(&bars->k_full[s]);
                k_armed[s] = (int)((kc / KST) & 1);
                mbar_arrive_expect_tx(f, Gm::T_BYTES);
#pragma unroll
                for (int h = 0; h < Gm::HALVES; ++h)
                    tma_load_3d(sbase + Gm::OFF_K + s * Gm::T_BYTES + h * (Gm::T_BYTES / Gm::HALVES), &tm_k, f,
                                h * 64, j * BN, it.bh);
                // V of this tile, once G of the previous tile is done with the buffer
                if (!mbar_wait(smem_u32(&bars->v_empty), (G & 1) ^ 1, wc)) { ok = false; break; }
                const uint32_t fv = smem_u32(&bars->v_full);
                v_armed = (int)(G & 1);
                mbar_arrive_expect_tx(fv, Gm::T_BYTES);
#pragma unroll
                for (int h = 0; h < Gm::HALVES; ++h)
                    tma_load_3d(sbase + Gm::OFF_V + h * (Gm::T_BYTES / Gm::HALVES), &tm_v, fv, h * 64, j * BN,
                                it.bh);
            }
        }
        if (qr_armed >= 0) mbar_wait_drain(smem_u32(&bars->qr_full), (uint32_t)qr_armed, DRAIN_NS);
        for (int s = 0; s < KST; ++s)
            if (k_armed[s] >= 0) mbar_wait_drain(smem_u32(&bars->k_full[s]), (uint32_t)k_armed[s], DRAIN_NS);
        if (v_armed >= 0) mbar_wait_drain(smem_u32(&bars->v_full), (uint32_t)v_armed, DRAIN_NS);
    } else if (warp == 1 && lane == 0) {
        // ============================================= score UMMA issuer ==
        // Tile G: S(G) into X(G & 1) once the dq products of tile G - 2 are
        // done with the region, A(G) once S(G) is read, G(G) once A(G) is read.
        uint32_t kc = 0, G = 0;
        bool ok = true;
        const uint64_t dq_ = sdesc_sw128(sbase + Gm::OFF_Q, 16, 1024);
        const uint64_t dr_ = sdesc_sw128(sbase + Gm::OFF_R, 16, 1024);
        const uint64_t dg_ = sdesc_sw128(sbase + Gm::OFF_G, 16, 1024);
        const uint64_t dk_ = sdesc_sw128(sbase + Gm::OFF_K, 16, 1024);   // stage s: + s * T_BYTES / 16
        const uint64_t dv_ = sdesc_sw128(sbase + Gm::OFF_V, 16, 1024);
        auto issue_scores = [&](uint32_t dcol, uint64_t da, uint64_t kd) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off =
                    ((uint32_t)(kk >> 2) * (Gm::T_BYTES / Gm::HALVES) + (uint32_t)(kk & 3) * 32) >> 4;
                umma_ss(tmem + dcol, da + off, kd + off, IDESC_S, kk > 0 ? 1u : 0u);
            }
        };
        for (uint32_t ic = 0; ok; ++ic) {
            int w;
            if (!next_item<SCHED>(bars, ic, w, wc)) break;
            mbar_arrive(smem_u32(&bars->sched_empty[ic % SCHED]));
            if (w >= items) break;
            const ItemB it = item_of_b(w, BH, nq, T, causal);
            if (!mbar_wait(smem_u32(&bars->qr_full), ic & 1, wc)) break;
            for (int j = 0; j < it.nkv; ++j, ++G, ++kc) {
                const int s = kc % KST;
                if (!mbar_wait(smem_u32(&bars->k_full[s]), (kc / KST) & 1, wc)) { ok = false; break; }
                if (G >= 2 && !mbar_wait(smem_u32(&bars->pv_done[G & 1]), ((G - 2) >> 1) & 1, wc)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t kd = dk_ + (uint64_t)(s * (Gm::T_BYTES >> 4));
                issue_scores(col_x(G), dq_, kd);
                tc_commit(smem_u32(&bars->s_full));
                if (!mbar_wait(smem_u32(&bars->s_free), G & 1, wc)) { ok = false; break; }
                tc_fence_after();
                issue_scores(col_x(G), dr_, kd);
                tc_commit(smem_u32(&bars->a_full));
                if (!mbar_wait(smem_u32(&bars->v_full), G & 1, wc)) { ok = false; break; }
                if (!mbar_wait(smem_u32(&bars->a_free), G & 1, wc)) { ok = false; break; }
                tc_fence_after();
                issue_scores(col_x(G), dg_, dv_);
                tc_commit(smem_u32(&bars->g_full));
                tc_commit(smem_u32(&bars->v_empty));
                if (j == it.nkv - 1) tc_commit(smem_u32(&bars->qr_empty));
            }
        }
        tc_commit(smem_u32(&bars->drain[0]));
        mbar_wait_drain(smem_u32(&bars->drain[0]), 0, DRAIN_NS);
    } else if (warp == DQ_WARP && lane == 0) {
        // ===================================== dq / drho UMMA issuer ==
        uint32_t kc = 0, G = 0;
        bool ok = true;
        constexpr uint32_t IDESC_DQ = idesc_dq<D>();
        // the K tile as the MN-major B operand [keys x d]: 16 keys = 2 KB per k-step
        const uint64_t dkm = sdesc_sw128(sbase + Gm::OFF_K, Gm::T_BYTES / Gm::HALVES, 1024);
        for (uint32_t ic = 0; ok; ++ic) {
            int w;
            if (!next_item<SCHED>(bars, ic, w, wc)) break;
            mbar_arrive(smem_u32(&bars->sched_empty[ic % SCHED]));
            if (w >= items) break;
            const ItemB it = item_of_b(w, BH, nq, T, causal);
            for (int j = 0; j < it.nkv && ok; ++j, ++G, ++kc) {
                const int s = kc % KST;
                if (!mbar_wait(smem_u32(&bars->p_full[G & 1]), (G >> 1) & 1, wc)) { ok = false; break; }
                // the first tile overwrites dQ and dR: the previous item's epilogue must have read them
                if (j == 0 && ic > 0 && !mbar_wait(smem_u32(&bars->om_free), (ic - 1) & 1, wc)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t kd = dkm + (uint64_t)(s * (Gm::T_BYTES >> 4));
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    const uint64_t bdesc = kd + (uint64_t)((kk * 16 * 128) >> 4);
                    const uint32_t acc = (j == 0 && kk == 0) ? 0u : 1u;
                    const uint32_t zc = tmem + col_x(G) + col_dz(kk);
                    umma_ts(tmem + COL_DQ, zc, bdesc, IDESC_DQ, acc);
                    umma_ts(tmem + COL_DR, zc + DA_SHIFT, bdesc, IDESC_DQ, acc);
                }
                tc_commit(smem_u32(&bars->k_empty[s]));
                tc_commit(smem_u32(&bars->pv_done[G & 1]));
            }
        }
        tc_commit(smem_u32(&bars->drain[1]));
        mbar_wait_drain(smem_u32(&bars->drain[1]), 0, DRAIN_NS);
    } else if (warp >= FIRST_SOFT_WARP && warp < DQ_WARP) {
        // =================================== elementwise + epilogue ==
        const int grp = (warp - FIRST_SOFT_WARP) >> 2;   // keys [32 grp, 32 grp + 32) of each tile
        const int quarter = warp & 3;                    // TMEM lane quarter this warp may access
        const int r = quarter * 32 + lane;               // query row within the tile == TMEM lane
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const float sc = LOG2E / sqrtf((float)D), inv_sqrt = 1.0f / sqrtf((float)D);
        uint32_t G = 0;
        bool ok = true;
        for (uint32_t ic = 0; ok; ++ic) {
            int w = 0;
            const bool got = next_item<SCHED>(bars, ic, w, wc);
            if (!__all_sync(0xffffffffu, got)) break;
            if (lane == 0) mbar_arrive(smem_u32(&bars->sched_empty[ic % SCHED]));
            if (w >= items) break;
            const ItemB it = item_of_b(w, BH, nq, T, causal);
            const int qrow = it.qt * BM + r;
            const bool live = qrow < T;
            const size_t ri = (size_t)it.bh * T + (live ? qrow : 0);
            // this row's statistics; rows past T get zero weights
            const float l2 = live ? lse[ri] * LOG2E : INFINITY;
            const float ab = live ? abar[ri] : 0.f, gov = live ? go[ri] : 0.f, dl = live ? delta[ri] : 0.f;
            const int kvis = causal ? min(T, qrow + 1) : T;   // keys visible to this row
            for (int j = 0; j < it.nkv; ++j, ++G) {
                const uint32_t xcol = tmem + lane_off + col_x(G) + grp * GCOLS;   // this group's columns
                // ---- s = exp(z - lse) of this group's 32 keys, as fp16 pairs ----
                if (!warp_wait(smem_u32(&bars->s_full), G & 1, wc)) { ok = false; break; }
                tc_fence_after();
                uint32_t sp[GCOLS / 2];
                {
                    uint32_t sr[GCOLS];
                    tmem_ld16(xcol, *reinterpret_cast<uint32_t(*)[16]>(&sr[0]));
                    tmem_ld16(xcol + 16, *reinterpret_cast<uint32_t(*)[16]>(&sr[16]));
                    tmem_wait_ld();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&bars->s_free));
                    const int limit = kvis - (j * BN + grp * GCOLS);
                    if (limit < GCOLS) {
#pragma unroll
                        for (int c = 0; c < GCOLS; ++c)
                            if (c >= limit) sr[c] = __float_as_uint(-INFINITY);
                    }
                    weights_f16(sr, sp, sc, -l2);
                }
                // ---- a of these keys ----
                if (!warp_wait(smem_u32(&bars->a_full), G & 1, wc)) { ok = false; break; }
                tc_fence_after();
                uint32_t ar[GCOLS];
                tmem_ld16(xcol, *reinterpret_cast<uint32_t(*)[16]>(&ar[0]));
                tmem_ld16(xcol + 16, *reinterpret_cast<uint32_t(*)[16]>(&ar[16]));
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&bars->a_free));
                // ---- G, 16 keys at a time: dZ / sqrt(d) and dA as bf16 over the G
                // columns just read, for the dq and drho products ----
                if (!warp_wait(smem_u32(&bars->g_full), G & 1, wc)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t gv[16];
                    tmem_ld16(xcol + 16 * c, gv);
                    tmem_wait_ld();
                    uint32_t zp[8], dp[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const uint32_t s2 = sp[8 * c + i];
                        const float s0 = __half2float(__ushort_as_half((unsigned short)(s2 & 0xFFFFu)));
                        const float s1 = __half2float(__ushort_as_half((unsigned short)(s2 >> 16)));
                        const float a0 = __uint_as_float(ar[16 * c + 2 * i]), a1 = __uint_as_float(ar[16 * c + 2 * i + 1]);
                        const float g0 = __uint_as_float(gv[2 * i]), g1 = __uint_as_float(gv[2 * i + 1]);
                        const float z0 = s0 * (fmaf(1.f + ab - a0, g0, a0 * gov) - dl) * inv_sqrt;
                        const float z1 = s1 * (fmaf(1.f + ab - a1, g1, a1 * gov) - dl) * inv_sqrt;
                        zp[i] = pack_bf16x2(z0, z1);
                        dp[i] = pack_bf16x2(s0 * (gov - g0), s1 * (gov - g1));
                    }
                    tmem_st8(xcol + 16 * c, zp);
                    tmem_st8(xcol + 16 * c + DA_SHIFT, dp);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&bars->p_full[G & 1]));
            }
            if (!ok) break;
            // ---------------------------------------------- epilogue --
            // the item's last dq / drho products are done: dQ and dR are final
            if (!warp_wait(smem_u32(&bars->pv_done[(G - 1) & 1]), ((G - 1) >> 1) & 1, wc)) break;
            tc_fence_after();
#pragma unroll 1
            for (int c = grp * Gm::OCOLS; c < grp * Gm::OCOLS + Gm::OCOLS; c += 16) {
                uint32_t oq[16], orr[16];
                tmem_ld16(tmem + lane_off + COL_DQ + c, oq);
                tmem_ld16(tmem + lane_off + COL_DR + c, orr);
                tmem_wait_ld();
                if (live) {
                    float4 *dst = reinterpret_cast<float4 *>(dq + ri * D + c);
                    float4 *dsr = reinterpret_cast<float4 *>(drho + ri * D + c);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        dst[i] = make_float4(__uint_as_float(oq[4 * i]), __uint_as_float(oq[4 * i + 1]),
                                             __uint_as_float(oq[4 * i + 2]), __uint_as_float(oq[4 * i + 3]));
                        dsr[i] = make_float4(__uint_as_float(orr[4 * i]), __uint_as_float(orr[4 * i + 1]),
                                             __uint_as_float(orr[4 * i + 2]), __uint_as_float(orr[4 * i + 3]));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bars->om_free));
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int D>
cudaError_t launch_dq_t(const BwdTensorMaps &tm, const float *lse, const float *abar, const float *go,
                        const float *delta, float *dq, float *drho, int BH, int T, int causal, int sm_count,
                        int *work_counter, const DeviceCtl &ctl, cudaStream_t s) {
    static std::atomic<unsigned long long> limit_set{0};
    auto kern = k_bwd_dq_tc<D>;
    if (cudaError_t e = ensure_smem_limit(kern, (int)smem_bytes_b<D>(), limit_set)) return e;
    const int items = ((T + BM - 1) / BM) * BH;
    const int grid = items < sm_count ? items : sm_count;
    cudaError_t e = cudaMemsetAsync(work_counter, 0, sizeof(int), s);
    if (e != cudaSuccess) return e;
    kern<<<grid, NTHREADS, smem_bytes_b<D>(), s>>>(tm.q, tm.r, tm.g, tm.k, tm.v, lse, abar, go, delta, dq, drho, BH,
                                                   T, causal, work_counter, ctl);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_dq_sm100(const BwdTensorMaps &tm, const float *lse, const float *abar, const float *go,
                                const float *delta, float *dq, float *drho, int B, int H, int T, int d, int causal,
                                int sm_count, int *work_counter, const DeviceCtl &ctl, cudaStream_t s) {
    if (d == 64)
        return launch_dq_t<64>(tm, lse, abar, go, delta, dq, drho, B * H, T, causal, sm_count, work_counter, ctl, s);
    return launch_dq_t<128>(tm, lse, abar, go, delta, dq, drho, B * H, T, causal, sm_count, work_counter, ctl, s);
}

}  // namespace plx
