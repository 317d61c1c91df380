// bwd_dkdv_sm100.cu -- dk and dv of the Parallax prefill on the tensor cores
// (tcgen05 + TMA + TMEM), the key-stationary half of the backward.
//
// With the definitions of bwd.cu (the chain rule through the forward; zubnet.ai
// news item on Parallax, paragraph 2, for the operator), per key j and query i
// with g_i = dY_i:
//   W_ij  = s_ij (1 + abar_i - a_ij)                      dv_j = sum_i W_ij g_i
//   dZ_ij = s_ij ((1 + abar_i - a_ij) G_ij + a_ij go_i - delta_i)
//   dA_ij = s_ij (go_i - G_ij)            dk_j = sum_i dZ_ij q_i / sqrt(d) + dA_ij rho_i.
// One CTA per SM, persistent over (head, 128-key tile) items, walks the query
// tiles (64 queries each) that see its keys.  The keys are the TMEM lanes: per
// query tile three products land one after another in a TMEM tile region
// (S^T = K Q^T, A^T = K R^T, G^T = V dY^T: bf16 in, fp32 out, N = 64), the
// elementwise warps read each once, write W^T (bf16) into a W region and
// dZ^T / sqrt(d), dA^T (bf16) over the G columns they have read, and the
// second issuing thread accumulates dv += W^T dY and dk += dZ^T Q + dA^T R in
// TMEM (the Q, R and dY tiles read as MN-major B operands).  The per-query
// statistics (lse log2 e, abar, go, delta) arrive beside the tile as 64 values
// of each in turn, so a thread reads its 16 queries' values of one statistic
// with four 16-byte loads.
//
// TMEM: one 64-column region per score product (S^T, A^T, G^T), so the three
// products of the next query tile can be issued as soon as the elementwise
// warps have read this tile's (the next S^T while this tile's A^T is being
// read, and so on); W regions W0, W1 (32 columns each, query tile t uses
// W(t mod 2)); accumulators dV, dK.
// Shared memory: K and V of the item, a 3-stage ring of (Q, R, dY, statistics)
// per query tile.
//
// Roles (640 threads, persistent, items longest-first from an atomic counter):
//   warp 0 lane 0   scheduler + TMA (K, V per item; the ring per query tile)
//   warp 1          TMEM owner; lane 0 issues S^T, A^T, G^T
//   warps 2..17     four warpgroups; group g takes queries [16g, 16g + 16) of
//                   each tile for all 128 keys (one key per thread); then the
//                   item's epilogue (group g writes d/4 columns of dk, dv)
//   warp 18 lane 0  issues dv += W^T dY, then dk += dZ^T Q + dA^T R
// Every wait is bounded; a wait that gives up lets every role leave its loop.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include "internal.h"
#include "sm100.cuh"
#include "softmax_sm100.cuh"

namespace plx {
namespace {

constexpr int BK = 128;                   // keys per item (TMEM lanes)
constexpr int BQ = 64;                    // queries per tile
constexpr int NGRP = 4;                   // elementwise warpgroups
constexpr int QCOLS = BQ / NGRP;          // queries per group and tile (16)
constexpr int RST = 3;                    // ring stages
constexpr int SCHED = 4;
constexpr int FIRST_SOFT_WARP = 2;
constexpr int NSOFT_WARPS = NGRP * 4;
constexpr int GR_WARP = FIRST_SOFT_WARP + NSOFT_WARPS;   // dk / dv issuer
constexpr int NTHREADS = (GR_WARP + 1) * 32;
constexpr float LOG2E = 1.4426950408889634f;
constexpr unsigned long long DRAIN_NS = 2000000ull;

template <int D> struct GeoK {
    static constexpr int HALVES = D / 64;
    static constexpr int KV_BYTES = BK * D * 2;          // one 128-row bf16 tile
    static constexpr int QT_BYTES = BQ * D * 2;          // one 64-row bf16 tile
    static constexpr int ST_BYTES = 4 * BQ * 4;          // statistics of a query tile: 4 x 64 floats
    static constexpr int STAGE_BYTES = 3 * QT_BYTES + ST_BYTES;   // Q | R | dY | statistics
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + KV_BYTES;
    static constexpr int OFF_RING = OFF_V + KV_BYTES;
    static constexpr int OFF_BARS = OFF_RING + RST * STAGE_BYTES;
    static constexpr int OCOLS = D / NGRP;               // dk / dv columns each group writes
    static_assert(OCOLS % 16 == 0, "16-column TMEM loads");
    static_assert(QT_BYTES % 1024 == 0 && STAGE_BYTES % 1024 == 0, "1024-byte aligned tiles");
};

// TMEM: S^T [0, 64), A^T [64, 128), G^T [128, 192), W0 [192, 224), W1 [224, 256), dV, dK.
constexpr uint32_t COL_S = 0, COL_A = 64, COL_G = 128, COL_W0 = 192, COL_DV = 256, COL_DK = 384;
__host__ __device__ constexpr uint32_t col_w(uint32_t t) { return COL_W0 + (t & 1) * (BQ / 2); }
// In the G region: the bf16 dZ^T of queries [16c, 16c + 16) in columns
// [16c, 16c + 8) and their dA^T in the next 8 (the G columns of those
// queries).  In W: the bf16 W^T of queries [16c, 16c + 16) in columns [8c, 8c + 8).
constexpr uint32_t DA_SHIFT = 8;

constexpr uint32_t IDESC_SC = idesc_f16(1, 1, 0, 0, BK, BQ);                          // bf16 K-major x bf16 K-major
template <int D> constexpr uint32_t idesc_gr() { return idesc_f16(1, 1, 0, 1, BK, D); }   // bf16 (TMEM) x bf16 MN-major

struct __align__(8) BarsK {
    uint64_t kv_full, kv_empty;
    uint64_t st_full[RST], st_empty[RST];
    uint64_t s_full, a_full, g_full;   // score products of the current query tile done
    uint64_t s_free, a_free;           // the elementwise warps have read S^T, A^T
    uint64_t w_full[2];                // per W region: W^T of its tile written
    uint64_t wv_done[2];               // per W region: dv products of its tile done
    uint64_t p_full;                   // dZ^T, dA^T of the current tile written
    uint64_t pv_done;                  // dk products of the current tile done
    uint64_t om_free;                  // the epilogue has read dV and dK
    uint64_t drain[2];
    uint64_t sched_full[SCHED], sched_empty[SCHED];
    int sched_item[SCHED];
    uint32_t tmem_base;
    int abort_flag;
};

template <int D> constexpr size_t smem_bytes_k() { return (size_t)GeoK<D>::OFF_BARS + sizeof(BarsK); }
static_assert(smem_bytes_k<128>() <= 232448, "shared memory budget");

struct ItemK {
    int bh, kt, q0t, nqt;   // head, key tile, first query tile (of 64), query tiles
};

__device__ __forceinline__ ItemK item_of_k(int w, int BH, int nk, int nq64, int causal) {
    ItemK it;
    it.kt = w / BH;          // key tile 0 sees the most queries: longest items first
    it.bh = w % BH;
    it.q0t = causal ? it.kt * (BK / BQ) : 0;
    it.nqt = nq64 - it.q0t;
    (void)nk;
    return it;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

__device__ __forceinline__ float4 ld_shared_f4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
    return v;
}

// 1-D bulk copy global -> shared; completion counted on `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

template <int D>
__global__ void __launch_bounds__(NTHREADS, 1)
    k_bwd_dkdv_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_r,
                  const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const float4 *__restrict__ stats, float *__restrict__ dk,
                  float *__restrict__ dv, int BH, int T, int Tpad, int causal, int *__restrict__ work_counter,
                  DeviceCtl ctl) {
    using Gm = GeoK<D>;
    extern __shared__ __align__(1024) uint8_t smem[];
    if (smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) atomicExch(ctl.err, PARALLAX_ERR_UNSUPPORTED);
        return;
    }
    BarsK *bars = reinterpret_cast<BarsK *>(smem + Gm::OFF_BARS);
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bars->kv_full), 1);
        mbar_init(smem_u32(&bars->kv_empty), 1);
        for (int s = 0; s < RST; ++s) {
            mbar_init(smem_u32(&bars->st_full[s]), 1);
            mbar_init(smem_u32(&bars->st_empty[s]), 1);
        }
        mbar_init(smem_u32(&bars->s_full), 1);
        mbar_init(smem_u32(&bars->a_full), 1);
        mbar_init(smem_u32(&bars->g_full), 1);
        mbar_init(smem_u32(&bars->s_free), NSOFT_WARPS);
        mbar_init(smem_u32(&bars->a_free), NSOFT_WARPS);
        for (int x = 0; x < 2; ++x) {
            mbar_init(smem_u32(&bars->w_full[x]), NSOFT_WARPS);
            mbar_init(smem_u32(&bars->wv_done[x]), 1);
        }
        mbar_init(smem_u32(&bars->p_full), NSOFT_WARPS);
        mbar_init(smem_u32(&bars->pv_done), 1);
        mbar_init(smem_u32(&bars->om_free), NSOFT_WARPS);
        mbar_init(smem_u32(&bars->drain[0]), 1);
        mbar_init(smem_u32(&bars->drain[1]), 1);
        for (int s = 0; s < SCHED; ++s) {
            mbar_init(smem_u32(&bars->sched_full[s]), 1);
            mbar_init(smem_u32(&bars->sched_empty[s]), 2 + NSOFT_WARPS);
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
    const int nk = (T + BK - 1) / BK;
    const int nq64 = Tpad / BQ;
    const int items = nk * BH;

    if (warp == 0 && lane == 0) {
        // ===================================== scheduler + TMA producer ==
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_r);
        tma_prefetch_desc(&tm_g);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        uint32_t tc = 0;
        int st_armed[RST], kv_armed = -1;
        for (int s = 0; s < RST; ++s) st_armed[s] = -1;
        bool ok = true;
        for (uint32_t ic = 0; ok; ++ic) {
            const uint32_t ss = ic % SCHED;
            if (!mbar_wait(smem_u32(&bars->sched_empty[ss]), ((ic / SCHED) & 1) ^ 1, wc)) break;
            const int w = ic == 0 ? (int)blockIdx.x : (int)gridDim.x + atomicAdd(work_counter, 1);
            bars->sched_item[ss] = w;
            mbar_arrive(smem_u32(&bars->sched_full[ss]));
            if (w >= items) break;
            const ItemK it = item_of_k(w, BH, nk, nq64, causal);
            if (!mbar_wait(smem_u32(&bars->kv_empty), (ic & 1) ^ 1, wc)) break;
            const uint32_t kf = smem_u32(&bars->kv_full);
            kv_armed = (int)(ic & 1);
            mbar_arrive_expect_tx(kf, 2 * Gm::KV_BYTES);
#pragma unroll
            for (int h = 0; h < Gm::HALVES; ++h) {
                const uint32_t hoff = h * (Gm::KV_BYTES / Gm::HALVES);
                tma_load_3d(sbase + Gm::OFF_K + hoff, &tm_k, kf, h * 64, it.kt * BK, it.bh);
                tma_load_3d(sbase + Gm::OFF_V + hoff, &tm_v, kf, h * 64, it.kt * BK, it.bh);
            }
            for (int t = 0; t < it.nqt; ++t, ++tc) {
                const int s = tc % RST;
                if (!mbar_wait(smem_u32(&bars->st_empty[s]), ((tc / RST) & 1) ^ 1, wc)) { ok = false; break; }
                const uint32_t f = smem_u32(&bars->st_full[s]);
                const uint32_t stage = sbase + Gm::OFF_RING + s * Gm::STAGE_BYTES;
                const int q0 = (it.q0t + t) * BQ;
                st_armed[s] = (int)((tc / RST) & 1);
                mbar_arrive_expect_tx(f, 3 * Gm::QT_BYTES + Gm::ST_BYTES);
#pragma unroll
                for (int h = 0; h < Gm::HALVES; ++h) {
                    const uint32_t hoff = h * (Gm::QT_BYTES / Gm::HALVES);
                    tma_load_3d(stage + hoff, &tm_q, f, h * 64, q0, it.bh);
                    tma_load_3d(stage + Gm::QT_BYTES + hoff, &tm_r, f, h * 64, q0, it.bh);
                    tma_load_3d(stage + 2 * Gm::QT_BYTES + hoff, &tm_g, f, h * 64, q0, it.bh);
                }
                bulk_load(stage + 3 * Gm::QT_BYTES, stats + (size_t)it.bh * Tpad + q0, Gm::ST_BYTES, f);
            }
        }
        if (kv_armed >= 0) mbar_wait_drain(smem_u32(&bars->kv_full), (uint32_t)kv_armed, DRAIN_NS);
        for (int s = 0; s < RST; ++s)
            if (st_armed[s] >= 0) mbar_wait_drain(smem_u32(&bars->st_full[s]), (uint32_t)st_armed[s], DRAIN_NS);
    } else if (warp == 1 && lane == 0) {
        // ============================================= score UMMA issuer ==
        // Query tile t: S^T(t) once S^T(t - 1) has been read, A^T(t) once
        // A^T(t - 1) has been read, G^T(t) once the dk products of tile t - 1
        // are done with the G region (they read dZ^T, dA^T there).
        uint32_t tc = 0;
        bool ok = true;
        const uint64_t dk_ = sdesc_sw128(sbase + Gm::OFF_K, 16, 1024);
        const uint64_t dv_ = sdesc_sw128(sbase + Gm::OFF_V, 16, 1024);
        const uint64_t dring = sdesc_sw128(sbase + Gm::OFF_RING, 16, 1024);   // stage s: + s * STAGE_BYTES / 16
        auto issue_scores = [&](uint32_t dcol, uint64_t da, uint64_t db) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t aoff = ((uint32_t)(kk >> 2) * (Gm::KV_BYTES / Gm::HALVES) + (uint32_t)(kk & 3) * 32) >> 4;
                const uint32_t boff = ((uint32_t)(kk >> 2) * (Gm::QT_BYTES / Gm::HALVES) + (uint32_t)(kk & 3) * 32) >> 4;
                umma_ss(tmem + dcol, da + aoff, db + boff, IDESC_SC, kk > 0 ? 1u : 0u);
            }
        };
        for (uint32_t ic = 0; ok; ++ic) {
            int w;
            if (!next_item<SCHED>(bars, ic, w, wc)) break;
            mbar_arrive(smem_u32(&bars->sched_empty[ic % SCHED]));
            if (w >= items) break;
            const ItemK it = item_of_k(w, BH, nk, nq64, causal);
            if (!mbar_wait(smem_u32(&bars->kv_full), ic & 1, wc)) break;
            for (int t = 0; t < it.nqt; ++t, ++tc) {
                const int s = tc % RST;
                if (!mbar_wait(smem_u32(&bars->st_full[s]), (tc / RST) & 1, wc)) { ok = false; break; }
                const uint64_t st = dring + (uint64_t)(s * (Gm::STAGE_BYTES >> 4));
                if (tc > 0 && !mbar_wait(smem_u32(&bars->s_free), (tc - 1) & 1, wc)) { ok = false; break; }
                tc_fence_after();
                issue_scores(COL_S, dk_, st);                                             // S^T = K Q^T
                tc_commit(smem_u32(&bars->s_full));
                if (tc > 0 && !mbar_wait(smem_u32(&bars->a_free), (tc - 1) & 1, wc)) { ok = false; break; }
                tc_fence_after();
                issue_scores(COL_A, dk_, st + (uint64_t)(Gm::QT_BYTES >> 4));              // A^T = K R^T
                tc_commit(smem_u32(&bars->a_full));
                if (tc > 0 && !mbar_wait(smem_u32(&bars->pv_done), (tc - 1) & 1, wc)) { ok = false; break; }
                tc_fence_after();
                issue_scores(COL_G, dv_, st + (uint64_t)((2 * Gm::QT_BYTES) >> 4));        // G^T = V dY^T
                tc_commit(smem_u32(&bars->g_full));
                if (t == it.nqt - 1) tc_commit(smem_u32(&bars->kv_empty));
            }
        }
        tc_commit(smem_u32(&bars->drain[0]));
        mbar_wait_drain(smem_u32(&bars->drain[0]), 0, DRAIN_NS);
    } else if (warp == GR_WARP && lane == 0) {
        // ======================================== dv / dk UMMA issuer ==
        uint32_t tc = 0;
        bool ok = true;
        constexpr uint32_t IDESC_GR = idesc_gr<D>();
        // Q, R, dY of a stage as MN-major B operands [queries x d]: 16 queries = 2 KB per k-step
        const uint64_t dring = sdesc_sw128(sbase + Gm::OFF_RING, Gm::QT_BYTES / Gm::HALVES, 1024);
        for (uint32_t ic = 0; ok; ++ic) {
            int w;
            if (!next_item<SCHED>(bars, ic, w, wc)) break;
            mbar_arrive(smem_u32(&bars->sched_empty[ic % SCHED]));
            if (w >= items) break;
            const ItemK it = item_of_k(w, BH, nk, nq64, causal);
            for (int t = 0; t < it.nqt && ok; ++t, ++tc) {
                const int s = tc % RST;
                const uint64_t st = dring + (uint64_t)(s * (Gm::STAGE_BYTES >> 4));
                if (!mbar_wait(smem_u32(&bars->w_full[tc & 1]), (tc >> 1) & 1, wc)) { ok = false; break; }
                // the first tile overwrites dV and dK: the previous item's epilogue must have read them
                if (t == 0 && ic > 0 && !mbar_wait(smem_u32(&bars->om_free), (ic - 1) & 1, wc)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < BQ / 16; ++kk) {   // dv += W^T dY
                    const uint64_t b = st + (uint64_t)((2 * Gm::QT_BYTES + kk * 16 * 128) >> 4);
                    umma_ts(tmem + COL_DV, tmem + col_w(tc) + 8 * kk, b, IDESC_GR, (t == 0 && kk == 0) ? 0u : 1u);
                }
                tc_commit(smem_u32(&bars->wv_done[tc & 1]));
                if (!mbar_wait(smem_u32(&bars->p_full), tc & 1, wc)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < BQ / 16; ++kk) {   // dk += dZ^T Q / sqrt(d) + dA^T R
                    const uint64_t bq = st + (uint64_t)((kk * 16 * 128) >> 4);
                    const uint64_t br = st + (uint64_t)((Gm::QT_BYTES + kk * 16 * 128) >> 4);
                    const uint32_t zc = tmem + COL_G + 16 * kk;
                    umma_ts(tmem + COL_DK, zc, bq, IDESC_GR, (t == 0 && kk == 0) ? 0u : 1u);
                    umma_ts(tmem + COL_DK, zc + DA_SHIFT, br, IDESC_GR, 1u);
                }
                tc_commit(smem_u32(&bars->st_empty[s]));
                tc_commit(smem_u32(&bars->pv_done));
            }
        }
        tc_commit(smem_u32(&bars->drain[1]));
        mbar_wait_drain(smem_u32(&bars->drain[1]), 0, DRAIN_NS);
    } else if (warp >= FIRST_SOFT_WARP && warp < GR_WARP) {
        // =================================== elementwise + epilogue ==
        const int grp = (warp - FIRST_SOFT_WARP) >> 2;   // queries [16 grp, 16 grp + 16) of each tile
        const int quarter = warp & 3;                    // TMEM lane quarter this warp may access
        const int r = quarter * 32 + lane;               // key within the item == TMEM lane
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const float sc = LOG2E / sqrtf((float)D), inv_sqrt = 1.0f / sqrtf((float)D);
        uint32_t tc = 0;
        bool ok = true;
        for (uint32_t ic = 0; ok; ++ic) {
            int w = 0;
            const bool got = next_item<SCHED>(bars, ic, w, wc);
            if (!__all_sync(0xffffffffu, got)) break;
            if (lane == 0) mbar_arrive(smem_u32(&bars->sched_empty[ic % SCHED]));
            if (w >= items) break;
            const ItemK it = item_of_k(w, BH, nk, nq64, causal);
            const int key = it.kt * BK + r;
            for (int t = 0; t < it.nqt; ++t, ++tc) {
                const int s = tc % RST;
                const uint32_t xcol = tmem + lane_off + grp * QCOLS;   // + COL_S, COL_A, COL_G
                // this group's 16 values of statistic k at stq + k * 256 (lse log2 e, abar, go, delta)
                const uint32_t stq = sbase + Gm::OFF_RING + s * Gm::STAGE_BYTES + 3 * Gm::QT_BYTES + grp * QCOLS * 4;
                const int qfirst = (it.q0t + t) * BQ + grp * QCOLS;   // this group's first query
                if (!warp_wait(smem_u32(&bars->st_full[s]), (tc / RST) & 1, wc)) { ok = false; break; }
                // ---- s = exp(z - lse) of this key and the group's 16 queries ----
                if (!warp_wait(smem_u32(&bars->s_full), tc & 1, wc)) { ok = false; break; }
                tc_fence_after();
                float sv[QCOLS];
                {
                    uint32_t sr[QCOLS];
                    tmem_ld16(xcol + COL_S, sr);
                    tmem_wait_ld();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&bars->s_free));
#pragma unroll
                    for (int c4 = 0; c4 < QCOLS / 4; ++c4) {
                        const float4 l2 = ld_shared_f4(stq + c4 * 16);   // +inf for queries past T
                        const float l2v[4] = {l2.x, l2.y, l2.z, l2.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int c = 4 * c4 + e;
                            const bool vis = !causal || qfirst + c >= key;
                            sv[c] = vis ? ex2(fmaf(__uint_as_float(sr[c]), sc, -l2v[e])) : 0.f;
                        }
                    }
                }
                // ---- a, then W^T = s (1 + abar - a) into the tile's W region ----
                if (!warp_wait(smem_u32(&bars->a_full), tc & 1, wc)) { ok = false; break; }
                tc_fence_after();
                uint32_t ar[QCOLS];
                tmem_ld16(xcol + COL_A, ar);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&bars->a_free));
                {
                    uint32_t wp[QCOLS / 2];
#pragma unroll
                    for (int c4 = 0; c4 < QCOLS / 4; ++c4) {
                        const float4 ab = ld_shared_f4(stq + 256 + c4 * 16);
                        const int c = 4 * c4;
                        wp[2 * c4] = pack_bf16x2(sv[c] * (1.f + ab.x - __uint_as_float(ar[c])),
                                                 sv[c + 1] * (1.f + ab.y - __uint_as_float(ar[c + 1])));
                        wp[2 * c4 + 1] = pack_bf16x2(sv[c + 2] * (1.f + ab.z - __uint_as_float(ar[c + 2])),
                                                     sv[c + 3] * (1.f + ab.w - __uint_as_float(ar[c + 3])));
                    }
                    // the region's previous tile has been consumed by its dv products
                    if (tc >= 2 && !warp_wait(smem_u32(&bars->wv_done[tc & 1]), ((tc - 2) >> 1) & 1, wc)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    tmem_st8(tmem + lane_off + col_w(tc) + 8 * grp, wp);
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&bars->w_full[tc & 1]));
                }
                // ---- G, then dZ^T / sqrt(d) and dA^T as bf16 over the G columns ----
                if (!warp_wait(smem_u32(&bars->g_full), tc & 1, wc)) { ok = false; break; }
                tc_fence_after();
                {
                    uint32_t gv[QCOLS];
                    tmem_ld16(xcol + COL_G, gv);
                    tmem_wait_ld();
                    uint32_t zp[QCOLS / 2], dp[QCOLS / 2];
#pragma unroll
                    for (int c4 = 0; c4 < QCOLS / 4; ++c4) {
                        const float4 ab4 = ld_shared_f4(stq + 256 + c4 * 16), go4 = ld_shared_f4(stq + 512 + c4 * 16),
                                     dl4 = ld_shared_f4(stq + 768 + c4 * 16);
                        const float abv[4] = {ab4.x, ab4.y, ab4.z, ab4.w}, gov[4] = {go4.x, go4.y, go4.z, go4.w},
                                    dlv[4] = {dl4.x, dl4.y, dl4.z, dl4.w};
                        float z[4], da[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int c = 4 * c4 + e;
                            const float a = __uint_as_float(ar[c]), g = __uint_as_float(gv[c]);
                            z[e] = sv[c] * (fmaf(1.f + abv[e] - a, g, a * gov[e]) - dlv[e]) * inv_sqrt;
                            da[e] = sv[c] * (gov[e] - g);
                        }
                        zp[2 * c4] = pack_bf16x2(z[0], z[1]);
                        zp[2 * c4 + 1] = pack_bf16x2(z[2], z[3]);
                        dp[2 * c4] = pack_bf16x2(da[0], da[1]);
                        dp[2 * c4 + 1] = pack_bf16x2(da[2], da[3]);
                    }
                    tmem_st8(xcol + COL_G, zp);
                    tmem_st8(xcol + COL_G + DA_SHIFT, dp);
                    tmem_wait_st();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&bars->p_full));
            }
            if (!ok) break;
            // ---------------------------------------------- epilogue --
            // the item's last dk products are done (its dv products came first): dV, dK are final
            if (!warp_wait(smem_u32(&bars->pv_done), (tc - 1) & 1, wc)) break;
            tc_fence_after();
            const bool store = key < T;
            const size_t row = (size_t)it.bh * T + (store ? key : 0);
#pragma unroll 1
            for (int c = grp * Gm::OCOLS; c < grp * Gm::OCOLS + Gm::OCOLS; c += 16) {
                uint32_t ov[16], ok2[16];
                tmem_ld16(tmem + lane_off + COL_DV + c, ov);
                tmem_ld16(tmem + lane_off + COL_DK + c, ok2);
                tmem_wait_ld();
                if (store) {
                    float4 *pv = reinterpret_cast<float4 *>(dv + row * D + c);
                    float4 *pk = reinterpret_cast<float4 *>(dk + row * D + c);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        pv[i] = make_float4(__uint_as_float(ov[4 * i]), __uint_as_float(ov[4 * i + 1]),
                                            __uint_as_float(ov[4 * i + 2]), __uint_as_float(ov[4 * i + 3]));
                        pk[i] = make_float4(__uint_as_float(ok2[4 * i]), __uint_as_float(ok2[4 * i + 1]),
                                            __uint_as_float(ok2[4 * i + 2]), __uint_as_float(ok2[4 * i + 3]));
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
cudaError_t launch_dkdv_t(const BwdTensorMaps &tm, const float4 *stats, float *dk, float *dv, int BH, int T, int causal,
                          int sm_count, int *work_counter, const DeviceCtl &ctl, cudaStream_t s) {
    static std::atomic<unsigned long long> limit_set{0};
    auto kern = k_bwd_dkdv_tc<D>;
    if (cudaError_t e = ensure_smem_limit(kern, (int)smem_bytes_k<D>(), limit_set)) return e;
    const int Tpad = (T + BQ - 1) / BQ * BQ;
    const int items = ((T + BK - 1) / BK) * BH;
    const int grid = items < sm_count ? items : sm_count;
    cudaError_t e = cudaMemsetAsync(work_counter, 0, sizeof(int), s);
    if (e != cudaSuccess) return e;
    kern<<<grid, NTHREADS, smem_bytes_k<D>(), s>>>(tm.q, tm.r, tm.g, tm.k, tm.v, stats, dk, dv, BH, T, Tpad, causal,
                                                   work_counter, ctl);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_dkdv_sm100(const BwdTensorMaps &tm, const void *stats, float *dk, float *dv, int B, int H, int T,
                                  int d, int causal, int sm_count, int *work_counter, const DeviceCtl &ctl,
                                  cudaStream_t s) {
    const float4 *st = static_cast<const float4 *>(stats);
    if (d == 64) return launch_dkdv_t<64>(tm, st, dk, dv, B * H, T, causal, sm_count, work_counter, ctl, s);
    return launch_dkdv_t<128>(tm, st, dk, dv, B * H, T, causal, sm_count, work_counter, ctl, s);
}

}  // namespace plx
