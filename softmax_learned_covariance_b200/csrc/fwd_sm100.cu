// fwd_sm100.cu -- Parallax prefill/forward on the tensor cores (tcgen05 + TMA + TMEM).
//
// Operator (zubnet.ai news item on Parallax, paragraph 2): softmax attention
// minus the softmax-weighted KV covariance projected by the probe rho_i,
//   y_i = o_i - (m_i - o_i abar_i),  a_ij = k_j . rho_i.
// The pages' kernel keeps FlashAttention's KV streaming and reuses each K/V
// tile for both branches (encorp.ai blog "Integraciones de IA personalizadas
// tras la atencion Parallax", section "Como cambia Parallax la historia del
// hardware en GPU Hopper").  Here each 64-key tile is brought into shared
// memory once by TMA and feeds four UMMAs per 128-row query tile:
//   S = Q K^T,  A = R K^T                       (bf16 x bf16 -> fp32, TMEM)
//   O += P V,   M' += (P o A') V                (fp16 x fp16 -> fp32, TMEM)
// with P = exp2(S log2e/sqrt(d) - m_ref) and A' = A / 256 staged as fp16 into
// the TMEM columns of S and A.  fp16 (not bf16) for these operands keeps the
// rounding of P o A inside the error budget; the row sums l = sum P and
// Abar' = sum P o A' are taken from the same rounded fp16 values the MMAs
// consume, so the result is exact for the rounded weights.  The 1/256 factor
// keeps P o A' finite for any |a| < 65504 while P may grow to 2^8 between
// rescales (the running max is only moved when it rises by more than 8 in
// log2 units; O and M are then rescaled in TMEM).
//
// Roles (384 threads, one CTA per SM, persistent over (head, query tile)
// items taken longest-first from an atomic work counter):
//   warp 0      scheduler + TMA producer: Q and R per item, K and V(fp16) rings
//   warp 1      TMEM owner and single-thread UMMA issuer
//   warps 4..11 two softmax warpgroups, one query row per thread in each; the
//               group g handles key columns [32g, 32g+32) of every 64-key tile,
//               the two exchange their partial row max through shared memory
// TMEM (512 columns): O [0,128) | M' [128,256) | S0 | A0 | S1 | A1 (64 each),
// S/A double-buffered so the score UMMAs of tile j+1 run while tile j is
// exponentiated.
//
// WITH_RHO = false is the softmax-only instantiation: the same code with the
// R loads, the A/M UMMAs and the correction arithmetic removed.  With rho = 0
// the full instantiation produces A = 0, M' = 0, Abar' = 0 and hence y = o,
// bit-for-bit the softmax-only result.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include "internal.h"
#include "sm100.cuh"

namespace plx {
namespace {

constexpr int D = 128;
constexpr int BM = 128;          // query rows per tile
constexpr int BN = 64;           // keys per tile
constexpr int HALF = BN / 2;     // key columns per softmax warpgroup
constexpr int KST = 4;           // K ring stages
constexpr int VST = 4;           // V ring stages
constexpr int SCHED = 4;         // scheduler ring depth (items in flight)
constexpr int NTHREADS = 384;
constexpr int NSOFT = 256;       // softmax threads (two warpgroups)
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;
constexpr float RESCALE_THRESHOLD = 8.0f;   // log2 units
constexpr float A_SCALE = 1.0f / 256.0f;
constexpr float A_UNSCALE = 256.0f;

constexpr int Q_BYTES = BM * D * 2;    // 32 KB, two 64-column halves of [128 x 128 B]
constexpr int K_BYTES = BN * D * 2;    // 16 KB, two halves of [64 x 128 B]
constexpr int V_BYTES = BN * D * 2;    // 16 KB fp16, two d-halves of [64 keys x 128 B]

// TMEM column map
constexpr uint32_t COL_O = 0, COL_M = 128;
__host__ __device__ constexpr uint32_t col_s(uint32_t b) { return 256 + b * 128; }
__host__ __device__ constexpr uint32_t col_a(uint32_t b) { return 256 + b * 128 + 64; }
// fp16 P (or P o A') of key group kk (16 keys) inside the S (or A) buffer: each
// warpgroup packs its 32 keys into the first 16 columns of its own 32-column half.
__host__ __device__ constexpr uint32_t col_p16(uint32_t kk) { return (kk >> 1) * 32 + (kk & 1) * 8; }

constexpr uint32_t IDESC_S = idesc_f16(1, 1, 0, 0, BM, BN);     // bf16 Q/R (K-major) x bf16 K (K-major)
constexpr uint32_t IDESC_PV = idesc_f16(0, 0, 0, 1, BM, D);     // f16 P (TMEM) x f16 V (MN-major)

struct __align__(8) Bars {
    uint64_t qr_full, qr_empty;
    uint64_t k_full[KST], k_empty[KST];
    uint64_t v_full[VST], v_empty[VST];
    uint64_t s_full[2], p_full[2], pv_done[2];
    uint64_t om_free;
    uint64_t sched_full[SCHED], sched_empty[SCHED];
    uint64_t xchg[2];            // per tile parity: both softmax groups posted their partial max
    uint64_t esum;               // per item: both softmax groups posted their partial sums
    int sched_item[SCHED];
    uint32_t tmem_base;
    int abort_flag;
    float red_max[2][2][BM];     // [tile parity][warpgroup][row] partial row max
    float red_sum[2][2][BM];     // [l or abar'][warpgroup][row] partial sums for the epilogue
};

constexpr size_t SMEM_BYTES = 1024 + 2 * (size_t)Q_BYTES + (size_t)KST * K_BYTES + (size_t)VST * V_BYTES + sizeof(Bars);

struct Item {
    int bh, qt, nkv;
};

__device__ __forceinline__ Item item_of(int w, int BH, int nq, int T, int causal) {
    Item it;
    it.qt = nq - 1 - w / BH;   // longest rows first
    it.bh = w % BH;
    const int kend = causal ? min(T, (it.qt + 1) * BM) : T;
    it.nkv = (kend + BN - 1) / BN;
    return it;
}

// Bounded wait whose outcome is the same for all 32 lanes (lanes that saw the
// phase complete still give up if another lane of the warp gave up), so the
// .sync.aligned tcgen05 instructions that follow are never reached divergently.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const WaitCtl &wc) {
    const bool got = mbar_wait(bar, parity, wc);
    return __all_sync(0xffffffffu, got);
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Consumers take the k-th scheduled item from the ring (same sequence in every role).
__device__ __forceinline__ bool next_item(Bars *bars, uint32_t k, int &w, const WaitCtl &wc) {
    const uint32_t s = k % SCHED;
    if (!mbar_wait(smem_u32(&bars->sched_full[s]), (k / SCHED) & 1, wc)) return false;
    w = bars->sched_item[s];
    return true;
}

template <bool WITH_RHO, typename Tout>
__global__ void __launch_bounds__(NTHREADS, 1)
    k_fwd(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
          const __grid_constant__ CUtensorMap tm_r, const __grid_constant__ CUtensorMap tm_v, Tout *__restrict__ y,
          float *__restrict__ lse, int BH, int T, int causal, int *__restrict__ work_counter, DeviceCtl ctl) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem;
    uint8_t *sR = sQ + Q_BYTES;
    uint8_t *sK = sR + Q_BYTES;
    uint8_t *sV = sK + KST * K_BYTES;
    Bars *bars = reinterpret_cast<Bars *>(sV + VST * V_BYTES);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bars->qr_full), 1);
        mbar_init(smem_u32(&bars->qr_empty), 1);
        for (int s = 0; s < KST; ++s) {
            mbar_init(smem_u32(&bars->k_full[s]), 1);
            mbar_init(smem_u32(&bars->k_empty[s]), 1);
        }
        for (int s = 0; s < VST; ++s) {
            mbar_init(smem_u32(&bars->v_full[s]), 1);
            mbar_init(smem_u32(&bars->v_empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&bars->s_full[b]), 1);
            mbar_init(smem_u32(&bars->p_full[b]), NSOFT);
            mbar_init(smem_u32(&bars->pv_done[b]), 1);
        }
        mbar_init(smem_u32(&bars->om_free), NSOFT);
        for (int s = 0; s < SCHED; ++s) {
            mbar_init(smem_u32(&bars->sched_full[s]), 1);
            mbar_init(smem_u32(&bars->sched_empty[s]), 1 + NSOFT / 32);   // UMMA thread + one lane per softmax warp
        }
        mbar_init(smem_u32(&bars->xchg[0]), NSOFT);
        mbar_init(smem_u32(&bars->xchg[1]), NSOFT);
        mbar_init(smem_u32(&bars->esum), NSOFT);
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
    WaitCtl wc{ctl.err, &bars->abort_flag, globaltimer_ns() + ctl.wait_ns};

    const int nq = (T + BM - 1) / BM;
    const int items = nq * BH;

    if (warp == 0 && lane == 0) {
        // ============================================= scheduler + producer ==
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        if (WITH_RHO) tma_prefetch_desc(&tm_r);
        uint32_t kc = 0, vc = 0;
        bool ok = true;
        for (uint32_t ic = 0; ok; ++ic) {
            const uint32_t ss = ic % SCHED;
            if (!mbar_wait(smem_u32(&bars->sched_empty[ss]), ((ic / SCHED) & 1) ^ 1, wc)) break;
            const int w = ic == 0 ? (int)blockIdx.x : (int)gridDim.x + atomicAdd(work_counter, 1);
            bars->sched_item[ss] = w;
            mbar_arrive(smem_u32(&bars->sched_full[ss]));
            if (w >= items) break;
            const Item it = item_of(w, BH, nq, T, causal);
            const int q0 = it.qt * BM;
            if (!mbar_wait(smem_u32(&bars->qr_empty), (ic & 1) ^ 1, wc)) break;
            const uint32_t qf = smem_u32(&bars->qr_full);
            mbar_arrive_expect_tx(qf, WITH_RHO ? 2 * Q_BYTES : Q_BYTES);
            tma_load_3d(smem_u32(sQ), &tm_q, qf, 0, q0, it.bh);
            tma_load_3d(smem_u32(sQ) + Q_BYTES / 2, &tm_q, qf, 64, q0, it.bh);
            if (WITH_RHO) {
                tma_load_3d(smem_u32(sR), &tm_r, qf, 0, q0, it.bh);
                tma_load_3d(smem_u32(sR) + Q_BYTES / 2, &tm_r, qf, 64, q0, it.bh);
            }
            for (int j = 0; j < it.nkv; ++j) {
                {
                    const int s = kc % KST;
                    if (!mbar_wait(smem_u32(&bars->k_empty[s]), ((kc / KST) & 1) ^ 1, wc)) { ok = false; break; }
                    const uint32_t f = smem_u32(&bars->k_full[s]);
                    const uint32_t dst = smem_u32(sK + s * K_BYTES);
                    const bool skip = (ctl.debug_flags & DEBUG_FWD_SKIP_FIRST_K_LOAD) && kc == 0;
                    if (!skip) {
                        mbar_arrive_expect_tx(f, K_BYTES);
                        tma_load_3d(dst, &tm_k, f, 0, j * BN, it.bh);
                        tma_load_3d(dst + K_BYTES / 2, &tm_k, f, 64, j * BN, it.bh);
                    }
                    ++kc;
                }
                {
                    const int s = vc % VST;
                    if (!mbar_wait(smem_u32(&bars->v_empty[s]), ((vc / VST) & 1) ^ 1, wc)) { ok = false; break; }
                    const uint32_t f = smem_u32(&bars->v_full[s]);
                    const uint32_t dst = smem_u32(sV + s * V_BYTES);
                    mbar_arrive_expect_tx(f, V_BYTES);
                    tma_load_3d(dst, &tm_v, f, 0, j * BN, it.bh);
                    tma_load_3d(dst + V_BYTES / 2, &tm_v, f, 64, j * BN, it.bh);
                    ++vc;
                }
            }
        }
    } else if (warp == 1 && lane == 0) {
        // ==================================================== UMMA issuer ==
        uint32_t kc = 0, vc = 0, G = 0;
        bool ok = true;
        const uint32_t q_base = smem_u32(sQ), r_base = smem_u32(sR);
        auto issue_pv = [&](uint32_t g, bool first, uint32_t icur) -> bool {
            const uint32_t b = g & 1;
            if (!mbar_wait(smem_u32(&bars->p_full[b]), (g >> 1) & 1, wc)) return false;
            const int s = vc % VST;
            if (!mbar_wait(smem_u32(&bars->v_full[s]), (vc / VST) & 1, wc)) return false;
            if (first && icur > 0)
                if (!mbar_wait(smem_u32(&bars->om_free), (icur - 1) & 1, wc)) return false;
            tc_fence_after();
            const uint32_t vb = smem_u32(sV + s * V_BYTES);
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk) {
                const uint64_t vdesc = sdesc_sw128(vb + kk * 16 * 128, V_BYTES / 2, 1024);
                const uint32_t acc = (!first || kk > 0) ? 1u : 0u;
                umma_ts(tmem + COL_O, tmem + col_s(b) + col_p16(kk), vdesc, IDESC_PV, acc);
                if constexpr (WITH_RHO) umma_ts(tmem + COL_M, tmem + col_a(b) + col_p16(kk), vdesc, IDESC_PV, acc);
            }
            tc_commit(smem_u32(&bars->v_empty[s]));
            tc_commit(smem_u32(&bars->pv_done[b]));
            ++vc;
            return true;
        };
        for (uint32_t ic = 0; ok; ++ic) {
            int w;
            if (!next_item(bars, ic, w, wc)) break;
            mbar_arrive(smem_u32(&bars->sched_empty[ic % SCHED]));
            if (w >= items) break;
            const Item it = item_of(w, BH, nq, T, causal);
            if (!mbar_wait(smem_u32(&bars->qr_full), ic & 1, wc)) break;
            for (int j = 0; j < it.nkv; ++j, ++G) {
                const uint32_t b = G & 1;
                const int s = kc % KST;
                if (!mbar_wait(smem_u32(&bars->k_full[s]), (kc / KST) & 1, wc)) { ok = false; break; }
                tc_fence_after();
                const uint32_t kb = smem_u32(sK + s * K_BYTES);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t half = kk >> 2, sub = kk & 3;
                    const uint64_t qdesc = sdesc_sw128(q_base + half * (Q_BYTES / 2) + sub * 32, 16, 1024);
                    const uint64_t kdesc = sdesc_sw128(kb + half * (K_BYTES / 2) + sub * 32, 16, 1024);
                    umma_ss(tmem + col_s(b), qdesc, kdesc, IDESC_S, kk > 0 ? 1u : 0u);
                    if constexpr (WITH_RHO) {
                        const uint64_t rdesc = sdesc_sw128(r_base + half * (Q_BYTES / 2) + sub * 32, 16, 1024);
                        umma_ss(tmem + col_a(b), rdesc, kdesc, IDESC_S, kk > 0 ? 1u : 0u);
                    }
                }
                tc_commit(smem_u32(&bars->k_empty[s]));
                tc_commit(smem_u32(&bars->s_full[b]));
                if (j == it.nkv - 1) tc_commit(smem_u32(&bars->qr_empty));
                ++kc;
                if (j >= 1 && !issue_pv(G - 1, j == 1, ic)) { ok = false; break; }
            }
            if (!ok) break;
            if (!issue_pv(G - 1, it.nkv == 1, ic)) break;
        }
    } else if (warp >= 4) {
        // ============================================ softmax + epilogue ==
        const int grp = (warp - 4) >> 2;                 // 0: key columns [0,32), 1: [32,64)
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;               // query row within the tile == TMEM lane
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const float scale_log2 = LOG2E / sqrtf((float)D);
        uint32_t G = 0, ni = 0;   // key tiles and items processed by this CTA
        bool ok = true;
        for (uint32_t ic = 0; ok; ++ic) {
            int w = 0;
            const bool got = next_item(bars, ic, w, wc);
            if (!__all_sync(0xffffffffu, got)) break;
            if (lane == 0) mbar_arrive(smem_u32(&bars->sched_empty[ic % SCHED]));
            if (w >= items) break;
            const Item it = item_of(w, BH, nq, T, causal);
            const int qrow = it.qt * BM + r;
            const int kvis = causal ? min(T, qrow + 1) : T;  // keys visible to this row
            float m_ref = -INFINITY;
            float l4[4] = {0.f, 0.f, 0.f, 0.f}, a4[4] = {0.f, 0.f, 0.f, 0.f};
            for (int j = 0; j < it.nkv; ++j, ++G) {
                const uint32_t b = G & 1;
                if (!warp_wait(smem_u32(&bars->s_full[b]), (G >> 1) & 1, wc)) { ok = false; break; }
                tc_fence_after();
                uint32_t sr[HALF];
                uint32_t ar[WITH_RHO ? HALF : 1];
                tmem_ld16(tmem + lane_off + col_s(b) + grp * HALF, *reinterpret_cast<uint32_t(*)[16]>(&sr[0]));
                tmem_ld16(tmem + lane_off + col_s(b) + grp * HALF + 16, *reinterpret_cast<uint32_t(*)[16]>(&sr[16]));
                if constexpr (WITH_RHO) {
                    tmem_ld16(tmem + lane_off + col_a(b) + grp * HALF, *reinterpret_cast<uint32_t(*)[16]>(&ar[0]));
                    tmem_ld16(tmem + lane_off + col_a(b) + grp * HALF + 16,
                              *reinterpret_cast<uint32_t(*)[16]>(&ar[16]));
                }
                tmem_wait_ld();
                // keys of this tile visible to this row: c < limit
                const int limit = kvis - (j * BN + grp * HALF);
                if (limit < HALF) {
#pragma unroll
                    for (int c = 0; c < HALF; ++c)
                        if (c >= limit) sr[c] = __float_as_uint(-INFINITY);
                }
                float mx;
                {
                    float t[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        t[i] = fmax3(__uint_as_float(sr[i]), __uint_as_float(sr[i + 8]),
                                     __uint_as_float(sr[i + 16]));
#pragma unroll
                    for (int i = 0; i < 8; ++i) t[i] = fmaxf(t[i], __uint_as_float(sr[i + 24]));
                    mx = fmaxf(fmax3(t[0], t[1], t[2]), fmax3(t[3], t[4], fmax3(t[5], t[6], t[7])));
                }
                bars->red_max[G & 1][grp][r] = mx;
                mbar_arrive(smem_u32(&bars->xchg[G & 1]));
                if (!warp_wait(smem_u32(&bars->xchg[G & 1]), (G >> 1) & 1, wc)) { ok = false; break; }
                mx = fmaxf(mx, bars->red_max[G & 1][grp ^ 1][r]) * scale_log2;
                float alpha = 1.f;
                bool moved = false;
                if (mx > m_ref + RESCALE_THRESHOLD) {
                    alpha = ex2(m_ref - mx);     // 0 when m_ref = -inf
                    m_ref = mx;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        l4[i] *= alpha;
                        a4[i] *= alpha;
                    }
                    moved = true;
                }
                // O and M' hold earlier tiles of this item: rescale them in TMEM,
                // each warpgroup its half of the columns.
                if (__any_sync(0xffffffffu, moved && j > 0)) {
                    const uint32_t gp = G - 1;
                    if (!warp_wait(smem_u32(&bars->pv_done[gp & 1]), (gp >> 1) & 1, wc)) { ok = false; break; }
                    tc_fence_after();
                    const float f = (moved && j > 0) ? alpha : 1.f;
#pragma unroll 1
                    for (int c = grp * 64; c < grp * 64 + 64; c += 16) {
                        uint32_t t[16];
                        tmem_ld16(tmem + lane_off + COL_O + c, t);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 16; ++i) t[i] = __float_as_uint(__uint_as_float(t[i]) * f);
                        tmem_st16(tmem + lane_off + COL_O + c, t);
                        if constexpr (WITH_RHO) {
                            tmem_ld16(tmem + lane_off + COL_M + c, t);
                            tmem_wait_ld();
#pragma unroll
                            for (int i = 0; i < 16; ++i) t[i] = __float_as_uint(__uint_as_float(t[i]) * f);
                            tmem_st16(tmem + lane_off + COL_M + c, t);
                        }
                    }
                }
                // P = exp2(z*log2e - m_ref) as fp16; P o A' as fp16; sums from the rounded values
                const float neg_m = -m_ref;
                uint32_t pk[HALF / 2];
                uint32_t pak[WITH_RHO ? HALF / 2 : 1];
#pragma unroll
                for (int i = 0; i < HALF / 2; ++i) {
                    const float p0 = ex2(fmaf(__uint_as_float(sr[2 * i]), scale_log2, neg_m));
                    const float p1 = ex2(fmaf(__uint_as_float(sr[2 * i + 1]), scale_log2, neg_m));
                    pk[i] = pack_f16x2(p0, p1);
                    l4[i & 3] = add_f16x2_to_f32(l4[i & 3], pk[i]);
                    if constexpr (WITH_RHO) {
                        const uint32_t ah = pack_f16x2(__uint_as_float(ar[2 * i]) * A_SCALE,
                                                       __uint_as_float(ar[2 * i + 1]) * A_SCALE);
                        pak[i] = hmul2(pk[i], ah);
                        a4[i & 3] = add_f16x2_to_f32(a4[i & 3], pak[i]);
                    }
                }
                tmem_st16(tmem + lane_off + col_s(b) + grp * HALF, pk);
                if constexpr (WITH_RHO) tmem_st16(tmem + lane_off + col_a(b) + grp * HALF, pak);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(smem_u32(&bars->p_full[b]));
            }
            if (!ok) break;
            // ---------------------------------------------- epilogue --
            bars->red_sum[0][grp][r] = (l4[0] + l4[1]) + (l4[2] + l4[3]);
            bars->red_sum[1][grp][r] = (a4[0] + a4[1]) + (a4[2] + a4[3]);
            mbar_arrive(smem_u32(&bars->esum));
            if (!warp_wait(smem_u32(&bars->esum), ni & 1, wc)) break;
            ++ni;
            const float l = bars->red_sum[0][0][r] + bars->red_sum[0][1][r];
            const float ab = bars->red_sum[1][0][r] + bars->red_sum[1][1][r];
            const uint32_t glast = G - 1;
            if (it.nkv >= 2) {
                const uint32_t gp = glast - 1;
                if (!warp_wait(smem_u32(&bars->pv_done[gp & 1]), (gp >> 1) & 1, wc)) break;
            }
            if (!warp_wait(smem_u32(&bars->pv_done[glast & 1]), (glast >> 1) & 1, wc)) break;
            tc_fence_after();
            const float inv_l = 1.0f / l;
            const float abar = ab * inv_l;
            const bool store = qrow < T;
            Tout *yrow = y + ((size_t)it.bh * T + (store ? qrow : 0)) * D;
#pragma unroll 1
            for (int c = grp * 64; c < grp * 64 + 64; c += 16) {
                uint32_t o[16], mm[16];
                tmem_ld16(tmem + lane_off + COL_O + c, o);
                if constexpr (WITH_RHO) tmem_ld16(tmem + lane_off + COL_M + c, mm);
                tmem_wait_ld();
                float out[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float ov = __uint_as_float(o[i]) * inv_l;
                    if constexpr (WITH_RHO) {
                        const float mv = __uint_as_float(mm[i]) * inv_l;
                        out[i] = ov - (mv - ov * abar) * A_UNSCALE;
                    } else {
                        out[i] = ov;
                    }
                }
                if (store) {
                    if constexpr (sizeof(Tout) == 4) {
                        float4 *dst = reinterpret_cast<float4 *>(yrow + c);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_float4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]);
                    } else {
                        uint32_t pb[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            __nv_bfloat162 h = __floats2bfloat162_rn(out[2 * i], out[2 * i + 1]);
                            pb[i] = *reinterpret_cast<uint32_t *>(&h);
                        }
                        uint4 *dst = reinterpret_cast<uint4 *>(yrow + c);
                        dst[0] = make_uint4(pb[0], pb[1], pb[2], pb[3]);
                        dst[1] = make_uint4(pb[4], pb[5], pb[6], pb[7]);
                    }
                }
            }
            if (store && grp == 0 && lse != nullptr) lse[(size_t)it.bh * T + qrow] = (m_ref + log2f(l)) * LN2;
            tc_fence_before();
            mbar_arrive(smem_u32(&bars->om_free));
        }
    }

    __syncthreads();
    if (bars->abort_flag) __nanosleep(100000);   // let in-flight copies and MMAs land
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <bool WITH_RHO, typename Tout>
cudaError_t launch_t(const FwdTensorMaps &tm, void *y, float *lse, int BH, int T, int causal, int sm_count,
                     int *work_counter, const DeviceCtl &ctl, cudaStream_t s) {
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(k_fwd<WITH_RHO, Tout>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    const int items = ((T + BM - 1) / BM) * BH;
    const int grid = items < sm_count ? items : sm_count;
    cudaError_t e = cudaMemsetAsync(work_counter, 0, sizeof(int), s);
    if (e != cudaSuccess) return e;
    k_fwd<WITH_RHO, Tout><<<grid, NTHREADS, SMEM_BYTES, s>>>(tm.q, tm.k, tm.r, tm.v16, static_cast<Tout *>(y), lse,
                                                             BH, T, causal, work_counter, ctl);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_sm100(const FwdTensorMaps &tm, bool with_rho, void *y, float *lse, int B, int H, int T,
                             int d, int causal, int out_dtype, int sm_count, int *work_counter, const DeviceCtl &ctl,
                             cudaStream_t s) {
    (void)d;
    const int BH = B * H;
    if (out_dtype == PARALLAX_F32) {
        if (with_rho) return launch_t<true, float>(tm, y, lse, BH, T, causal, sm_count, work_counter, ctl, s);
        return launch_t<false, float>(tm, y, lse, BH, T, causal, sm_count, work_counter, ctl, s);
    }
    if (with_rho) return launch_t<true, __nv_bfloat16>(tm, y, lse, BH, T, causal, sm_count, work_counter, ctl, s);
    return launch_t<false, __nv_bfloat16>(tm, y, lse, BH, T, causal, sm_count, work_counter, ctl, s);
}

}  // namespace plx
