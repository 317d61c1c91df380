// fwd_sm100.cu -- Parallax prefill/forward on the tensor cores (tcgen05 + TMA + TMEM).
//
// Operator (zubnet.ai news item on Parallax, paragraph 2): softmax attention
// minus the softmax-weighted KV covariance projected by the probe rho_i,
//   y_i = o_i - (m_i - o_i abar_i),  a_ij = k_j . rho_i.
// The pages' kernel keeps FlashAttention's KV streaming and reuses each K/V
// tile for both branches (encorp.ai blog "Integraciones de IA personalizadas
// tras la atencion Parallax", section "Como cambia Parallax la historia del
// hardware en GPU Hopper").  Here each 128-key tile is brought into shared
// memory once by TMA and feeds four UMMA chains per 128-row query tile:
//   S = Q K^T,  A = R K^T                       (bf16 x bf16 -> fp32, TMEM)
//   O += P V,   M' += (P o A') V                (fp16 x fp16 -> fp32, TMEM)
// with P = exp2(S log2e/sqrt(d) - m_ref) and A' = A / 256, both rounded to
// fp16 and written back into TMEM as the A operands of the P.V UMMAs.  fp16
// (not bf16) for these operands keeps the rounding of P o A inside the error
// budget; the row sums l = sum P and Abar' = sum P o A' are taken from the same
// rounded fp16 values the MMAs consume, so the result is exact for the rounded
// weights.  The running max is only moved when it rises by more than 8 in log2
// units (O and M are then rescaled in TMEM), so P <= 2^8 between moves, and the
// 1/256 on A keeps P o A' finite for |a| < 65504.
//
// V arrives as fp16 in blocks of 64 keys (one V stage), each scaled by its own
// power of two 2^-e (convert.cu chooses e from the block's largest |v|, so V
// keeps fp16 precision from about 1e-5 up to 2^23).  The stored P and P o A'
// of that stage are multiplied by 2^e (exact in fp16's range), so P.V is
// unchanged; the row sums are taken before that scaling.  Each softmax warp
// reads its block's exponent (one byte) at the start of the tile.  (Folding
// 2^e into the exponentials, or passing it through the V producer, put the
// exponent on a critical path: measured 7-12% slower.)
// An output that is still not finite (|v| >= 2^23, |a| >= 65504, non-finite
// inputs) records PARALLAX_ERR_DEVICE_RANGE in the device error word.
//
// Why this shape (measured on B200): a tcgen05.mma costs at least ~45-50
// cycles to issue, so UMMAs with N = 64 run at ~60% of the tensor rate while
// N >= 128 runs at full rate; and shared memory delivers ~128 B/cycle, which
// an SS UMMA with M = N = 128 already uses up.  The score UMMAs therefore
// cover 128 keys, and P, P o A' stay in TMEM so the P.V UMMAs read only V from
// shared memory.  Issuing is the other limit: the issuing thread shares its SM
// sub-partition with four softmax warps, and every barrier wait or commit it
// makes between UMMAs leaves the tensor pipe idle.  Two threads therefore
// issue: one the score UMMAs S(j), A(j), one the P.V UMMAs, so a wait of one
// chain never stalls the other.  TMEM holds two 128-column tile regions X0, X1
// and the accumulators O and M.  Key tile G uses X(G mod 2): S(G) lands there,
// then A(G) once the softmax has read S(G), and the softmax writes the fp16 P
// and P o A' over the S/A columns it has read; the region takes tile G + 2's S
// once the P.V UMMAs of tile G are done, so the next tile's S never waits for
// this tile's softmax.  While the four groups exchange their row maxima, each
// forms P with the current reference when its own scores do not move it (and
// rescales P if another group's do).
// (Measured and dropped: a 768-thread layout with a separate epilogue
// warpgroup; converting V inside the kernel; two softmax teams of 8 warps on
// alternate tiles; y through a shared-memory staging tile and TMA stores; the
// epilogue deferred past the next item's first tile.  Each slowed the softmax
// warps, which set the pace, or added register spills, more than it saved.)
//
// Roles (640 threads, one CTA per SM, persistent over (head, query tile)
// items taken longest-first from an atomic work counter):
//   warp 0 lane 0   scheduler + TMA for Q, R (per item) and K (128-key tiles)
//   warp 1          TMEM owner; lane 0 issues the score UMMAs S(j), A(j)
//   warps 2..17     four softmax warpgroups; group g takes key columns
//                   [32g, 32g+32) of every tile for all 128 rows, one row per
//                   thread; the four exchange their partial row max through
//                   shared memory and an mbarrier; then the item's epilogue
//   warp 18 lane 0  issues the P.V UMMAs
//   warp 19 lane 0  TMA for V (fp16, 64-key stages)
// Every wait is a bounded mbarrier wait (no named barriers), so a wait that
// gives up lets every role leave its loop and the kernel return.
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
#include "softmax_sm100.cuh"

namespace plx {
namespace {

constexpr int BM = 128;                   // query rows per tile
constexpr int BN = 128;                   // keys per tile
constexpr int NGRP = 4;                   // softmax warpgroups
constexpr int GCOLS = BN / NGRP;          // key columns per group
constexpr int KST = 2;                    // K ring stages (whole 128-key tiles)
constexpr int VKEYS = 64;                 // keys per V stage
constexpr int VST = 4;                    // V ring stages (two tiles ahead)
constexpr int VPER = BN / VKEYS;          // V stages per key tile
constexpr int SCHED = 4;                  // scheduler ring depth (items in flight)
constexpr int FIRST_SOFT_WARP = 2;
constexpr int NSOFT_WARPS = NGRP * 4;
constexpr int PV_WARP = FIRST_SOFT_WARP + NSOFT_WARPS;   // P.V UMMA issuer
constexpr int V_WARP = PV_WARP + 1;                       // V producer
constexpr int NTHREADS = (V_WARP + 1) * 32;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;
constexpr float RESCALE_THRESHOLD = 8.0f;   // log2 units
constexpr float A_SCALE = 1.0f / 256.0f;
constexpr float A_UNSCALE = 256.0f;
constexpr unsigned long long DRAIN_NS = 2000000ull;   // bound of the exit-time drain waits

// Shared-memory map for head dim D (every tile region 1024-byte aligned).
template <int D> struct Geo {
    static constexpr int HALVES = D / 64;                // 128-byte (64-element) column blocks of a row
    static constexpr int Q_BYTES = BM * D * 2;           // HALVES x [128 rows x 128 B]
    static constexpr int K_BYTES = BN * D * 2;           // HALVES x [128 keys x 128 B]
    static constexpr int V_BYTES = VKEYS * D * 2;        // fp16: HALVES x [64 keys x 128 B]
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_R = OFF_Q + Q_BYTES;
    static constexpr int OFF_K = OFF_R + Q_BYTES;
    static constexpr int OFF_V = OFF_K + KST * K_BYTES;
    static constexpr int OFF_BARS = OFF_V + VST * V_BYTES;
    static constexpr int OCOLS = D / NGRP;               // O/M columns each softmax group handles
    static_assert(OCOLS % 16 == 0, "16-column TMEM loads");
};

// TMEM column map: two tile regions X0, X1 and the accumulators O, M' (on
// 128-column boundaries for both head dims).  Key tile G of the CTA uses
// region X(G & 1): S(G) lands there, then A(G), and group g writes its fp16 P
// (16 columns) and P o A' (16 columns) over [32g, 32g + 32) of the region --
// the S and A columns it has already read -- where the P.V UMMAs read them.
constexpr uint32_t COL_X0 = 0, COL_O = 256, COL_M = 384;
__host__ __device__ constexpr uint32_t col_x(uint32_t G) { return COL_X0 + (G & 1) * BN; }
__host__ __device__ constexpr uint32_t col_p(uint32_t kk) { return (kk >> 1) * GCOLS + (kk & 1) * 8; }
constexpr uint32_t PA_SHIFT = GCOLS / 2;   // P o A' sits 16 columns after P

constexpr uint32_t IDESC_S = idesc_f16(1, 1, 0, 0, BM, BN);     // bf16 Q/R (K-major) x bf16 K (K-major)
template <int D> constexpr uint32_t idesc_pv() { return idesc_f16(0, 0, 0, 1, BM, D); }   // f16 P (TMEM) x f16 V (MN-major)

struct __align__(8) Bars {
    uint64_t qr_full, qr_empty;
    uint64_t r_tmem, r_smem;      // fused probe: R = X W_R in TMEM; R converted into shared memory
    uint64_t k_full[KST], k_empty[KST];
    uint64_t v_full[VST], v_empty[VST];
    uint64_t s_full, a_full;      // S, A UMMAs of the current tile done
    uint64_t s_free;              // softmax has loaded S out of TMEM
    uint64_t p_full[2];           // per region: P and P o A' of its tile are in TMEM
    uint64_t pv_done[2];          // per region: P.V UMMAs of its tile done
    uint64_t om_free;             // epilogue has read O and M
    uint64_t xchg[2];             // per tile parity: every softmax warp posted its partial max
    uint64_t esum;                // per item: partial sums posted
    uint64_t drain[2];            // last commit of each UMMA issuer (all its MMAs complete)
    uint64_t sched_full[SCHED], sched_empty[SCHED];
    int sched_item[SCHED];
    uint32_t tmem_base;
    int abort_flag;
    float red_max[2][NGRP][BM];   // [tile parity][group][row] partial row max
    float red_sum[2][NGRP][BM];   // [l or abar'][group][row] partial sums for the epilogue
};

template <int D> constexpr size_t smem_bytes() { return (size_t)Geo<D>::OFF_BARS + sizeof(Bars); }
static_assert(smem_bytes<128>() <= 232448, "shared memory budget");

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

template <int D, bool WITH_RHO, bool FUSED, typename Tout>
__global__ void __launch_bounds__(NTHREADS, 1)
    k_fwd(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
          const __grid_constant__ CUtensorMap tm_r, const __grid_constant__ CUtensorMap tm_v,
          const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w, Tout *__restrict__ y,
          float *__restrict__ lse, float *__restrict__ o_out, float *__restrict__ abar_out,
          const signed char *__restrict__ vexp_g, int BH, int H, int T, int d_model, int causal,
          int *__restrict__ work_counter, DeviceCtl ctl) {
    using Gm = Geo<D>;
    static_assert(!FUSED || (WITH_RHO && D == 128), "the fused probe needs the correction branch and d = 128");
    // fused probe: X W_R is accumulated over d_model in chunks of 64 that
    // stream through the K ring (X chunk [128 rows x 64], W_R chunk [64 x d])
    constexpr int XC_BYTES = BM * 64 * 2, WC_BYTES = 64 * D * 2;
    static_assert(!FUSED || XC_BYTES + WC_BYTES <= Gm::K_BYTES, "an X / W_R chunk fits a K stage");
    const int nchunk = FUSED ? d_model / 64 : 0;
    extern __shared__ __align__(1024) uint8_t smem[];
    // The swizzled tiles need a 1024-byte aligned base; there is no slack left
    // in the budget to realign, so refuse (recorded as a device error) if not.
    if (smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) atomicExch(ctl.err, PARALLAX_ERR_UNSUPPORTED);
        return;
    }
    Bars *bars = reinterpret_cast<Bars *>(smem + Gm::OFF_BARS);
    const uint32_t sbase = smem_u32(smem);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bars->qr_full), 1);
        mbar_init(smem_u32(&bars->qr_empty), 1);
        mbar_init(smem_u32(&bars->r_tmem), 1);
        mbar_init(smem_u32(&bars->r_smem), NSOFT_WARPS);
        for (int s = 0; s < KST; ++s) {
            mbar_init(smem_u32(&bars->k_full[s]), 1);
            mbar_init(smem_u32(&bars->k_empty[s]), 1);
        }
        for (int s = 0; s < VST; ++s) {
            mbar_init(smem_u32(&bars->v_full[s]), 1);
            mbar_init(smem_u32(&bars->v_empty[s]), 1);
        }
        mbar_init(smem_u32(&bars->s_full), 1);
        mbar_init(smem_u32(&bars->a_full), 1);
        mbar_init(smem_u32(&bars->s_free), NSOFT_WARPS);
        for (int x = 0; x < 2; ++x) {
            mbar_init(smem_u32(&bars->p_full[x]), NSOFT_WARPS);
            mbar_init(smem_u32(&bars->pv_done[x]), 1);
        }
        mbar_init(smem_u32(&bars->om_free), NSOFT_WARPS);
        mbar_init(smem_u32(&bars->xchg[0]), NSOFT_WARPS);
        mbar_init(smem_u32(&bars->xchg[1]), NSOFT_WARPS);
        mbar_init(smem_u32(&bars->esum), NSOFT_WARPS);
        mbar_init(smem_u32(&bars->drain[0]), 1);
        mbar_init(smem_u32(&bars->drain[1]), 1);
        for (int s = 0; s < SCHED; ++s) {
            mbar_init(smem_u32(&bars->sched_full[s]), 1);
            mbar_init(smem_u32(&bars->sched_empty[s]), 3 + NSOFT_WARPS);   // two UMMA threads, V producer, softmax warps
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
        // ===================================== scheduler + Q/R/K producer ==
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        if (WITH_RHO && !FUSED) tma_prefetch_desc(&tm_r);
        if (FUSED) {
            tma_prefetch_desc(&tm_x);
            tma_prefetch_desc(&tm_w);
        }
        uint32_t kc = 0;
        int k_armed[KST], qr_armed = -1;   // parity of each buffer's last fill still to land, -1 if none
        for (int s = 0; s < KST; ++s) k_armed[s] = -1;
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
            qr_armed = (int)(ic & 1);
            mbar_arrive_expect_tx(qf, (WITH_RHO && !FUSED) ? 2 * Gm::Q_BYTES : Gm::Q_BYTES);
#pragma unroll
            for (int h = 0; h < Gm::HALVES; ++h) {
                tma_load_3d(sbase + Gm::OFF_Q + h * (Gm::Q_BYTES / Gm::HALVES), &tm_q, qf, h * 64, q0, it.bh);
                if (WITH_RHO && !FUSED)
                    tma_load_3d(sbase + Gm::OFF_R + h * (Gm::Q_BYTES / Gm::HALVES), &tm_r, qf, h * 64, q0, it.bh);
            }
            if constexpr (FUSED) {
                // X rows of this query tile (row b*T + t of x) and head h's
                // columns of W_R, 64 of d_model at a time, through the K ring
                const int xrow = (it.bh / H) * T + q0, wcol = (it.bh % H) * D;
                for (int c = 0; c < nchunk && ok; ++c, ++kc) {
                    const int s = kc % KST;
                    if (!mbar_wait(smem_u32(&bars->k_empty[s]), ((kc / KST) & 1) ^ 1, wc)) { ok = false; break; }
                    const uint32_t f = smem_u32(&bars->k_full[s]);
                    const uint32_t dst = sbase + Gm::OFF_K + s * Gm::K_BYTES;
                    if ((ctl.debug_flags & DEBUG_FWD_SKIP_FIRST_K_LOAD) && kc == 0) continue;
                    k_armed[s] = (int)((kc / KST) & 1);
                    mbar_arrive_expect_tx(f, XC_BYTES + WC_BYTES);
                    tma_load_2d(dst, &tm_x, f, c * 64, xrow);
#pragma unroll
                    for (int h = 0; h < Gm::HALVES; ++h)
                        tma_load_2d(dst + XC_BYTES + h * (64 * 64 * 2), &tm_w, f, wcol + h * 64, c * 64);
                }
                if (!ok) break;
            }
            for (int j = 0; j < it.nkv; ++j, ++kc) {
                const int s = kc % KST;
                if (!mbar_wait(smem_u32(&bars->k_empty[s]), ((kc / KST) & 1) ^ 1, wc)) { ok = false; break; }
                const uint32_t f = smem_u32(&bars->k_full[s]);
                const uint32_t dst = sbase + Gm::OFF_K + s * Gm::K_BYTES;
                const bool skip = (ctl.debug_flags & DEBUG_FWD_SKIP_FIRST_K_LOAD) && kc == 0;
                if (!skip) {
                    k_armed[s] = (int)((kc / KST) & 1);
                    mbar_arrive_expect_tx(f, Gm::K_BYTES);
#pragma unroll
                    for (int h = 0; h < Gm::HALVES; ++h)
                        tma_load_3d(dst + h * (Gm::K_BYTES / Gm::HALVES), &tm_k, f, h * 64, j * BN, it.bh);
                }
            }
        }
        // no copy of this thread may still be landing when the CTA exits
        if (qr_armed >= 0) mbar_wait_drain(smem_u32(&bars->qr_full), (uint32_t)qr_armed, DRAIN_NS);
        for (int s = 0; s < KST; ++s)
            if (k_armed[s] >= 0) mbar_wait_drain(smem_u32(&bars->k_full[s]), (uint32_t)k_armed[s], DRAIN_NS);
    } else if (warp == V_WARP && lane == 0) {
        // ==================================================== V producer ==
        tma_prefetch_desc(&tm_v);
        uint32_t vc = 0;
        int v_armed[VST];
        for (int s = 0; s < VST; ++s) v_armed[s] = -1;
        bool ok = true;
        for (uint32_t ic = 0; ok; ++ic) {
            int w;
            if (!next_item<SCHED>(bars, ic, w, wc)) break;
            mbar_arrive(smem_u32(&bars->sched_empty[ic % SCHED]));
            if (w >= items) break;
            const Item it = item_of(w, BH, nq, T, causal);
            for (int j = 0; j < it.nkv && ok; ++j) {
                for (int vs = 0; vs < VPER; ++vs, ++vc) {
                    const int s = vc % VST;
                    if (!mbar_wait(smem_u32(&bars->v_empty[s]), ((vc / VST) & 1) ^ 1, wc)) { ok = false; break; }
                    const uint32_t f = smem_u32(&bars->v_full[s]);
                    v_armed[s] = (int)((vc / VST) & 1);
                    const uint32_t dst = sbase + Gm::OFF_V + s * Gm::V_BYTES;
                    mbar_arrive_expect_tx(f, Gm::V_BYTES);
#pragma unroll
                    for (int h = 0; h < Gm::HALVES; ++h)
                        tma_load_3d(dst + h * (Gm::V_BYTES / Gm::HALVES), &tm_v, f, h * 64, j * BN + vs * VKEYS,
                                    it.bh);
                }
            }
        }
        for (int s = 0; s < VST; ++s)
            if (v_armed[s] >= 0) mbar_wait_drain(smem_u32(&bars->v_full[s]), (uint32_t)v_armed[s], DRAIN_NS);
    } else if (warp == 1 && lane == 0) {
        // ============================================= score UMMA issuer ==
        // Key tile G: S(G) into region X(G & 1) once the P.V UMMAs of tile
        // G - 2 (the region's previous tile) are done, then A(G) there once the
        // softmax has loaded S(G).  The shared-memory descriptors are built once; each
        // UMMA adds a compile-time offset, keeping this thread's instruction
        // stream short.
        uint32_t kc = 0, G = 0;
        bool ok = true;
        const uint64_t dq = sdesc_sw128(sbase + Gm::OFF_Q, 16, 1024);
        const uint64_t dr = sdesc_sw128(sbase + Gm::OFF_R, 16, 1024);
        const uint64_t dk = sdesc_sw128(sbase + Gm::OFF_K, 16, 1024);   // stage s: + s * K_BYTES / 16
        // fused probe: R[128 x d] += X chunk (K-major) x W_R chunk (MN-major) into a tile region
        constexpr uint32_t IDESC_R = idesc_f16(1, 1, 0, 1, BM, D);
        auto issue_probe_chunk = [&](uint32_t dcol, uint32_t stage_addr, bool first) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t adesc = sdesc_sw128(stage_addr + kk * 32, 16, 1024);
                const uint64_t bdesc = sdesc_sw128(stage_addr + XC_BYTES + kk * 16 * 128, 64 * 128, 1024);
                umma_ss(tmem + dcol, adesc, bdesc, IDESC_R, (first && kk == 0) ? 0u : 1u);
            }
        };
        auto issue_scores = [&](uint32_t dcol, uint64_t da, uint64_t kd) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = ((uint32_t)(kk >> 2) * (Gm::Q_BYTES / Gm::HALVES) + (uint32_t)(kk & 3) * 32) >> 4;
                const uint32_t koff =
                    ((uint32_t)(kk >> 2) * (Gm::K_BYTES / Gm::HALVES) + (uint32_t)(kk & 3) * 32) >> 4;
                umma_ss(tmem + dcol, da + off, kd + koff, IDESC_S, kk > 0 ? 1u : 0u);
            }
        };
        for (uint32_t ic = 0; ok; ++ic) {
            int w;
            if (!next_item<SCHED>(bars, ic, w, wc)) break;
            mbar_arrive(smem_u32(&bars->sched_empty[ic % SCHED]));
            if (w >= items) break;
            const Item it = item_of(w, BH, nq, T, causal);
            if (!mbar_wait(smem_u32(&bars->qr_full), ic & 1, wc)) break;
            if constexpr (FUSED) {
                // R of this item into region X(G + 1) (that of the item's second
                // tile) once the last P.V UMMAs of the previous item are done with
                // it (this overlaps that item's epilogue, which reads O and M);
                // S(G + 1) lands there only after A(G), which waits for the
                // softmax to have moved R into shared memory
                if (G > 0 && !mbar_wait(smem_u32(&bars->pv_done[(G - 1) & 1]), ((G - 1) >> 1) & 1, wc)) break;
                for (int c = 0; c < nchunk; ++c, ++kc) {
                    const int s = kc % KST;
                    if (!mbar_wait(smem_u32(&bars->k_full[s]), (kc / KST) & 1, wc)) { ok = false; break; }
                    tc_fence_after();
                    issue_probe_chunk(col_x(G + 1), sbase + Gm::OFF_K + s * Gm::K_BYTES, c == 0);
                    tc_commit(smem_u32(&bars->k_empty[s]));
                }
                if (!ok) break;
                tc_commit(smem_u32(&bars->r_tmem));
            }
            for (int j = 0; j < it.nkv; ++j, ++G, ++kc) {
                const int s = kc % KST;
                if (!mbar_wait(smem_u32(&bars->k_full[s]), (kc / KST) & 1, wc)) { ok = false; break; }
                // the region's previous tile has been consumed by its P.V UMMAs
                if (G >= 2 && !mbar_wait(smem_u32(&bars->pv_done[G & 1]), ((G - 2) >> 1) & 1, wc)) {
                    ok = false;
                    break;
                }
                // without the A UMMAs, nothing else orders S(G) after the
                // softmax's load of S(G - 1), which keeps s_full one phase ahead
                if (!WITH_RHO && G > 0 && !mbar_wait(smem_u32(&bars->s_free), (G - 1) & 1, wc)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t kd = dk + (uint64_t)(s * (Gm::K_BYTES >> 4));
                issue_scores(col_x(G), dq, kd);
                tc_commit(smem_u32(&bars->s_full));
                if constexpr (WITH_RHO) {
                    // fused probe: the softmax warps have put R into shared memory
                    if (FUSED && j == 0 && !mbar_wait(smem_u32(&bars->r_smem), ic & 1, wc)) { ok = false; break; }
                    if (!mbar_wait(smem_u32(&bars->s_free), G & 1, wc)) { ok = false; break; }
                    tc_fence_after();
                    issue_scores(col_x(G), dr, kd);
                    tc_commit(smem_u32(&bars->a_full));
                }
                tc_commit(smem_u32(&bars->k_empty[s]));
                if (j == it.nkv - 1) tc_commit(smem_u32(&bars->qr_empty));
            }
        }
        // every MMA this thread issued has completed before TMEM is released
        tc_commit(smem_u32(&bars->drain[0]));
        mbar_wait_drain(smem_u32(&bars->drain[0]), 0, DRAIN_NS);
    } else if (warp == PV_WARP && lane == 0) {
        // ============================================== P.V UMMA issuer ==
        uint32_t vc = 0, G = 0;
        bool ok = true;
        constexpr uint32_t IDESC_PV = idesc_pv<D>();
        const uint64_t dv = sdesc_sw128(sbase + Gm::OFF_V, Gm::V_BYTES / Gm::HALVES, 1024);   // + s * V_BYTES / 16
        for (uint32_t ic = 0; ok; ++ic) {
            int w;
            if (!next_item<SCHED>(bars, ic, w, wc)) break;
            mbar_arrive(smem_u32(&bars->sched_empty[ic % SCHED]));
            if (w >= items) break;
            const Item it = item_of(w, BH, nq, T, causal);
            for (int j = 0; j < it.nkv && ok; ++j, ++G) {
                if (!mbar_wait(smem_u32(&bars->p_full[G & 1]), (G >> 1) & 1, wc)) { ok = false; break; }
                // the first tile overwrites O and M': the epilogue of the
                // previous item must have read them
                if (j == 0 && ic > 0 && !mbar_wait(smem_u32(&bars->om_free), (ic - 1) & 1, wc)) {
                    ok = false;
                    break;
                }
                for (int vs = 0; vs < VPER; ++vs, ++vc) {
                    const int s = vc % VST;
                    if (!mbar_wait(smem_u32(&bars->v_full[s]), (vc / VST) & 1, wc)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t vd = dv + (uint64_t)(s * (Gm::V_BYTES >> 4));
#pragma unroll
                    for (int k2 = 0; k2 < VKEYS / 16; ++k2) {
                        const int kk = vs * (VKEYS / 16) + k2;     // 16-key step within the tile
                        const uint64_t vdesc = vd + (uint64_t)((k2 * 16 * 128) >> 4);
                        const uint32_t acc = (j == 0 && kk == 0) ? 0u : 1u;
                        const uint32_t pc = tmem + col_x(G) + col_p(kk);
                        umma_ts(tmem + COL_O, pc, vdesc, IDESC_PV, acc);
                        if constexpr (WITH_RHO) umma_ts(tmem + COL_M, pc + PA_SHIFT, vdesc, IDESC_PV, acc);
                    }
                    tc_commit(smem_u32(&bars->v_empty[s]));
                }
                if (ok) tc_commit(smem_u32(&bars->pv_done[G & 1]));
            }
        }
        tc_commit(smem_u32(&bars->drain[1]));
        mbar_wait_drain(smem_u32(&bars->drain[1]), 0, DRAIN_NS);
    } else if (warp >= FIRST_SOFT_WARP && warp < PV_WARP) {
        // ============================================ softmax + epilogue ==
        const int grp = (warp - FIRST_SOFT_WARP) >> 2;   // key columns [32 grp, 32 grp + 32)
        const int quarter = warp & 3;                    // TMEM lane quarter this warp may access
        const int r = quarter * 32 + lane;               // query row within the tile == TMEM lane
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const float scale_log2 = LOG2E / sqrtf((float)D);
        // 32-byte output stores (half the store instructions of 16-byte ones)
        // when the output rows are 32-byte aligned; the same for every thread
        const bool wide = ((reinterpret_cast<uintptr_t>(y) | reinterpret_cast<uintptr_t>(o_out)) & 31) == 0;
        const int vsg = (grp * GCOLS) / VKEYS;           // the V block (within a tile) of this group's keys
        const int nblk = (T + VKEYS - 1) / VKEYS;        // 64-key V blocks per head, one exponent each
        uint32_t G = 0, ni = 0;   // key tiles and items processed by this CTA
        bool ok = true;
        for (uint32_t ic = 0; ok; ++ic) {
            int w = 0;
            const bool got = next_item<SCHED>(bars, ic, w, wc);
            if (!__all_sync(0xffffffffu, got)) break;
            if (lane == 0) mbar_arrive(smem_u32(&bars->sched_empty[ic % SCHED]));
            if (w >= items) break;
            const Item it = item_of(w, BH, nq, T, causal);
            const int qrow = it.qt * BM + r;
            const int kvis = causal ? min(T, qrow + 1) : T;  // keys visible to this row
            float m_ref = -INFINITY, l = 0.f, ab = 0.f;
            if constexpr (FUSED) {
                // ---- the probe tile R = X W_R of this item: TMEM (region
                // X(G + 1)) -> bf16 -> shared memory, in the swizzled K-major
                // layout a TMA load of rho would give, for the A UMMAs.  Group g
                // converts columns [32g, 32g + 32) of its rows. ----
                if (!warp_wait(smem_u32(&bars->r_tmem), ic & 1, wc)) { ok = false; break; }
                tc_fence_after();
                uint32_t rr[GCOLS];
                const uint32_t rcol = tmem + lane_off + col_x(G + 1) + grp * GCOLS;
                tmem_ld16(rcol, *reinterpret_cast<uint32_t(*)[16]>(&rr[0]));
                tmem_ld16(rcol + 16, *reinterpret_cast<uint32_t(*)[16]>(&rr[16]));
                tmem_wait_ld();
                uint8_t *rrow = smem + Gm::OFF_R + ((grp * GCOLS) / 64) * (Gm::Q_BYTES / Gm::HALVES) + r * 128;
#pragma unroll
                for (int c = 0; c < GCOLS / 8; ++c) {
                    const int c16 = ((grp * GCOLS) % 64) / 8 + c;   // 16-byte chunk within the 128-byte row
                    uint32_t pb[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(rr[8 * c + 2 * i]),
                                                                       __uint_as_float(rr[8 * c + 2 * i + 1]));
                        pb[i] = *reinterpret_cast<const uint32_t *>(&h);
                    }
                    *reinterpret_cast<uint4 *>(rrow + ((c16 ^ (r & 7)) << 4)) = make_uint4(pb[0], pb[1], pb[2], pb[3]);
                }
                fence_proxy_async_smem();   // read by the A UMMAs (async proxy)
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&bars->r_smem));
            }
            for (int j = 0; j < it.nkv; ++j, ++G) {
                // the exponent of this group's V block, needed only when P is stored
                const int vblk = j * VPER + vsg;   // past the last block the keys read as zero
                const int e = vblk < nblk ? (int)__ldg(vexp_g + (size_t)it.bh * nblk + vblk) : 0;
                // ---- scores of this group's 32 keys, then release S ----
                if (!warp_wait(smem_u32(&bars->s_full), G & 1, wc)) { ok = false; break; }
                tc_fence_after();
                const uint32_t xcol = tmem + lane_off + col_x(G) + grp * GCOLS;   // this group's columns of the tile's region
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
                // ---- row max across the four groups ----
                bars->red_max[G & 1][grp][r] = mx;
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&bars->xchg[G & 1]));
                float alpha = 1.f;
                bool moved = false;
                uint32_t pk[GCOLS / 2];
                // ---- P = exp2(z log2e - m_ref) as fp16.  While the other groups'
                // maxima arrive, P is formed with the current reference when no
                // score of this warp's own keys needs it moved (after an item's
                // first tile, nearly always); if another group's keys move it, the
                // fp16 P is scaled to the new reference (weights below 2^8, so no
                // overflow).  Otherwise P waits for the row max as usual. ----
                const bool spec =
                    __all_sync(0xffffffffu, m_ref != -INFINITY && mx * scale_log2 <= m_ref + RESCALE_THRESHOLD);
                if (spec) {
                    weights_f16(sr, pk, scale_log2, -m_ref);
                    if (!warp_wait(smem_u32(&bars->xchg[G & 1]), (G >> 1) & 1, wc)) { ok = false; break; }
                    mx = fmaxf(fmaxf(bars->red_max[G & 1][0][r], bars->red_max[G & 1][1][r]),
                               fmaxf(bars->red_max[G & 1][2][r], bars->red_max[G & 1][3][r])) *
                         scale_log2;
                    if (mx > m_ref + RESCALE_THRESHOLD) {
                        alpha = ex2(m_ref - mx);
                        m_ref = mx;
                        l *= alpha;
                        ab *= alpha;
                        moved = true;
                        const __half2 f2 = __float2half2_rn(alpha);
                        const uint32_t fh = *reinterpret_cast<const uint32_t *>(&f2);
#pragma unroll
                        for (int i = 0; i < GCOLS / 2; ++i) pk[i] = hmul2(pk[i], fh);
                    }
                } else {
                    if (!warp_wait(smem_u32(&bars->xchg[G & 1]), (G >> 1) & 1, wc)) { ok = false; break; }
                    mx = fmaxf(fmaxf(bars->red_max[G & 1][0][r], bars->red_max[G & 1][1][r]),
                               fmaxf(bars->red_max[G & 1][2][r], bars->red_max[G & 1][3][r])) *
                         scale_log2;
                    if (mx > m_ref + RESCALE_THRESHOLD) {
                        alpha = ex2(m_ref - mx);     // 0 when m_ref = -inf
                        m_ref = mx;
                        l *= alpha;
                        ab *= alpha;
                        moved = true;
                    }
                    weights_f16(sr, pk, scale_log2, -m_ref);
                }
                // ---- row sums from the rounded weights the MMAs read ----
                {
                    float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int i = 0; i < GCOLS / 2; ++i) l4[i & 3] = add_f16x2_to_f32(l4[i & 3], pk[i]);
                    l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
                }
                uint32_t pak[WITH_RHO ? GCOLS / 2 : 1];
                if constexpr (WITH_RHO) {
                    // ---- A of this group's 32 keys (its P goes over them) ----
                    if (!warp_wait(smem_u32(&bars->a_full), G & 1, wc)) { ok = false; break; }
                    tc_fence_after();
                    uint32_t ar[GCOLS];
                    tmem_ld16(xcol, *reinterpret_cast<uint32_t(*)[16]>(&ar[0]));
                    tmem_ld16(xcol + 16, *reinterpret_cast<uint32_t(*)[16]>(&ar[16]));
                    tmem_wait_ld();
                    float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int i = 0; i < GCOLS / 2; ++i) {
                        float a0, a1;
                        ffma2(a0, a1, __uint_as_float(ar[2 * i]), __uint_as_float(ar[2 * i + 1]), A_SCALE, 0.f);
                        pak[i] = hmul2(pk[i], pack_f16x2(a0, a1));
                        a4[i & 3] = add_f16x2_to_f32(a4[i & 3], pak[i]);
                    }
                    ab += (a4[0] + a4[1]) + (a4[2] + a4[3]);
                }
                // ---- V of this block holds v 2^-e: P and P o A' are stored as
                // 2^e P and 2^e P o A', so the P.V products are unchanged (a
                // power-of-two multiply is exact in fp16's range; e = 0 for
                // ordinary magnitudes, and the branch is uniform in the warp) ----
                {
                    if (e != 0) {
                        const __half2 two_e = __float2half2_rn(__int_as_float((127 + e) << 23));
                        const uint32_t h2 = *reinterpret_cast<const uint32_t *>(&two_e);
#pragma unroll
                        for (int i = 0; i < GCOLS / 2; ++i) {
                            pk[i] = hmul2(pk[i], h2);
                            if constexpr (WITH_RHO) pak[i] = hmul2(pak[i], h2);
                        }
                    }
                }
                // a moved reference max rescales O and M' (each group d/4 columns)
                // once the previous tile's P.V UMMAs are done: O and M' then hold
                // every earlier tile of this item, and this tile's are not issued
                if (__any_sync(0xffffffffu, moved && j > 0)) {
                    if (!warp_wait(smem_u32(&bars->pv_done[(G - 1) & 1]), ((G - 1) >> 1) & 1, wc)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const float f = (moved && j > 0) ? alpha : 1.f;
#pragma unroll 1
                    for (int c = grp * Gm::OCOLS; c < grp * Gm::OCOLS + Gm::OCOLS; c += 16) {
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
                // ---- P and P o A' over this group's S and A columns, for the P.V UMMAs ----
                tmem_st16(xcol, pk);
                if constexpr (WITH_RHO) tmem_st16(xcol + PA_SHIFT, pak);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&bars->p_full[G & 1]));
            }
            if (!ok) break;
            // ---------------------------------------------- epilogue --
            bars->red_sum[0][grp][r] = l;
            bars->red_sum[1][grp][r] = ab;
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bars->esum));
            if (!warp_wait(smem_u32(&bars->esum), ni & 1, wc)) break;
            ++ni;
            const float lt = (bars->red_sum[0][0][r] + bars->red_sum[0][1][r]) +
                             (bars->red_sum[0][2][r] + bars->red_sum[0][3][r]);
            const float abt = (bars->red_sum[1][0][r] + bars->red_sum[1][1][r]) +
                              (bars->red_sum[1][2][r] + bars->red_sum[1][3][r]);
            // the last P.V UMMAs of this item are done: O and M' are final
            if (!warp_wait(smem_u32(&bars->pv_done[(G - 1) & 1]), ((G - 1) >> 1) & 1, wc)) break;
            tc_fence_after();
            const float inv_l = 1.0f / lt;
            const float abar = abt * inv_l;
            const bool store = qrow < T;
            Tout *yrow = y + ((size_t)it.bh * T + (store ? qrow : 0)) * D;
            bool finite = true;
#pragma unroll 1
            for (int c = grp * Gm::OCOLS; c < grp * Gm::OCOLS + Gm::OCOLS; c += 16) {
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
                    finite = finite && isfinite(out[i]);
                }
                if (store && o_out != nullptr) {   // training forward: o = O / l for the backward
                    float *dst = o_out + ((size_t)it.bh * T + qrow) * D + c;
                    if (wide) {
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            uint32_t w8[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i) w8[i] = __float_as_uint(__uint_as_float(o[8 * h + i]) * inv_l);
                            st_global_v8(dst + 8 * h, w8);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            reinterpret_cast<float4 *>(dst)[i] =
                                make_float4(__uint_as_float(o[4 * i]) * inv_l, __uint_as_float(o[4 * i + 1]) * inv_l,
                                            __uint_as_float(o[4 * i + 2]) * inv_l, __uint_as_float(o[4 * i + 3]) * inv_l);
                    }
                }
                if (store) {
                    if constexpr (sizeof(Tout) == 4) {
                        if (wide) {
#pragma unroll
                            for (int h = 0; h < 2; ++h)
                                st_global_v8(yrow + c + 8 * h, *reinterpret_cast<const uint32_t(*)[8]>(&out[8 * h]));
                        } else {
                            float4 *dst = reinterpret_cast<float4 *>(yrow + c);
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                dst[i] = make_float4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]);
                        }
                    } else {
                        uint32_t pb[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            __nv_bfloat162 h = __floats2bfloat162_rn(out[2 * i], out[2 * i + 1]);
                            pb[i] = *reinterpret_cast<uint32_t *>(&h);
                        }
                        if (wide) {
                            st_global_v8(yrow + c, pb);
                        } else {
                            uint4 *dst = reinterpret_cast<uint4 *>(yrow + c);
                            dst[0] = make_uint4(pb[0], pb[1], pb[2], pb[3]);
                            dst[1] = make_uint4(pb[4], pb[5], pb[6], pb[7]);
                        }
                    }
                }
            }
            if (store && grp == 0 && lse != nullptr) lse[(size_t)it.bh * T + qrow] = (m_ref + log2f(lt)) * LN2;
            if (store && grp == 0 && abar_out != nullptr) abar_out[(size_t)it.bh * T + qrow] = abar * A_UNSCALE;
            // an output that is not finite: an input outside the kernel's range
            if (__any_sync(0xffffffffu, store && !finite) && lane == 0) atomicCAS(ctl.err, 0, PARALLAX_ERR_DEVICE_RANGE);
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

template <int D, bool WITH_RHO, bool FUSED, typename Tout>
cudaError_t launch_t(const FwdTensorMaps &tm, void *y, float *lse, float *o_out, float *abar_out,
                     const signed char *vexp, int BH, int H, int T, int d_model, int causal, int sm_count,
                     int *work_counter, const DeviceCtl &ctl, cudaStream_t s) {
    static std::atomic<unsigned long long> limit_set{0};
    auto kern = k_fwd<D, WITH_RHO, FUSED, Tout>;
    if (cudaError_t e = ensure_smem_limit(kern, (int)smem_bytes<D>(), limit_set)) return e;
    const int items = ((T + BM - 1) / BM) * BH;
    const int grid = items < sm_count ? items : sm_count;
    cudaError_t e = cudaMemsetAsync(work_counter, 0, sizeof(int), s);
    if (e != cudaSuccess) return e;
    kern<<<grid, NTHREADS, smem_bytes<D>(), s>>>(tm.q, tm.k, tm.r, tm.v, tm.x, tm.w, static_cast<Tout *>(y), lse,
                                                 o_out, abar_out, vexp, BH, H, T, d_model, causal, work_counter, ctl);
    return cudaGetLastError();
}

template <int D, bool FUSED>
cudaError_t launch_d(const FwdTensorMaps &tm, bool with_rho, void *y, float *lse, float *o_out, float *abar_out,
                     const signed char *vexp, int BH, int H, int T, int d_model, int causal, int out_dtype,
                     int sm_count, int *work_counter, const DeviceCtl &ctl, cudaStream_t s) {
    if constexpr (FUSED) {
        if (out_dtype == PARALLAX_F32)
            return launch_t<D, true, true, float>(tm, y, lse, o_out, abar_out, vexp, BH, H, T, d_model, causal, sm_count, work_counter,
                                                  ctl, s);
        return launch_t<D, true, true, __nv_bfloat16>(tm, y, lse, o_out, abar_out, vexp, BH, H, T, d_model, causal, sm_count,
                                                      work_counter, ctl, s);
    } else {
        if (out_dtype == PARALLAX_F32) {
            if (with_rho)
                return launch_t<D, true, false, float>(tm, y, lse, o_out, abar_out, vexp, BH, H, T, 0, causal, sm_count, work_counter,
                                                       ctl, s);
            return launch_t<D, false, false, float>(tm, y, lse, o_out, abar_out, vexp, BH, H, T, 0, causal, sm_count, work_counter,
                                                    ctl, s);
        }
        if (with_rho)
            return launch_t<D, true, false, __nv_bfloat16>(tm, y, lse, o_out, abar_out, vexp, BH, H, T, 0, causal, sm_count,
                                                           work_counter, ctl, s);
        return launch_t<D, false, false, __nv_bfloat16>(tm, y, lse, o_out, abar_out, vexp, BH, H, T, 0, causal, sm_count, work_counter,
                                                        ctl, s);
    }
}

}  // namespace

cudaError_t launch_fwd_sm100(const FwdTensorMaps &tm, bool with_rho, void *y, float *lse, float *o_out,
                             float *abar_out, const signed char *vexp, int B, int H, int T, int d, int causal,
                             int out_dtype, int sm_count, int *work_counter, const DeviceCtl &ctl, cudaStream_t s) {
    const int BH = B * H;
    if (d == 64)
        return launch_d<64, false>(tm, with_rho, y, lse, o_out, abar_out, vexp, BH, H, T, 0, causal, out_dtype,
                                   sm_count, work_counter, ctl, s);
    return launch_d<128, false>(tm, with_rho, y, lse, o_out, abar_out, vexp, BH, H, T, 0, causal, out_dtype, sm_count,
                                work_counter, ctl, s);
}

cudaError_t launch_fwd_fused_sm100(const FwdTensorMaps &tm, void *y, float *lse, const signed char *vexp, int B,
                                   int H, int T, int d_model, int causal, int out_dtype, int sm_count,
                                   int *work_counter, const DeviceCtl &ctl, cudaStream_t s) {
    return launch_d<128, true>(tm, true, y, lse, nullptr, nullptr, vexp, B * H, H, T, d_model, causal, out_dtype,
                               sm_count, work_counter, ctl, s);
}

}  // namespace plx
