// decode_gqa.cu -- the paged decode (any number of query heads per KV head) on
// the tensor cores.
//
// When G = Hq / Hkv query heads share one key/value head, every K row meets
// 2G probe vectors (G queries q_g and G probes rho_g; zubnet.ai news item on
// Parallax, paragraph 2: one KV stream feeds both branches) and every V row
// meets 2G weights (p and p a per head).  Done per head on the CUDA cores
// that is G times the unpack/FMA/shuffle work of one head per byte loaded;
// here the 2G vectors are the rows of a 16-row tensor-core operand, so one
// K or V load serves all of them:
//   [Q; R] (16 x d)  x  K^T (d x 16 tokens)  -> z and a of every head     (bf16 MMA)
//   [P; P o A] (16 x 16 tokens)  x  V (16 tokens x d)  -> O and M of every head   (fp16 MMA)
// Rows 0..7 carry q (then p), rows 8..15 carry rho (then p a) of up to eight
// heads, so the score MMA's accumulator is already laid out as the P.V
// MMA's A operand (no data movement between the two).  The weights are
// rounded to fp16 (bf16 would put the rounding of p a outside the error
// budget for large |a|) and V is converted to fp16 as its fragments are read.
//
// With one query head per KV head the operand is mostly zero rows, but the
// per-warp cp.async ring still hides the page indirection better than the
// per-head CUDA-core decode did (B=64 ctx 4096: 0.92 against 0.68 of HBM).
//
// A CTA of 4 warps takes one (sequence, KV head, up to 8 query heads, chunk)
// unit; each warp streams its own 16-token tiles of the chunk through a
// 2-stage cp.async ring in shared memory (128-byte-row swizzle, read back with
// ldmatrix) and keeps its own online-softmax state; the four states are
// merged at the end and written as the same partials (or y) as the split
// kernel, so the split combine applies unchanged.
//
// A 16-token tile starts on a multiple of 16 tokens and a page holds at least
// 16, so the tile's rows share one page: its block-table entry is read once,
// one iteration before the tile is copied, and that load overlaps the current
// tile's arithmetic (read per row and chunk, just before the copies, it held
// every copy back by a dependent global load: 0.85 of HBM at B=64 Hq=32 Hkv=8
// ctx 4096 against 0.92 now, and 0.83 against 0.98 at B=256 with 16-token pages).
//
// Occupancy over depth (measured, B=64 Hq=32 Hkv=8 ctx 4096, before the page
// read moved ahead): a 3-stage ring at 2 CTAs per SM (210 registers, 96 KB
// each) streamed 0.73 of HBM; a 2-stage ring at 3 CTAs per SM (registers
// capped at 170, no spills) 0.84, and 0.92 with one query head per KV head; 4
// CTAs per SM (128 registers) spilled and fell to 0.69.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include "internal.h"

namespace plx {
namespace {

constexpr int WARPS = 4;
constexpr int TILE = 16;      // tokens per warp step
constexpr int STAGES = 2;    // tiles in flight per warp: STAGES - 1
constexpr int MIN_CTAS = 3;  // resident CTAs per SM (registers capped at 170, 64 KB of ring each)
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

__device__ __forceinline__ float fex2(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte global -> shared copy; src_bytes = 0 writes zeros and reads nothing.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void cp_async_wait_0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_f16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// (lo, hi) fp32 -> packed fp16x2 (lo in the low half)
__device__ __forceinline__ uint32_t f16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
// packed bf16x2 -> packed fp16x2
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t u) {
    return f16x2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}
__device__ __forceinline__ float f16_lo(uint32_t u) { return __half2float(__ushort_as_half((unsigned short)(u & 0xFFFF))); }
__device__ __forceinline__ float f16_hi(uint32_t u) { return __half2float(__ushort_as_half((unsigned short)(u >> 16))); }

template <typename Tout> __device__ __forceinline__ void store_y(Tout *p, float v);
template <> __device__ __forceinline__ void store_y<float>(float *p, float v) { *p = v; }
template <> __device__ __forceinline__ void store_y<__nv_bfloat16>(__nv_bfloat16 *p, float v) {
    *p = __float2bfloat16_rn(v);
}

// Byte offset of 16-byte chunk `c` of tile row `r` (rows of D bf16, chunks
// XOR-swizzled by the row so that ldmatrix's 8 rows hit 8 different banks).
template <int D> __device__ __forceinline__ uint32_t tile_off(int r, int c) {
    return (uint32_t)(r * D * 2 + ((c ^ (r & 7)) << 4));
}

template <int D> struct GqaSmem {
    static constexpr int STAGE_BYTES = 2 * TILE * D * 2;              // K tile + V tile
    static constexpr int RING_BYTES = WARPS * STAGES * STAGE_BYTES;
    static constexpr int MERGE_BYTES = WARPS * 8 * (2 * D + 3) * 4;    // per warp: 8 heads x (O, M, mu, l, abar)
    static constexpr int BYTES = RING_BYTES > MERGE_BYTES ? RING_BYTES : MERGE_BYTES;
};

template <int D, typename Tout>
__global__ void __launch_bounds__(WARPS * 32, MIN_CTAS) k_decode_gqa(
    const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ rho, const __nv_bfloat16 *__restrict__ kp,
    const __nv_bfloat16 *__restrict__ vp, const int *__restrict__ seqlens, Tout *__restrict__ y,
    float *__restrict__ lse, int Hq, int chunk, int nsplit, long units_per_split, int htiles, PagedKV pg,
    float *__restrict__ partials, int *__restrict__ err) {
    extern __shared__ __align__(128) uint8_t smem[];
    constexpr int NCH = D / 8;                 // 16-byte chunks per row
    constexpr int KS = D / 16;                 // 16-wide d slices
    constexpr int NT = D / 8;                  // 8-wide output column tiles
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int r = lane / 4, t4 = lane % 4;     // fragment row (head) and column pair
    const float scale_log2 = LOG2E / sqrtf((float)D);
    const int pmask = (1 << pg.pshift) - 1;
    const long units = units_per_split * nsplit;

    for (long u = blockIdx.x; u < units; u += gridDim.x) {
        const long ut = u % units_per_split;    // chunk-major
        const int split = (int)(u / units_per_split);
        const int b = (int)(ut / ((long)pg.Hkv * htiles));
        const int rem = (int)(ut % ((long)pg.Hkv * htiles));
        const int kvh = rem / htiles, ht = rem % htiles;
        const int g0 = ht * 8;                                   // first head of this tile within the group
        const int nh = min(8, pg.group - g0);                    // heads in this tile
        const long h0 = (long)b * Hq + (long)kvh * pg.group + g0;   // flat (b, h) of the tile's first head
        const int L = min(max(seqlens[b], 0), pg.max_pages << pg.pshift);
        const int t0 = split * chunk;
        if (t0 >= L && nsplit > 1) continue;
        const int t1 = min(L, t0 + chunk);
        const int ntiles = (t1 - t0 + TILE - 1) / TILE;

        // ---- [Q; R] fragments (rows r: q of head r, rows r + 8: rho of head r) ----
        uint32_t qa[KS][4];
        {
            const bool live = r < nh;
            const uint32_t *qrow = reinterpret_cast<const uint32_t *>(q + (h0 + (live ? r : 0)) * D);
            const uint32_t *rrow = reinterpret_cast<const uint32_t *>(rho + (h0 + (live ? r : 0)) * D);
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                qa[ks][0] = live ? __ldg(qrow + ks * 8 + t4) : 0u;
                qa[ks][1] = live ? __ldg(rrow + ks * 8 + t4) : 0u;
                qa[ks][2] = live ? __ldg(qrow + ks * 8 + 4 + t4) : 0u;
                qa[ks][3] = live ? __ldg(rrow + ks * 8 + 4 + t4) : 0u;
            }
        }
        float oacc[NT][4];
#pragma unroll
        for (int j = 0; j < NT; ++j) oacc[j][0] = oacc[j][1] = oacc[j][2] = oacc[j][3] = 0.f;
        float m_run = -INFINITY, l_run = 0.f, ab_run = 0.f;

        uint8_t *ring = smem + warp * STAGES * GqaSmem<D>::STAGE_BYTES;
        // page of tile i: its 16 tokens start on a multiple of 16 and pages hold
        // at least 16 tokens, so they share one page; i < ntiles keeps the
        // table index below max_pages
        auto page_of = [&](int i) -> int {
            return pg.table[(size_t)b * pg.max_pages + ((t0 + i * TILE) >> pg.pshift)];
        };
        // copy tile i of this warp (tokens t0 + 16 i ..) from page `id` into stage s;
        // rows past t1 are zero-filled
        auto issue = [&](int i, int s, int id) {
            uint8_t *kt = ring + s * GqaSmem<D>::STAGE_BYTES;
            uint8_t *vt = kt + TILE * D * 2;
            const bool bad = id < 0 || id >= pg.num_pages;
            if (bad) atomicExch(err, PARALLAX_ERR_DEVICE_INDEX);
#pragma unroll
            for (int k = 0; k < TILE * NCH / 32; ++k) {
                const int idx = lane + 32 * k;
                const int row = idx / NCH, ch = idx % NCH;
                const int t = t0 + i * TILE + row;
                const __nv_bfloat16 *ksrc = kp, *vsrc = vp;
                uint32_t bytes = 0;
                if (t < t1) {
                    if (!bad) {
                        const size_t off = (((size_t)id * pg.Hkv + kvh) * (size_t)(pmask + 1) + (t & pmask)) * D + ch * 8;
                        ksrc = kp + off;
                        vsrc = vp + off;
                        bytes = 16;
                    }
                }
                cp_async16(smem_addr(kt + tile_off<D>(row, ch)), ksrc, bytes);
                cp_async16(smem_addr(vt + tile_off<D>(row, ch)), vsrc, bytes);
            }
        };

        // this warp's tiles are i = warp + WARPS k; tile k lives in stage k % STAGES
#pragma unroll
        for (int k = 0; k < STAGES - 1; ++k) {
            if (warp + WARPS * k < ntiles) issue(warp + WARPS * k, k, page_of(warp + WARPS * k));
            cp_async_commit();
        }
        // the page of the next tile to copy is read one iteration ahead, so its
        // load overlaps this iteration's arithmetic
        int id_next = warp + WARPS * (STAGES - 1) < ntiles ? page_of(warp + WARPS * (STAGES - 1)) : 0;
        int s = 0;
        for (int i = warp, k = 0; i < ntiles; i += WARPS, ++k, s = (s + 1 == STAGES) ? 0 : s + 1) {
            const int inext = i + WARPS * (STAGES - 1);
            if (inext < ntiles) issue(inext, (s + STAGES - 1) % STAGES, id_next);   // the stage computed last iteration
            cp_async_commit();
            if (inext + WARPS < ntiles) id_next = page_of(inext + WARPS);
            cp_async_wait<STAGES - 1>();
            __syncwarp();
            const uint8_t *kt = ring + s * GqaSmem<D>::STAGE_BYTES;
            const uint8_t *vt = kt + TILE * D * 2;
            const uint32_t kbase = smem_addr(kt), vbase = smem_addr(vt);

            // ---- scores: sacc[nt] = (z, z, a, a) of head r at tokens 8 nt + 2 t4 + {0, 1} ----
            float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                const int mi = lane >> 3;
                const int row = (mi >> 1) * 8 + (lane & 7);
                const int ch = 2 * ks + (mi & 1);
                uint32_t b0, b1, b2, b3;
                ldsm_x4(kbase + tile_off<D>(row, ch), b0, b1, b2, b3);
                mma_bf16(sacc[0], qa[ks], b0, b1);
                mma_bf16(sacc[1], qa[ks], b2, b3);
            }
            // ---- online softmax for head r over the tile's 16 tokens ----
            const int nvalid = t1 - (t0 + i * TILE);                 // tokens of this tile inside [t0, t1)
            float z[4], a[4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int tok = nt * 8 + 2 * t4 + e;
                    z[2 * nt + e] = tok < nvalid ? sacc[nt][e] * scale_log2 : -INFINITY;
                    a[2 * nt + e] = sacc[nt][2 + e];
                }
            float mx = fmaxf(fmaxf(z[0], z[1]), fmaxf(z[2], z[3]));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float m_new = fmaxf(m_run, mx);
            const float alpha = m_run == -INFINITY ? 0.f : fex2(m_run - m_new);
            if (__any_sync(0xffffffffu, m_new != m_run)) {
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    oacc[j][0] *= alpha;
                    oacc[j][1] *= alpha;
                    oacc[j][2] *= alpha;
                    oacc[j][3] *= alpha;
                }
                l_run *= alpha;
                ab_run *= alpha;
            }
            m_run = m_new;
            // p and p a as fp16 (rows of heads past nh stay zero); sums from the rounded values
            uint32_t pf[4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                float p0 = (r < nh && z[2 * nt] != -INFINITY) ? fex2(z[2 * nt] - m_new) : 0.f;
                float p1 = (r < nh && z[2 * nt + 1] != -INFINITY) ? fex2(z[2 * nt + 1] - m_new) : 0.f;
                const uint32_t pp = f16x2(p0, p1);
                const uint32_t pa = f16x2(f16_lo(pp) * a[2 * nt], f16_hi(pp) * a[2 * nt + 1]);
                l_run += f16_lo(pp) + f16_hi(pp);
                ab_run += f16_lo(pa) + f16_hi(pa);
                pf[2 * nt] = pp;        // A rows r, tokens 8 nt + 2 t4 + {0, 1}
                pf[2 * nt + 1] = pa;    // A rows r + 8
            }
            const uint32_t afr[4] = {pf[0], pf[1], pf[2], pf[3]};
            // ---- O += P V and M += (P o A) V over the 16 tokens ----
#pragma unroll
            for (int j = 0; j < NT; j += 2) {
                const int mi = lane >> 3;
                const int row = (mi & 1) * 8 + (lane & 7);
                const int ch = j + (mi >> 1);
                uint32_t v0, v1, v2, v3;
                ldsm_x4_t(vbase + tile_off<D>(row, ch), v0, v1, v2, v3);
                mma_f16(oacc[j], afr, bf16x2_to_f16x2(v0), bf16x2_to_f16x2(v1));
                mma_f16(oacc[j + 1], afr, bf16x2_to_f16x2(v2), bf16x2_to_f16x2(v3));
            }
            __syncwarp();   // this stage is refilled by the next iteration's copies
        }
        cp_async_wait_0();

        // ---- merge the four warps' states per head ----
        l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
        l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
        ab_run += __shfl_xor_sync(0xffffffffu, ab_run, 1);
        ab_run += __shfl_xor_sync(0xffffffffu, ab_run, 2);
        __syncthreads();   // every warp is done with its ring: reuse it for the merge
        float *mg = reinterpret_cast<float *>(smem) + (size_t)warp * 8 * (2 * D + 3);
        float *mrow = mg + r * (2 * D + 3);
        if (t4 == 0) {
            mrow[0] = m_run;
            mrow[1] = l_run;
            mrow[2] = ab_run;
        }
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            mrow[3 + j * 8 + 2 * t4] = oacc[j][0];
            mrow[3 + j * 8 + 2 * t4 + 1] = oacc[j][1];
            mrow[3 + D + j * 8 + 2 * t4] = oacc[j][2];
            mrow[3 + D + j * 8 + 2 * t4 + 1] = oacc[j][3];
        }
        __syncthreads();
        const float *mgall = reinterpret_cast<const float *>(smem);
        for (int idx = threadIdx.x; idx < nh * D; idx += WARPS * 32) {
            const int hh = idx / D, e = idx % D;
            float mu = -INFINITY;
#pragma unroll
            for (int w = 0; w < WARPS; ++w) mu = fmaxf(mu, mgall[(w * 8 + hh) * (2 * D + 3)]);
            float l = 0.f, ab = 0.f, o = 0.f, m = 0.f;
#pragma unroll
            for (int w = 0; w < WARPS; ++w) {
                const float *src = mgall + (w * 8 + hh) * (2 * D + 3);
                const float f = src[0] == -INFINITY ? 0.f : fex2(src[0] - mu);
                l = fmaf(f, src[1], l);
                ab = fmaf(f, src[2], ab);
                o = fmaf(f, src[3 + e], o);
                m = fmaf(f, src[3 + D + e], m);
            }
            const long bh = h0 + hh;
            if (nsplit == 1) {
                float out = 0.f;
                if (l > 0.f) {
                    const float inv = 1.0f / l;
                    const float oo = o * inv;
                    out = oo - (m * inv - oo * (ab * inv));
                }
                store_y<Tout>(y + bh * D + e, out);
                if (e == 0 && lse != nullptr) lse[bh] = l > 0.f ? (mu + log2f(l)) * LN2 : -INFINITY;
            } else {
                float *P = partials + ((size_t)bh * nsplit + split) * (2 * D + 3);
                P[3 + e] = o;
                P[3 + D + e] = m;
                if (e == 0) {
                    P[0] = mu;
                    P[1] = l;
                    P[2] = ab;
                }
            }
        }
        __syncthreads();   // the merge area is the next unit's ring
    }
}

template <int D, typename Tout>
cudaError_t launch_t(const void *q, const void *rho, const void *kpages, const void *vpages, const PagedKV &pg,
                     const int *seqlens, void *y, float *lse, int B, int Hq, const DecodePlan &p, float *partials,
                     int *err, cudaStream_t s) {
    constexpr int SMEM = GqaSmem<D>::BYTES;
    static std::atomic<unsigned long long> limit_set{0};
    if (cudaError_t e = ensure_smem_limit(k_decode_gqa<D, Tout>, SMEM, limit_set)) return e;
    const int htiles = (pg.group + 7) / 8;
    const long per_split = (long)B * pg.Hkv * htiles;
    const long units = per_split * p.nsplit;
    const long grid = units < 0x7fffffffL ? units : 0x7fffffffL;
    k_decode_gqa<D, Tout><<<(unsigned)grid, WARPS * 32, SMEM, s>>>(
        (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)rho, (const __nv_bfloat16 *)kpages,
        (const __nv_bfloat16 *)vpages, seqlens, (Tout *)y, lse, Hq, p.chunk, p.nsplit, per_split, htiles, pg,
        partials, err);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_gqa_split(const void *q, const void *rho, const void *kpages, const void *vpages,
                                    const PagedKV &pg, const int *seqlens, void *y, float *lse, int B, int Hq, int d,
                                    int out_dtype, const DecodePlan &p, float *partials, int *err, cudaStream_t s) {
    if (d == 64) {
        if (out_dtype == PARALLAX_F32)
            return launch_t<64, float>(q, rho, kpages, vpages, pg, seqlens, y, lse, B, Hq, p, partials, err, s);
        return launch_t<64, __nv_bfloat16>(q, rho, kpages, vpages, pg, seqlens, y, lse, B, Hq, p, partials, err, s);
    }
    if (out_dtype == PARALLAX_F32)
        return launch_t<128, float>(q, rho, kpages, vpages, pg, seqlens, y, lse, B, Hq, p, partials, err, s);
    return launch_t<128, __nv_bfloat16>(q, rho, kpages, vpages, pg, seqlens, y, lse, B, Hq, p, partials, err, s);
}

}  // namespace plx
