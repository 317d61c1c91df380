// decode.cu -- split-KV decode of one query token per sequence (HBM-bound).
//
// The pages' decode kernel reuses one KV stream for both branches (zubnet.ai
// news item on Parallax, paragraph 2; encorp.ai blog, section "Como cambia
// Parallax la historia del hardware en GPU Hopper"): per cached token the
// kernel reads k_j once and forms both z_j = q.k_j/sqrt(d) and a_j = k_j.rho,
// then reads v_j once and accumulates both o and m.  Per token: 8d flops for
// 4d bytes of K and V.
//
// Work is cut into units of (b, h, chunk of tokens), one small CTA per unit,
// ordered chunk-major: every head's first chunks (full length for any ragged
// mix) come first and the short or empty tails last, so the hardware block
// scheduler balances ragged sequence lengths without a host-side read of
// seqlens.  Within a unit each token row is read by D/8 lanes (16 bytes each,
// fully coalesced); a warp holds 32/(D/8) rows at a time and a lane group
// keeps its own online-softmax state over the rows it reads: per step it loads
// the K and V rows of UNF tokens together, forms z and a from the K row, moves
// its reference max only when a score exceeds it by more than 2^8 (so the
// rescale of its accumulators is rare), and accumulates o and m from the V
// row.  The lane groups' states meet once per unit in shared memory.  A unit
// writes either the final y (one unit per sequence) or its partial state
// (mu, l, abar, O, M) for the combine kernel, which merges the partials with
// max-rescaling.
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"

namespace plx {
namespace {

// Measured on B200 (bench shape B=64 H=16 ctx 4096, CUDA events):
// * one pass with K and V rows loaded together and per-lane-group softmax
//   state, 4 tokens per lane group in flight, 2-warp CTAs at 12 per SM (80
//   registers): 0.31 ms, within 2 % of the softmax-only instantiation;
// * the same with 2 tokens in flight: 0.34 ms; with 8 tokens at 8 CTAs per SM,
//   or 4-warp CTAs: within 2 % of the 4-token form, slower on short caches;
// * two passes per 512-token sub-chunk (K pass staging z and a in shared
//   memory, block max, V pass), 16 CTAs per SM: 0.38 ms -- the barrier-separated
//   phases left loads idle while the Parallax arithmetic ran, 17 % behind the
//   softmax-only instantiation of the same code;
// * 8-warp CTAs or a TMA-ring variant: 0.47-0.6 ms.
// The K dot products take bf16 operands straight from the loaded words
// (mixed-precision fma with f32 accumulation: exact products, as after a
// widening), which saves the unpacking of K and keeps q and rho packed.
constexpr int NW = 2;            // warps per CTA
constexpr int NTHREADS = NW * 32;
constexpr int UNF = 4;           // tokens a lane group has in flight per step (K and V rows)
constexpr int MIN_BLOCKS = 12;   // resident CTAs per SM the register budget targets
constexpr float RESCALE_LOG2 = 8.0f;   // reference max moves when a score exceeds it by this
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

__device__ __forceinline__ float fex2(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ uint4 ldg_stream(const uint4 *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void unpack8(const uint4 &u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        f[2 * t] = __uint_as_float(w[t] << 16);
        f[2 * t + 1] = __uint_as_float(w[t] & 0xFFFF0000u);
    }
}

template <typename Tout> __device__ __forceinline__ void store_out(Tout *p, float v);
template <> __device__ __forceinline__ void store_out<float>(float *p, float v) { *p = v; }
template <> __device__ __forceinline__ void store_out<__nv_bfloat16>(__nv_bfloat16 *p, float v) {
    *p = __float2bfloat16_rn(v);
}

// c + a.b with a, b the low (hi = false) or high bf16 halves of two packed
// words, f32 accumulation (the product of two bf16 values is exact in f32).
__device__ __forceinline__ float fma_bf16_half(uint32_t a, uint32_t b, float c, bool hi) {
    float r;
    if (hi)
        asm("{.reg .b16 al, ah, bl, bh;\n mov.b32 {al, ah}, %1;\n mov.b32 {bl, bh}, %2;\n"
            " fma.rn.f32.bf16 %0, ah, bh, %3;\n}"
            : "=f"(r) : "r"(a), "r"(b), "f"(c));
    else
        asm("{.reg .b16 al, ah, bl, bh;\n mov.b32 {al, ah}, %1;\n mov.b32 {bl, bh}, %2;\n"
            " fma.rn.f32.bf16 %0, al, bl, %3;\n}"
            : "=f"(r) : "r"(a), "r"(b), "f"(c));
    return r;
}

// Dot product of 8 packed bf16 values with 8 others, f32 accumulation.
__device__ __forceinline__ float dot8_bf16(const uint4 &x, const uint4 &k) {
    const uint32_t xw[4] = {x.x, x.y, x.z, x.w}, kw[4] = {k.x, k.y, k.z, k.w};
    float acc = 0.f;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        acc = fma_bf16_half(xw[t], kw[t], acc, false);
        acc = fma_bf16_half(xw[t], kw[t], acc, true);
    }
    return acc;
}

// WITH_RHO = false: plain softmax attention decode (no probe, no correction
// branch) -- the reference point the pages compare the Parallax decode with.
template <int D, typename Tout, bool WITH_RHO = true>
__global__ void __launch_bounds__(NTHREADS, MIN_BLOCKS) k_decode_split(
    const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ rho, const __nv_bfloat16 *__restrict__ kc,
    const __nv_bfloat16 *__restrict__ vc, const int *__restrict__ seqlens, Tout *__restrict__ y,
    float *__restrict__ lse, int H, int Tcap, int chunk, int nsplit, long BH, float *__restrict__ partials) {
    constexpr int LPT = D / 8;               // lanes per token row
    constexpr int TPW = 32 / LPT;            // token rows per warp
    constexpr int GROUPS = NW * TPW;         // lane groups (token slots) per CTA
    constexpr int STEP = GROUPS * UNF;       // token rows per CTA step
    __shared__ float red_o[GROUPS][D];
    __shared__ float red_m[GROUPS][D];
    __shared__ float red_s[3][GROUPS];

    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int g = lane / LPT;                 // lane group within the warp
    const int c = lane % LPT;                 // 16-byte column within the row
    const int slot = warp * TPW + g;          // lane group within the CTA
    const float scale_log2 = LOG2E / sqrtf((float)D);

    const long units = BH * nsplit;
    for (long u = blockIdx.x; u < units; u += gridDim.x) {
        const long bh = u % BH;                 // chunk-major unit order
        const int split = (int)(u / BH);
        const int b = (int)(bh / H);
        const int L = min(max(seqlens[b], 0), Tcap);   // never read past the cache
        const int t0 = split * chunk;
        if (t0 >= L && nsplit > 1) continue;  // beyond this sequence: no partial
        const int t1 = min(L, t0 + chunk);

        const uint4 qp = __ldg(reinterpret_cast<const uint4 *>(q + bh * D) + c);
        uint4 rp = make_uint4(0, 0, 0, 0);
        if constexpr (WITH_RHO) rp = __ldg(reinterpret_cast<const uint4 *>(rho + bh * D) + c);
        const uint4 *kbase = reinterpret_cast<const uint4 *>(kc + (size_t)bh * Tcap * D) + c;
        const uint4 *vbase = reinterpret_cast<const uint4 *>(vc + (size_t)bh * Tcap * D) + c;

        // this lane group's state: reference max (log2 units), sums, and its 8 columns of O, M
        float mref = -INFINITY, lsum = 0.f, asum = 0.f;
        float O[8], M[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) O[e] = M[e] = 0.f;

        for (int base = t0; base < t1; base += STEP) {
            uint4 kr[UNF], vr[UNF];
#pragma unroll
            for (int x = 0; x < UNF; ++x) {
                const int tok = base + x * GROUPS + slot;
                const bool ok = tok < t1;
                kr[x] = ok ? ldg_stream(kbase + (size_t)tok * LPT) : make_uint4(0, 0, 0, 0);
                vr[x] = ok ? ldg_stream(vbase + (size_t)tok * LPT) : make_uint4(0, 0, 0, 0);
            }
            float z[UNF], a[UNF];
            float bm = -INFINITY;
#pragma unroll
            for (int x = 0; x < UNF; ++x) {
                float dz = dot8_bf16(qp, kr[x]);
                float da = 0.f;
                if constexpr (WITH_RHO) da = dot8_bf16(rp, kr[x]);
                // butterfly over the row's lanes: every lane ends with the same sums
#pragma unroll
                for (int off = LPT / 2; off > 0; off >>= 1) {
                    dz += __shfl_xor_sync(0xffffffffu, dz, off);
                    if constexpr (WITH_RHO) da += __shfl_xor_sync(0xffffffffu, da, off);
                }
                const int tok = base + x * GROUPS + slot;
                z[x] = tok < t1 ? dz * scale_log2 : -INFINITY;
                a[x] = da;
                bm = fmaxf(bm, z[x]);
            }
            if (bm > mref + RESCALE_LOG2) {   // the same decision in every lane of the group
                const float alpha = fex2(mref - bm);   // 0 while mref = -inf
                mref = bm;
                lsum *= alpha;
                asum *= alpha;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    O[e] *= alpha;
                    M[e] *= alpha;
                }
            }
#pragma unroll
            for (int x = 0; x < UNF; ++x) {
                const float p = z[x] == -INFINITY ? 0.f : fex2(z[x] - mref);
                const float pa = p * a[x];
                lsum += p;
                asum += pa;
                float vf[8];
                unpack8(vr[x], vf);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    O[e] = fmaf(p, vf[e], O[e]);
                    if constexpr (WITH_RHO) M[e] = fmaf(pa, vf[e], M[e]);
                }
            }
        }

        // ---- merge the lane groups: common reference max mu, then the sums ----
        if (c == 0) red_s[0][slot] = mref;
        __syncthreads();
        float mu = red_s[0][0];
#pragma unroll
        for (int s = 1; s < GROUPS; ++s) mu = fmaxf(mu, red_s[0][s]);
        const float w = mref == -INFINITY ? 0.f : fex2(mref - mu);   // a group that read no token adds 0
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            red_o[slot][c * 8 + e] = O[e] * w;
            red_m[slot][c * 8 + e] = M[e] * w;
        }
        if (c == 0) {
            red_s[1][slot] = lsum * w;
            red_s[2][slot] = asum * w;
        }
        __syncthreads();
        {
            float l = 0.f, ab = 0.f;
#pragma unroll
            for (int s = 0; s < GROUPS; ++s) {
                l += red_s[1][s];
                ab += red_s[2][s];
            }
            float *P = partials + ((size_t)bh * nsplit + split) * (2 * D + 3);
            // one output dimension per thread, striding when the CTA is narrower than d
            for (int e = tid; e < D; e += NTHREADS) {
                float o = 0.f, m = 0.f;
#pragma unroll
                for (int s = 0; s < GROUPS; ++s) {
                    o += red_o[s][e];
                    m += red_m[s][e];
                }
                if (nsplit == 1) {
                    float out = 0.f;
                    if (l > 0.f) {
                        const float inv = 1.0f / l;
                        const float oo = o * inv;
                        out = oo - (m * inv - oo * (ab * inv));
                    }
                    store_out<Tout>(y + bh * D + e, out);
                } else {
                    P[3 + e] = o;
                    P[3 + D + e] = m;
                }
            }
            if (tid == 0) {
                if (nsplit == 1) {
                    if (lse != nullptr) lse[bh] = l > 0.f ? (mu + log2f(l)) * LN2 : -INFINITY;
                } else {
                    P[0] = mu;
                    P[1] = l;
                    P[2] = ab;
                }
            }
        }
        __syncthreads();   // the shared arrays are reused by the next unit
    }
}

// Merge of the split partials of one (b, h): mu* = max mu_s, w_s = 2^(mu_s - mu*),
// then l, abar, O, M are the w-weighted sums and y follows as in the split
// kernel.  The splits of a head are spread over the warps of the block (two in
// flight per warp) because a head can have hundreds of them; the warps' sums
// meet in shared memory.  Few splits take a 4-warp block, many a 16-warp one.
template <int D, typename Tout, int CMB_WARPS>
__global__ void __launch_bounds__(CMB_WARPS * 32) k_decode_combine(const float *__restrict__ partials,
                                                                  const int *__restrict__ seqlens,
                                                                  Tout *__restrict__ y, float *__restrict__ lse,
                                                                  int H, int chunk, int nsplit) {
    constexpr int PER = D / 32;   // head dimensions per lane
    constexpr int STRIDE = 2 * D + 3;
    __shared__ float red[CMB_WARPS][2 * D + 2];
    __shared__ float wmax[CMB_WARPS];
    const long bh = blockIdx.x;
    const int b = (int)(bh / H);
    const int L = min(max(seqlens[b], 0), chunk * nsplit);
    const int nvalid = min(nsplit, (L + chunk - 1) / chunk);
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const float *P = partials + (size_t)bh * nsplit * STRIDE;
    if (nvalid <= 0) {
        for (int e = tid; e < D; e += CMB_WARPS * 32) store_out<Tout>(y + bh * D + e, 0.f);
        if (lse != nullptr && tid == 0) lse[bh] = -INFINITY;
        return;
    }
    // ---- mu* ----
    float mu = -INFINITY;
    for (int s2 = tid; s2 < nvalid; s2 += CMB_WARPS * 32) mu = fmaxf(mu, P[(size_t)s2 * STRIDE]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mu = fmaxf(mu, __shfl_xor_sync(0xffffffffu, mu, off));
    if (lane == 0) wmax[warp] = mu;
    __syncthreads();
    mu = wmax[0];
#pragma unroll
    for (int w = 1; w < CMB_WARPS; ++w) mu = fmaxf(mu, wmax[w]);
    // ---- weighted sums, warp w takes splits w, w + CMB_WARPS, ... ----
    float l = 0.f, ab = 0.f, o[PER], m[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) o[i] = m[i] = 0.f;
    int s2 = warp;
    for (; s2 + CMB_WARPS < nvalid; s2 += 2 * CMB_WARPS) {
        const float *P0 = P + (size_t)s2 * STRIDE, *P1 = P0 + (size_t)CMB_WARPS * STRIDE;
        const float h0 = P0[0], h1 = P1[0], l0 = P0[1], l1 = P1[1], a0 = P0[2], a1 = P1[2];
        float ov0[PER], ov1[PER], mv0[PER], mv1[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            ov0[i] = P0[3 + lane + 32 * i];
            ov1[i] = P1[3 + lane + 32 * i];
            mv0[i] = P0[3 + D + lane + 32 * i];
            mv1[i] = P1[3 + D + lane + 32 * i];
        }
        const float w0 = fex2(h0 - mu), w1 = fex2(h1 - mu);
        l = fmaf(w1, l1, fmaf(w0, l0, l));
        ab = fmaf(w1, a1, fmaf(w0, a0, ab));
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            o[i] = fmaf(w1, ov1[i], fmaf(w0, ov0[i], o[i]));
            m[i] = fmaf(w1, mv1[i], fmaf(w0, mv0[i], m[i]));
        }
    }
    if (s2 < nvalid) {
        const float *P0 = P + (size_t)s2 * STRIDE;
        const float w0 = fex2(P0[0] - mu);
        l = fmaf(w0, P0[1], l);
        ab = fmaf(w0, P0[2], ab);
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            o[i] = fmaf(w0, P0[3 + lane + 32 * i], o[i]);
            m[i] = fmaf(w0, P0[3 + D + lane + 32 * i], m[i]);
        }
    }
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        red[warp][lane + 32 * i] = o[i];
        red[warp][D + lane + 32 * i] = m[i];
    }
    if (lane == 0) {
        red[warp][2 * D] = l;
        red[warp][2 * D + 1] = ab;
    }
    __syncthreads();
    float lt = 0.f, at = 0.f;
#pragma unroll
    for (int w = 0; w < CMB_WARPS; ++w) {
        lt += red[w][2 * D];
        at += red[w][2 * D + 1];
    }
    const float inv = 1.0f / lt;
    for (int e = tid; e < D; e += CMB_WARPS * 32) {   // one output dimension per thread
        float ot = 0.f, mt = 0.f;
#pragma unroll
        for (int w = 0; w < CMB_WARPS; ++w) {
            ot += red[w][e];
            mt += red[w][D + e];
        }
        const float oo = ot * inv;
        store_out<Tout>(y + bh * D + e, oo - (mt * inv - oo * (at * inv)));
    }
    if (lse != nullptr && tid == 0) lse[bh] = (mu + log2f(lt)) * LN2;
}

template <int D, typename Tout>
cudaError_t launch_combine(const float *partials, const int *seqlens, void *y, float *lse, int B, int H,
                           const DecodePlan &p, cudaStream_t s) {
    if (p.nsplit <= 16)
        k_decode_combine<D, Tout, 4><<<(unsigned)(B * H), 4 * 32, 0, s>>>(partials, seqlens, (Tout *)y, lse, H,
                                                                          p.chunk, p.nsplit);
    else
        k_decode_combine<D, Tout, 16><<<(unsigned)(B * H), 16 * 32, 0, s>>>(partials, seqlens, (Tout *)y, lse, H,
                                                                            p.chunk, p.nsplit);
    return cudaGetLastError();
}

template <int D, typename Tout, bool WITH_RHO = true>
cudaError_t launch_t(const void *q, const void *rho, const void *kc, const void *vc, const int *seqlens, void *y,
                     float *lse, int B, int H, int Tcap, const DecodePlan &p, float *partials, cudaStream_t s) {
    const long BH = (long)B * H;
    const long units = BH * p.nsplit;
    const long grid = units < 0x7fffffffL ? units : 0x7fffffffL;   // one CTA per unit
    k_decode_split<D, Tout, WITH_RHO><<<(unsigned)grid, NTHREADS, 0, s>>>(
        (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)rho, (const __nv_bfloat16 *)kc, (const __nv_bfloat16 *)vc,
        seqlens, (Tout *)y, lse, H, Tcap, p.chunk, p.nsplit, BH, partials);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || p.nsplit == 1) return e;
    return launch_combine<D, Tout>(partials, seqlens, y, lse, B, H, p, s);
}

}  // namespace

cudaError_t launch_decode(const void *q, const void *rho, const void *kc, const void *vc, const int *seqlens,
                          void *y, float *lse, int B, int H, int Tcap, int d, int out_dtype, const DecodePlan &p,
                          float *partials, int sm_count, const DeviceCtl &ctl, cudaStream_t s) {
    (void)ctl;   // this kernel has no device-side waits
    (void)sm_count;
    if (d == 64) {
        if (out_dtype == PARALLAX_F32)
            return launch_t<64, float>(q, rho, kc, vc, seqlens, y, lse, B, H, Tcap, p, partials, s);
        return launch_t<64, __nv_bfloat16>(q, rho, kc, vc, seqlens, y, lse, B, H, Tcap, p, partials, s);
    }
    if (out_dtype == PARALLAX_F32)
        return launch_t<128, float>(q, rho, kc, vc, seqlens, y, lse, B, H, Tcap, p, partials, s);
    return launch_t<128, __nv_bfloat16>(q, rho, kc, vc, seqlens, y, lse, B, H, Tcap, p, partials, s);
}

cudaError_t launch_softmax_decode(const void *q, const void *kc, const void *vc, const int *seqlens, void *y,
                                  float *lse, int B, int H, int Tcap, int d, int out_dtype, const DecodePlan &p,
                                  float *partials, cudaStream_t s) {
    const bool f32 = out_dtype == PARALLAX_F32;
    if (d == 64)
        return f32 ? launch_t<64, float, false>(q, nullptr, kc, vc, seqlens, y, lse, B, H, Tcap, p, partials, s)
                   : launch_t<64, __nv_bfloat16, false>(q, nullptr, kc, vc, seqlens, y, lse, B, H, Tcap, p, partials, s);
    if (d == 128)
        return f32 ? launch_t<128, float, false>(q, nullptr, kc, vc, seqlens, y, lse, B, H, Tcap, p, partials, s)
                   : launch_t<128, __nv_bfloat16, false>(q, nullptr, kc, vc, seqlens, y, lse, B, H, Tcap, p, partials,
                                                         s);
    return f32 ? launch_t<256, float, false>(q, nullptr, kc, vc, seqlens, y, lse, B, H, Tcap, p, partials, s)
               : launch_t<256, __nv_bfloat16, false>(q, nullptr, kc, vc, seqlens, y, lse, B, H, Tcap, p, partials, s);
}

cudaError_t launch_decode_paged(const void *q, const void *rho, const void *kpages, const void *vpages,
                                const PagedKV &pg, const int *seqlens, void *y, float *lse, int B, int Hq, int d,
                                int out_dtype, const DecodePlan &p, float *partials, const DeviceCtl &ctl,
                                cudaStream_t s) {
    cudaError_t e = launch_decode_gqa_split(q, rho, kpages, vpages, pg, seqlens, y, lse, B, Hq, d, out_dtype, p,
                                            partials, ctl.err, s);
    if (e != cudaSuccess || p.nsplit == 1) return e;
    if (d == 64)
        return out_dtype == PARALLAX_F32 ? launch_combine<64, float>(partials, seqlens, y, lse, B, Hq, p, s)
                                         : launch_combine<64, __nv_bfloat16>(partials, seqlens, y, lse, B, Hq, p, s);
    return out_dtype == PARALLAX_F32 ? launch_combine<128, float>(partials, seqlens, y, lse, B, Hq, p, s)
                                     : launch_combine<128, __nv_bfloat16>(partials, seqlens, y, lse, B, Hq, p, s);
}

}  // namespace plx
