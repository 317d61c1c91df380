// softmax_sm100.cuh -- device helpers shared by the tcgen05 prefill kernels:
// bounded warp-uniform waits, the persistent scheduler ring, packed fp32x2
// FMAs and the FMA-pipe exponential.
#pragma once
#include <cstdint>

#include "sm100.cuh"

namespace plx {
namespace {

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Bounded wait whose outcome is the same for all 32 lanes (lanes that saw the
// phase complete still give up if another lane of the warp gave up), so the
// .sync.aligned tcgen05 instructions that follow are never reached divergently.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const WaitCtl &wc) {
    const bool got = mbar_wait(bar, parity, wc);
    return __all_sync(0xffffffffu, got);
}

// Everyone but the scheduler takes the k-th scheduled item from the ring of
// SCHED slots (sched_full[] barriers and sched_item[] values of the Bars type).
template <int SCHED, typename Bars>
__device__ __forceinline__ bool next_item(Bars *bars, uint32_t k, int &w, const WaitCtl &wc) {
    const uint32_t s = k % SCHED;
    if (!mbar_wait(smem_u32(&bars->sched_full[s]), (k / SCHED) & 1, wc)) return false;
    w = bars->sched_item[s];
    return true;
}

// d0,d1 = a0,a1 * b + c as one packed fp32x2 FMA.
__device__ __forceinline__ void ffma2(float &d0, float &d1, float a0, float a1, float b, float c) {
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %4};\n\tmov.b64 rc, {%5, %5};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d0), "=f"(d1)
        : "f"(a0), "f"(a1), "f"(b), "f"(c));
}

// d = a * b + c elementwise on two fp32 pairs (one packed FMA).
__device__ __forceinline__ void fma2v(float &d0, float &d1, float a0, float a1, float b0, float b1, float c0,
                                      float c1) {
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d0), "=f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}

// 2^x for a pair on the FMA pipe.  The special-function unit does 16
// exponentials per clock per SM, which bounds the softmax; a share of them is
// taken here instead.  Range reduction: j = round(x) is read from the low
// mantissa bits of x + 1.5 * 2^23, f = x - j lies in [-1/2, 1/2], and 2^f is a
// degree-3 polynomial whose coefficients are the relative-error minimax fit on
// [-1/2, 1/2] from a Remez exchange (max relative error 7.5e-5, well under the
// fp16 rounding of P).  2^j is added to the exponent field.  x is clamped at
// -125 so the exponent stays normal; results there (and for x = -inf) are
// below 2^-124 and round to 0 in fp16.
constexpr float EXP2_C0 = 0.99992806f, EXP2_C1 = 0.69326097f, EXP2_C2 = 0.24261113f, EXP2_C3 = 0.05517167f;
__device__ __forceinline__ void exp2_poly2(float &y0, float &y1, float x0, float x1) {
    constexpr float kRound = 12582912.0f;   // 1.5 * 2^23
    x0 = fmaxf(x0, -125.0f);
    x1 = fmaxf(x1, -125.0f);
    float t0, t1, r0, r1, f0, f1, p0, p1;
    ffma2(t0, t1, x0, x1, 1.0f, kRound);    // kRound + round(x)
    ffma2(r0, r1, t0, t1, 1.0f, -kRound);   // round(x), exact
    fma2v(f0, f1, r0, r1, -1.0f, -1.0f, x0, x1);
    fma2v(p0, p1, f0, f1, EXP2_C3, EXP2_C3, EXP2_C2, EXP2_C2);
    fma2v(p0, p1, p0, p1, f0, f1, EXP2_C1, EXP2_C1);
    fma2v(p0, p1, p0, p1, f0, f1, EXP2_C0, EXP2_C0);
    // bits(t) << 23 == round(x) << 23 (mod 2^32): the low 9 bits of bits(1.5 * 2^23) are zero
    y0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
    y1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
}

// exp2(s c - m) for N pairs of fp32 values s, rounded to fp16 pairs (the
// softmax weights P of the prefill, s of the backward); three pairs in eight
// go through the FMA-pipe polynomial.
template <int N>
__device__ __forceinline__ void weights_f16(const uint32_t (&sr)[2 * N], uint32_t (&pk)[N], float scale_log2,
                                            float neg_m) {
#pragma unroll
    for (int i = 0; i < N; ++i) {
        float x0, x1;
        ffma2(x0, x1, __uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1]), scale_log2, neg_m);
        float e0, e1;
        if ((i & 7) == 1 || (i & 7) == 4 || (i & 7) == 7) {
            exp2_poly2(e0, e1, x0, x1);
        } else {
            e0 = ex2(x0);
            e1 = ex2(x1);
        }
        pk[i] = pack_f16x2(e0, e1);
    }
}

// One 32-byte global store (8 words); the address must be 32-byte aligned.
__device__ __forceinline__ void st_global_v8(void *p, const uint32_t (&w)[8]) {
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]),
                 "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                 : "memory");
}

}  // namespace
}  // namespace plx
