// convert.cu -- V bf16 -> scaled fp16 blocks, the operand of the prefill's P.V products.
//
// The forward kernel feeds its P.V and (P o A).V products from fp16 operands:
// fp16 keeps 3 more mantissa bits than bf16, which keeps the rounding of the
// staged correction weights P o A inside the error budget, and both operands
// of one product must share a type.  fp16 has far less range than bf16, so V
// is converted in blocks of 64 keys (one V stage of the forward kernel) of one
// head, each with its own power-of-two scale 2^-e chosen from the block's
// largest |v|: e = 0 for ordinary magnitudes, e = -4 when the largest |v| is
// below 2^-6 (out of fp16's subnormal range), e = E - 14 (at most 7) when it
// is 2^E >= 2^15 (under fp16's maximum).  The forward kernel multiplies that
// block's softmax weights by 2^e, so every product P.V is unchanged exactly.
//
// One CTA of 128 threads per (head, 64-key block); HBM-bound: 2 bytes read and
// 2 written per element plus one byte per block.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"

namespace plx {
namespace {

constexpr int KEYS = 64;        // keys per block (one V stage of the forward kernel)
constexpr int NT = 128;         // threads per block

__device__ __forceinline__ int block_exponent(uint32_t maxbits) {
    if (maxbits == 0) return 0;
    const int E = (int)(maxbits >> 7) - 127;   // unbiased exponent of the largest magnitude
    if (E >= 15) return min(E - 14, 7);
    if (E < -6) return -4;
    return 0;
}

template <int D>
__global__ void __launch_bounds__(NT) k_v_to_f16_blocks(const uint4 *__restrict__ v, uint4 *__restrict__ v16,
                                                         signed char *__restrict__ vexp, int T, int nblk) {
    constexpr int VEC = KEYS * D * 2 / 16 / NT;   // 16-byte vectors per thread (8 at d = 128)
    __shared__ uint32_t wmax[NT / 32];
    const long blk = blockIdx.x;                  // (bh, block) flattened
    const long bh = blk / nblk;
    const int kb = (int)(blk % nblk);
    const int rows = min(KEYS, T - kb * KEYS);    // keys in this block (the last one may be short)
    const int nvec = rows * D / 8;                // valid 16-byte vectors
    const size_t base = ((size_t)bh * T + (size_t)kb * KEYS) * D / 8;
    uint4 u[VEC];
    uint32_t m2 = 0;
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
        const int idx = threadIdx.x + i * NT;
        u[i] = idx < nvec ? __ldg(v + base + idx) : make_uint4(0, 0, 0, 0);
        m2 = __vmaxu2(m2, u[i].x & 0x7FFF7FFFu);
        m2 = __vmaxu2(m2, u[i].y & 0x7FFF7FFFu);
        m2 = __vmaxu2(m2, u[i].z & 0x7FFF7FFFu);
        m2 = __vmaxu2(m2, u[i].w & 0x7FFF7FFFu);
    }
    uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
    __syncthreads();
    m = max(max(wmax[0], wmax[1]), max(wmax[2], wmax[3]));
    const int e = block_exponent(m);
    const float sc = __int_as_float((127 - e) << 23);   // 2^-e, exact
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
        const int idx = threadIdx.x + i * NT;
        if (idx >= nvec) continue;
        const uint32_t w[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
        uint32_t o[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            // exact: a power-of-two multiple of a bf16 value, then fp16 rounding
            const __half2 h = __floats2half2_rn(__uint_as_float(w[t] << 16) * sc, __uint_as_float(w[t] & 0xFFFF0000u) * sc);
            o[t] = *reinterpret_cast<const uint32_t *>(&h);
        }
        v16[base + idx] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    if (threadIdx.x == 0) vexp[blk] = (signed char)e;
}

}  // namespace

int v16_blocks(int T) { return (T + KEYS - 1) / KEYS; }

cudaError_t launch_v_to_f16_blocks(const void *v, void *v16, signed char *vexp, int BH, int T, int d,
                                   cudaStream_t s) {
    const int nblk = v16_blocks(T);
    const long grid = (long)BH * nblk;
    if (grid > 0x7fffffffL) return cudaErrorInvalidConfiguration;
    if (d == 64)
        k_v_to_f16_blocks<64><<<(unsigned)grid, NT, 0, s>>>(static_cast<const uint4 *>(v), static_cast<uint4 *>(v16),
                                                            vexp, T, nblk);
    else
        k_v_to_f16_blocks<128><<<(unsigned)grid, NT, 0, s>>>(static_cast<const uint4 *>(v), static_cast<uint4 *>(v16),
                                                             vexp, T, nblk);
    return cudaGetLastError();
}

}  // namespace plx
