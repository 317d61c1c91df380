// convert.cu -- V bf16 -> fp16, the operand precision of the tensor-core P.V products.
//
// The forward kernel feeds its P.V and (P o A).V products from fp16 operands:
// fp16 keeps 3 more mantissa bits than bf16, which keeps the rounding of the
// staged correction weights P o A (|a| up to tens at d_model-2048 shapes) well
// inside the error budget.  Both UMMA operands of one product must share a
// type, so V is converted once per call.  HBM-bound: 2 bytes read + 2 written
// per element, 16-byte vectors, grid-stride.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"

namespace plx {
namespace {

__global__ void __launch_bounds__(256) k_bf16_to_f16(const uint4 *__restrict__ src, uint4 *__restrict__ dst,
                                                     size_t nvec) {
    size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (; i < nvec; i += stride) {
        uint4 in = __ldg(src + i);
        uint32_t w[4] = {in.x, in.y, in.z, in.w};
        uint32_t o[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            float lo = __uint_as_float(w[t] << 16);
            float hi = __uint_as_float(w[t] & 0xFFFF0000u);
            __half2 h = __floats2half2_rn(lo, hi);
            o[t] = *reinterpret_cast<uint32_t *>(&h);
        }
        dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

}  // namespace

cudaError_t launch_convert_bf16_to_f16(const void *src, void *dst, size_t n, cudaStream_t s) {
    // n is a multiple of 8 (d is 64 or 128), pointers 16-byte aligned (checked by the API).
    const size_t nvec = n / 8;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    size_t blocks = (nvec + 255) / 256;
    const size_t cap = (size_t)sms * 8;
    if (blocks > cap) blocks = cap;
    if (blocks == 0) return cudaSuccess;
    k_bf16_to_f16<<<(unsigned)blocks, 256, 0, s>>>(static_cast<const uint4 *>(src), static_cast<uint4 *>(dst), nvec);
    return cudaGetLastError();
}

}  // namespace plx
