// decode_noalloc.cu -- parallax_decode_noalloc: the split-KV decode without any allocation.
//
// Some callers cannot let a library allocate device memory on their behalf:
// serving engines that reserve the whole device through their own pool at
// start-up and run under a fixed budget, latency-critical decode loops where a
// cudaMalloc or the device-wide synchronization of a cudaFree would stall every
// stream, and plugin interfaces whose execute callbacks forbid allocation.
// parallax_decode takes its scratch from a library memory pool with a
// stream-ordered allocation per call, which reaches the driver's allocator
// whenever the pool has to grow; this entry point instead keeps the split
// partials in a fixed-size array compiled into the library, so it never
// allocates.
//
// The array lives in device memory of every GPU that loads the library and
// stays there until the process exits.  In host code its name is only a
// host-side stand-in, so its device address is fetched once per device with
// cudaGetSymbolAddress (with that device current) and passed to the kernels.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "internal.h"
#include "parallax.h"

namespace {

constexpr size_t kScratchBytes = PARALLAX_DECODE_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;
// The split plan caps the partials at 64 units per SM of 2d + 3 floats, so on
// any device with up to this many SMs (a B200 has 148) every shape fits and the
// size check below never rejects.
constexpr int kSmsAlwaysFit = 252;
static_assert(plx::decode_partials_bound(kSmsAlwaysFit, 128) <= kScratchBytes,
              "the static decode scratch must hold the partials of every shape on these devices");

// Shared by every call on a device; keeps the last call's contents.
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];
// Where this entry point's kernels record a bounded wait that gave up
// (read and cleared by parallax_last_device_error).
static __device__ int g_noalloc_err;

struct NoallocDevice {
    bool ready = false;
    void *scratch = nullptr;   // device address of g_decode_scratch on this device
    int *err = nullptr;        // device address of g_noalloc_err on this device
    int sms = 0;
};
std::mutex g_noalloc_mu;
NoallocDevice g_noalloc_dev[kMaxDevices];

// One-time set-up for the current device.  Returns a parallax_status_t.
int noalloc_setup(int dev, NoallocDevice **out) {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    NoallocDevice &s = g_noalloc_dev[dev];
    if (!s.ready) {
        void *p = nullptr, *e = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return PARALLAX_ERR_CUDA;
        if (cudaGetSymbolAddress(&e, g_noalloc_err) != cudaSuccess || e == nullptr) return PARALLAX_ERR_CUDA;
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
            return PARALLAX_ERR_CUDA;
        s.scratch = p;
        s.err = static_cast<int *>(e);
        s.sms = sms;
        s.ready = true;
    }
    *out = &s;
    return PARALLAX_OK;
}

}  // namespace

int *plx::noalloc_error_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    return g_noalloc_dev[dev].ready ? g_noalloc_dev[dev].err : nullptr;
}

namespace {

bool is_aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" PARALLAX_API int parallax_decode_noalloc(const void *q, const void *rho, const void *kcache,
                                                    const void *vcache, const int *seqlens, void *y, float *lse,
                                                    int B, int H, int Tcap, int d, int in_dtype, int out_dtype,
                                                    parallax_stream_t stream) {
    if (!q || !rho || !kcache || !vcache || !seqlens || !y) return PARALLAX_ERR_NULL;
    if (B < 1 || H < 1 || Tcap < 1 || (d != 64 && d != 128)) return PARALLAX_ERR_SHAPE;
    if ((long long)B * H * Tcap * d > (1ll << 40)) return PARALLAX_ERR_SHAPE;
    if (!is_aligned(q, 16) || !is_aligned(rho, 16) || !is_aligned(kcache, 16) || !is_aligned(vcache, 16) ||
        !is_aligned(seqlens, 4) || !is_aligned(y, 16) || (lse && !is_aligned(lse, 4)))
        return PARALLAX_ERR_ALIGN;
    if (in_dtype != PARALLAX_BF16 || (out_dtype != PARALLAX_F32 && out_dtype != PARALLAX_BF16))
        return PARALLAX_ERR_DTYPE;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PARALLAX_ERR_CUDA;
    NoallocDevice *s = nullptr;
    if (int st = noalloc_setup(dev, &s)) return st;

    const plx::DecodePlan plan = plx::plan_decode(B, H, Tcap, d, s->sms);
    // Every partial the combine step reads is written earlier in the same call,
    // so nothing in the array has to be cleared between calls.
    if (plx::decode_partials_bytes(B, H, d, plan) > kScratchBytes) return PARALLAX_ERR_SHAPE;
    const cudaError_t e = plx::launch_decode(q, rho, kcache, vcache, seqlens, y, lse, B, H, Tcap, d, out_dtype, plan,
                                             static_cast<float *>(s->scratch), s->sms, plx::ctl_from_env(s->err),
                                             static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PARALLAX_OK : PARALLAX_ERR_CUDA;
}
