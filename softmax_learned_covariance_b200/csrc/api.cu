// api.cu -- the C ABI declared in include/parallax.h.
//
// Host side only: argument validation, per-device state (device error word and
// a stream-ordered memory pool for per-call scratch), TMA descriptor encoding
// and kernel launches.  Every compute step runs in the CUDA kernels of this
// directory; there is no host fallback.
//
// Scratch.  A call that needs scratch (the prefill's work counter and
// block-scaled fp16 copy of V, the split partials of the decodes) takes it
// from the
// library's pool with cudaMallocFromPoolAsync on the call's own stream and
// hands it back with cudaFreeAsync on that stream right after enqueueing its
// kernels.  Stream order therefore keeps the memory alive exactly as long as
// the call's kernels run: calls on different streams, or from different host
// threads, never share scratch, and no buffer is ever freed while a kernel that
// was handed it may still run.  The pool keeps freed memory for reuse (its
// release threshold is unlimited), so steady-state calls do not reach the
// driver's allocator.
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "internal.h"
#include "parallax.h"

using namespace plx;

namespace {

constexpr int MAX_DEVICES = 64;

struct DevState {
    bool init = false;
    int sms = 0;
    int *err = nullptr;              // device error word
    cudaMemPool_t pool = nullptr;    // per-call scratch, stream-ordered
};

std::mutex g_mu;
DevState g_dev[MAX_DEVICES];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int status_of(cudaError_t e) { return e == cudaSuccess ? PARALLAX_OK : PARALLAX_ERR_CUDA; }

int get_state(DevState **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return PARALLAX_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    DevState &s = g_dev[dev];
    if (!s.init) {
        if (cudaDeviceGetAttribute(&s.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return PARALLAX_ERR_CUDA;
        if (cudaMalloc(&s.err, 256) != cudaSuccess) return PARALLAX_ERR_CUDA;
        if (cudaMemset(s.err, 0, 256) != cudaSuccess) return PARALLAX_ERR_CUDA;
        cudaMemPoolProps props;
        std::memset(&props, 0, sizeof(props));
        props.allocType = cudaMemAllocationTypePinned;
        props.handleTypes = cudaMemHandleTypeNone;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        if (cudaMemPoolCreate(&s.pool, &props) != cudaSuccess) return PARALLAX_ERR_CUDA;
        unsigned long long keep = ~0ull;
        if (cudaMemPoolSetAttribute(s.pool, cudaMemPoolAttrReleaseThreshold, &keep) != cudaSuccess)
            return PARALLAX_ERR_CUDA;
        s.init = true;
    }
    *out = &s;
    return PARALLAX_OK;
}

// Scratch of one call: taken from the pool in the call's stream order, given
// back in the same order when this object goes out of scope (after the call
// has enqueued its kernels, so the free runs after them on the device).
class CallScratch {
  public:
    CallScratch(const DevState *s, cudaStream_t st) : s_(s), st_(st) {}
    CallScratch(const CallScratch &) = delete;
    CallScratch &operator=(const CallScratch &) = delete;
    ~CallScratch() {
        if (p_) cudaFreeAsync(p_, st_);
    }
    // 256-byte aligned device memory of at least `bytes` (nullptr for 0 bytes).
    int get(size_t bytes, void **out) {
        *out = nullptr;
        if (bytes == 0) return PARALLAX_OK;
        if (cudaMallocFromPoolAsync(&p_, bytes, s_->pool, st_) != cudaSuccess) {
            p_ = nullptr;
            return PARALLAX_ERR_CUDA;
        }
        *out = p_;
        return PARALLAX_OK;
    }

  private:
    const DevState *s_;
    cudaStream_t st_;
    void *p_ = nullptr;
};

}  // namespace

DeviceCtl plx::ctl_from_env(int *err) {
    DeviceCtl c;
    c.err = err;
    unsigned long long ms = 2000;
    if (const char *e = std::getenv("PARALLAX_WAIT_TIMEOUT_MS")) {
        const long v = std::strtol(e, nullptr, 10);
        if (v > 0) ms = (unsigned long long)v;
    }
    c.wait_ns = ms * 1000000ull;
    c.debug_flags = 0;
    if (const char *e = std::getenv("PARALLAX_DEBUG_FLAGS")) c.debug_flags = (unsigned)std::strtoul(e, nullptr, 0);
    return c;
}

namespace {

DeviceCtl make_ctl(const DevState *s) { return ctl_from_env(s->err); }

int ensure_encoder() {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_encode) return PARALLAX_OK;
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
        return PARALLAX_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    return PARALLAX_OK;
}

// Row-major tensor seen as up to 3 dims (inner first), 128-byte swizzled boxes.
int encode(CUtensorMap *m, CUtensorMapDataType dt, const void *base, int rank, const uint64_t *dims,
           const uint32_t *box, uint32_t elem_bytes) {
    cuuint64_t gdim[3], gstride[2];
    cuuint32_t gbox[3], estr[3] = {1, 1, 1};
    uint64_t stride = elem_bytes;
    for (int i = 0; i < rank; ++i) {
        gdim[i] = dims[i];
        gbox[i] = box[i];
        if (i > 0) gstride[i - 1] = stride;
        stride *= dims[i];
    }
    CUresult r = g_encode(m, dt, (cuuint32_t)rank, const_cast<void *>(base), gdim, gstride, gbox, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? PARALLAX_OK : PARALLAX_ERR_CUDA;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// Common part of the tensor-core prefill calls: per-call scratch (the work
// counter, the block exponents of V and V as block-scaled fp16), the
// conversion of V, and the tensor maps of q, k and the fp16 V.  tm->r, tm->x
// and tm->w are set to a valid map the caller replaces when it needs them.
int prepare_fwd(const void *q, const void *k, const void *v, int B, int H, int T, int d, cudaStream_t cs,
                CallScratch &scratch, FwdTensorMaps *tm, signed char **vexp, int **counter) {
    const size_t n = (size_t)B * H * T * d;
    const size_t nexp = ((size_t)B * H * v16_blocks(T) + 255) & ~(size_t)255;
    void *ws = nullptr;
    int st;
    if ((st = scratch.get(256 + nexp + n * 2, &ws))) return st;
    *counter = static_cast<int *>(ws);
    *vexp = static_cast<signed char *>(ws) + 256;
    void *v16 = static_cast<char *>(ws) + 256 + nexp;
    if (launch_v_to_f16_blocks(v, v16, *vexp, B * H, T, d, cs) != cudaSuccess) return PARALLAX_ERR_CUDA;
    const uint64_t dims[3] = {(uint64_t)d, (uint64_t)T, (uint64_t)B * H};
    // boxes: 64 head-dim columns (128 B, the swizzle span) x {128 query rows, 128 keys, 64 keys}
    const uint32_t box_q[3] = {64, 128, 1}, box_k[3] = {64, 128, 1}, box_v[3] = {64, 64, 1};
    if ((st = encode(&tm->q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q, 3, dims, box_q, 2))) return st;
    if ((st = encode(&tm->k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, k, 3, dims, box_k, 2))) return st;
    if ((st = encode(&tm->v, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, v16, 3, dims, box_v, 2))) return st;
    tm->r = tm->x = tm->w = tm->q;
    return PARALLAX_OK;
}

}  // namespace

extern "C" {

const char *parallax_strerror(int status) {
    switch (status) {
        case PARALLAX_OK: return "ok";
        case PARALLAX_ERR_NULL: return "a required pointer is NULL";
        case PARALLAX_ERR_SHAPE: return "a size argument is out of range";
        case PARALLAX_ERR_ALIGN: return "a pointer is not suitably aligned (16 bytes for tensors)";
        case PARALLAX_ERR_DTYPE: return "unsupported dtype or dtype combination";
        case PARALLAX_ERR_UNSUPPORTED: return "request not served by this build";
        case PARALLAX_ERR_CUDA: return "a CUDA call failed";
        case PARALLAX_ERR_DEVICE_TIMEOUT: return "a device-side wait gave up (bounded wait expired)";
        case PARALLAX_ERR_DEVICE_INDEX: return "a device-side index (a page id) was out of range";
        case PARALLAX_ERR_DEVICE_RANGE: return "a result was not finite (an input outside the kernel's range)";
        default: return "unknown status";
    }
}

int parallax_device_sm_count(void) {
    DevState *s = nullptr;
    if (get_state(&s) != PARALLAX_OK) return 0;
    return s->sms;
}

int parallax_last_device_error(parallax_stream_t stream) {
    DevState *s = nullptr;
    int st = get_state(&s);
    if (st) return st;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return PARALLAX_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, s->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return PARALLAX_ERR_CUDA;
    if (v != 0 && cudaMemset(s->err, 0, sizeof(int)) != cudaSuccess) return PARALLAX_ERR_CUDA;
    if (int *w = noalloc_error_word()) {
        int v2 = 0;
        if (cudaMemcpy(&v2, w, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return PARALLAX_ERR_CUDA;
        if (v2 != 0 && cudaMemset(w, 0, sizeof(int)) != cudaSuccess) return PARALLAX_ERR_CUDA;
        if (v == 0) v = v2;
    }
    return v;
}

int parallax_fwd(const void *q, const void *k, const void *v, const void *rho, void *y, float *lse, int B, int H,
                 int T, int d, int causal, int in_dtype, int out_dtype, parallax_stream_t stream) {
    if (!q || !k || !v || !y) return PARALLAX_ERR_NULL;
    if (B < 1 || H < 1 || T < 1 || (d != 64 && d != 128)) return PARALLAX_ERR_SHAPE;
    if ((long long)B * H * T * d > (1ll << 40) || (long long)B * H > (1ll << 30)) return PARALLAX_ERR_SHAPE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(y) || (rho && !aligned16(rho)) ||
        (lse && !aligned4(lse)))
        return PARALLAX_ERR_ALIGN;
    const bool f32 = in_dtype == PARALLAX_F32 && out_dtype == PARALLAX_F32;
    const bool bf16 = in_dtype == PARALLAX_BF16 && (out_dtype == PARALLAX_F32 || out_dtype == PARALLAX_BF16);
    if (!f32 && !bf16) return PARALLAX_ERR_DTYPE;

    DevState *s = nullptr;
    int st = get_state(&s);
    if (st) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);

    if (f32) return status_of(launch_fwd_simt(q, k, v, rho, y, lse, B, H, T, d, causal, in_dtype, out_dtype, cs));

    if ((st = ensure_encoder())) return st;
    CallScratch scratch(s, cs);
    FwdTensorMaps tm;
    signed char *vexp = nullptr;
    int *counter = nullptr;
    if ((st = prepare_fwd(q, k, v, B, H, T, d, cs, scratch, &tm, &vexp, &counter))) return st;
    if (rho) {
        const uint64_t dims[3] = {(uint64_t)d, (uint64_t)T, (uint64_t)B * H};
        const uint32_t box_q[3] = {64, 128, 1};
        if ((st = encode(&tm.r, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rho, 3, dims, box_q, 2))) return st;
    }
    return status_of(launch_fwd_sm100(tm, rho != nullptr, y, lse, nullptr, nullptr, vexp, B, H, T, d, causal,
                                      out_dtype, s->sms, counter, make_ctl(s), cs));
}

int parallax_fwd_train(const void *q, const void *k, const void *v, const void *rho, float *y, float *lse, float *o,
                       float *abar, int B, int H, int T, int d, int causal, int in_dtype, parallax_stream_t stream) {
    if (!q || !k || !v || !rho || !y || !lse || !o || !abar) return PARALLAX_ERR_NULL;
    if (B < 1 || H < 1 || T < 1 || (d != 64 && d != 128)) return PARALLAX_ERR_SHAPE;
    if ((long long)B * H * T * d > (1ll << 40) || (long long)B * H > (1ll << 30)) return PARALLAX_ERR_SHAPE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(rho) || !aligned16(y) || !aligned16(o) ||
        !aligned4(lse) || !aligned4(abar))
        return PARALLAX_ERR_ALIGN;
    if (in_dtype != PARALLAX_BF16) return PARALLAX_ERR_DTYPE;
    DevState *s = nullptr;
    int st = get_state(&s);
    if (st) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if ((st = ensure_encoder())) return st;
    CallScratch scratch(s, cs);
    FwdTensorMaps tm;
    signed char *vexp = nullptr;
    int *counter = nullptr;
    if ((st = prepare_fwd(q, k, v, B, H, T, d, cs, scratch, &tm, &vexp, &counter))) return st;
    const uint64_t dims[3] = {(uint64_t)d, (uint64_t)T, (uint64_t)B * H};
    const uint32_t box_q[3] = {64, 128, 1};
    if ((st = encode(&tm.r, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rho, 3, dims, box_q, 2))) return st;
    return status_of(launch_fwd_sm100(tm, true, y, lse, o, abar, vexp, B, H, T, d, causal, PARALLAX_F32, s->sms,
                                      counter, make_ctl(s), cs));
}

int parallax_bwd(const void *q, const void *k, const void *v, const void *rho, const float *y, const float *o,
                 const float *abar, const float *lse, const void *dy, float *dq, float *dk, float *dv, float *drho,
                 int B, int H, int T, int d, int causal, int in_dtype, parallax_stream_t stream) {
    if (!q || !k || !v || !rho || !y || !o || !abar || !lse || !dy || !dq || !dk || !dv || !drho)
        return PARALLAX_ERR_NULL;
    if (B < 1 || H < 1 || T < 1 || (d != 64 && d != 128)) return PARALLAX_ERR_SHAPE;
    if ((long long)B * H * T * d > (1ll << 40) || (long long)B * H > 65535) return PARALLAX_ERR_SHAPE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(rho) || !aligned16(y) || !aligned16(o) ||
        !aligned16(dy) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(drho) || !aligned4(abar) ||
        !aligned4(lse))
        return PARALLAX_ERR_ALIGN;
    if (in_dtype != PARALLAX_BF16) return PARALLAX_ERR_DTYPE;
    DevState *s = nullptr;
    int st = get_state(&s);
    if (st) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if ((st = ensure_encoder())) return st;
    // scratch: the two gradient kernels' work counters, go and delta per row,
    // then the packed per-query statistics (rows padded to a multiple of 64 per head)
    CallScratch scratch(s, cs);
    void *ws = nullptr;
    const size_t rows = (size_t)B * H * T, prows = (size_t)B * H * bwd_tpad(T);
    const size_t off_st = (256 + 2 * rows * sizeof(float) + 255) & ~(size_t)255;
    if ((st = scratch.get(off_st + prows * 16, &ws))) return st;
    int *counters = static_cast<int *>(ws);
    float *go = reinterpret_cast<float *>(static_cast<char *>(ws) + 256), *delta = go + rows;
    void *st4 = static_cast<char *>(ws) + off_st;
    BwdTensorMaps tq, tk;
    const uint64_t dims[3] = {(uint64_t)d, (uint64_t)T, (uint64_t)B * H};
    const uint32_t box128[3] = {64, 128, 1}, box64[3] = {64, 64, 1};
    const void *src[5] = {q, rho, dy, k, v};
    CUtensorMap *mq[5] = {&tq.q, &tq.r, &tq.g, &tq.k, &tq.v}, *mk[5] = {&tk.q, &tk.r, &tk.g, &tk.k, &tk.v};
    for (int i = 0; i < 5; ++i) {
        if ((st = encode(mq[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, src[i], 3, dims, box128, 2))) return st;
        if ((st = encode(mk[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, src[i], 3, dims, i < 3 ? box64 : box128, 2)))
            return st;
    }
    return status_of(launch_bwd(dy, y, o, abar, lse, go, delta, st4, dq, dk, dv, drho, B, H, T, d, causal, tq, tk,
                                s->sms, counters, make_ctl(s), cs));
}

int parallax_fwd_fused(const void *q, const void *k, const void *v, const void *x, const void *W_R, void *y,
                       float *lse, int B, int H, int T, int d, int d_model, int causal, int in_dtype, int out_dtype,
                       parallax_stream_t stream) {
    if (!q || !k || !v || !x || !W_R || !y) return PARALLAX_ERR_NULL;
    if (B < 1 || H < 1 || T < 1 || (d != 64 && d != 128) || d_model < 64 || d_model % 64 != 0)
        return PARALLAX_ERR_SHAPE;
    if ((long long)B * H * T * d > (1ll << 40) || (long long)B * H > (1ll << 30) || (long long)B * T > (1ll << 31) - 1 ||
        (long long)d_model * H * d > (1ll << 40))
        return PARALLAX_ERR_SHAPE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(x) || !aligned16(W_R) || !aligned16(y) ||
        (lse && !aligned4(lse)))
        return PARALLAX_ERR_ALIGN;
    if (in_dtype != PARALLAX_BF16 || (out_dtype != PARALLAX_F32 && out_dtype != PARALLAX_BF16))
        return PARALLAX_ERR_DTYPE;
    if (d != 128) return PARALLAX_ERR_UNSUPPORTED;
    DevState *s = nullptr;
    int st = get_state(&s);
    if (st) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if ((st = ensure_encoder())) return st;
    CallScratch scratch(s, cs);
    FwdTensorMaps tm;
    signed char *vexp = nullptr;
    int *counter = nullptr;
    if ((st = prepare_fwd(q, k, v, B, H, T, d, cs, scratch, &tm, &vexp, &counter))) return st;
    // x as [B*T, d_model] in boxes of 64 x 128 rows; W_R as [d_model, H*d] in boxes of 64 x 64
    const uint64_t dx[2] = {(uint64_t)d_model, (uint64_t)B * T};
    const uint32_t bx[2] = {64, 128};
    const uint64_t dw[2] = {(uint64_t)H * d, (uint64_t)d_model};
    const uint32_t bw[2] = {64, 64};
    if ((st = encode(&tm.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, 2, dx, bx, 2))) return st;
    if ((st = encode(&tm.w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W_R, 2, dw, bw, 2))) return st;
    return status_of(launch_fwd_fused_sm100(tm, y, lse, vexp, B, H, T, d_model, causal, out_dtype, s->sms, counter,
                                            make_ctl(s), cs));
}

size_t parallax_decode_workspace_bytes(int B, int H, int Tcap, int d) {
    if (B < 1 || H < 1 || Tcap < 1 || (d != 64 && d != 128)) return 0;
    DevState *s = nullptr;
    if (get_state(&s) != PARALLAX_OK) return 0;
    return decode_partials_bytes(B, H, d, plan_decode(B, H, Tcap, d, s->sms));
}

static int decode_impl(const void *q, const void *rho, const void *kcache, const void *vcache, const int *seqlens,
                       void *y, float *lse, int B, int H, int Tcap, int d, int in_dtype, int out_dtype,
                       void *workspace, size_t workspace_bytes, bool own_workspace, parallax_stream_t stream) {
    if (!q || !rho || !kcache || !vcache || !seqlens || !y) return PARALLAX_ERR_NULL;
    if (B < 1 || H < 1 || Tcap < 1 || (d != 64 && d != 128)) return PARALLAX_ERR_SHAPE;
    if ((long long)B * H * Tcap * d > (1ll << 40)) return PARALLAX_ERR_SHAPE;
    if (!aligned16(q) || !aligned16(rho) || !aligned16(kcache) || !aligned16(vcache) || !aligned4(seqlens) ||
        !aligned16(y) || (lse && !aligned4(lse)))
        return PARALLAX_ERR_ALIGN;
    if (in_dtype != PARALLAX_BF16 || (out_dtype != PARALLAX_F32 && out_dtype != PARALLAX_BF16))
        return PARALLAX_ERR_DTYPE;
    DevState *s = nullptr;
    int st = get_state(&s);
    if (st) return st;
    const DecodePlan plan = plan_decode(B, H, Tcap, d, s->sms);
    const size_t need = decode_partials_bytes(B, H, d, plan);
    void *ws = nullptr;
    CallScratch scratch(s, static_cast<cudaStream_t>(stream));
    if (own_workspace) {
        if ((st = scratch.get(need, &ws))) return st;
    } else {
        if (need > 0 && (!workspace)) return PARALLAX_ERR_NULL;
        if (workspace_bytes < need) return PARALLAX_ERR_SHAPE;
        if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return PARALLAX_ERR_ALIGN;
        ws = workspace;
    }
    return status_of(launch_decode(q, rho, kcache, vcache, seqlens, y, lse, B, H, Tcap, d, out_dtype, plan,
                                   static_cast<float *>(ws), s->sms, make_ctl(s), static_cast<cudaStream_t>(stream)));
}

int parallax_decode(const void *q, const void *rho, const void *kcache, const void *vcache, const int *seqlens,
                    void *y, float *lse, int B, int H, int Tcap, int d, int in_dtype, int out_dtype,
                    parallax_stream_t stream) {
    return decode_impl(q, rho, kcache, vcache, seqlens, y, lse, B, H, Tcap, d, in_dtype, out_dtype, nullptr, 0, true,
                       stream);
}

int parallax_softmax_decode(const void *q, const void *kcache, const void *vcache, const int *seqlens, void *y,
                            float *lse, int B, int H, int Tcap, int d, int in_dtype, int out_dtype,
                            parallax_stream_t stream) {
    if (!q || !kcache || !vcache || !seqlens || !y) return PARALLAX_ERR_NULL;
    if (B < 1 || H < 1 || Tcap < 1 || (d != 64 && d != 128 && d != 256)) return PARALLAX_ERR_SHAPE;
    if ((long long)B * H * Tcap * d > (1ll << 40)) return PARALLAX_ERR_SHAPE;
    if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned4(seqlens) || !aligned16(y) ||
        (lse && !aligned4(lse)))
        return PARALLAX_ERR_ALIGN;
    if (in_dtype != PARALLAX_BF16 || (out_dtype != PARALLAX_F32 && out_dtype != PARALLAX_BF16))
        return PARALLAX_ERR_DTYPE;
    DevState *s = nullptr;
    int st = get_state(&s);
    if (st) return st;
    const DecodePlan plan = plan_decode(B, H, Tcap, d, s->sms);
    void *ws = nullptr;
    CallScratch scratch(s, static_cast<cudaStream_t>(stream));
    if ((st = scratch.get(decode_partials_bytes(B, H, d, plan), &ws))) return st;
    return status_of(launch_softmax_decode(q, kcache, vcache, seqlens, y, lse, B, H, Tcap, d, out_dtype, plan,
                                           static_cast<float *>(ws), static_cast<cudaStream_t>(stream)));
}

int parallax_decode_paged(const void *q, const void *rho, const void *kpages, const void *vpages,
                          const int *block_table, const int *seqlens, void *y, float *lse, int B, int Hq, int Hkv,
                          int page_size, int max_pages, int num_pages, int d, int in_dtype, int out_dtype,
                          parallax_stream_t stream) {
    if (!q || !rho || !kpages || !vpages || !block_table || !seqlens || !y) return PARALLAX_ERR_NULL;
    if (B < 1 || Hkv < 1 || Hq < Hkv || Hq % Hkv != 0 || max_pages < 1 || num_pages < 1 || (d != 64 && d != 128))
        return PARALLAX_ERR_SHAPE;
    if (page_size < 16 || page_size > 4096 || (page_size & (page_size - 1)) != 0) return PARALLAX_ERR_SHAPE;
    int pshift = 0;
    while ((1 << pshift) < page_size) ++pshift;
    if ((long long)max_pages * page_size > (1ll << 30)) return PARALLAX_ERR_SHAPE;
    if ((long long)num_pages * Hkv * page_size * d > (1ll << 40)) return PARALLAX_ERR_SHAPE;
    if (!aligned16(q) || !aligned16(rho) || !aligned16(kpages) || !aligned16(vpages) || !aligned4(block_table) ||
        !aligned4(seqlens) || !aligned16(y) || (lse && !aligned4(lse)))
        return PARALLAX_ERR_ALIGN;
    if (in_dtype != PARALLAX_BF16 || (out_dtype != PARALLAX_F32 && out_dtype != PARALLAX_BF16))
        return PARALLAX_ERR_DTYPE;
    DevState *s = nullptr;
    int st = get_state(&s);
    if (st) return st;
    const int Tcap = max_pages * page_size;
    const DecodePlan plan = plan_decode_paged(B, Hq, Hkv, Tcap, d, s->sms);
    void *ws = nullptr;
    CallScratch scratch(s, static_cast<cudaStream_t>(stream));
    if ((st = scratch.get(decode_partials_bytes(B, Hq, d, plan), &ws))) return st;
    const PagedKV pg{block_table, max_pages, num_pages, pshift, Hkv, Hq / Hkv};
    return status_of(launch_decode_paged(q, rho, kpages, vpages, pg, seqlens, y, lse, B, Hq, d, out_dtype, plan,
                                         static_cast<float *>(ws), make_ctl(s), static_cast<cudaStream_t>(stream)));
}

int parallax_decode_ex(const void *q, const void *rho, const void *kcache, const void *vcache, const int *seqlens,
                       void *y, float *lse, int B, int H, int Tcap, int d, int in_dtype, int out_dtype,
                       void *workspace, size_t workspace_bytes, parallax_stream_t stream) {
    return decode_impl(q, rho, kcache, vcache, seqlens, y, lse, B, H, Tcap, d, in_dtype, out_dtype, workspace,
                       workspace_bytes, false, stream);
}

int parallax_rho_proj(const void *x, const void *W_R, void *rho, int B, int T, int d_model, int H, int d, int dtype,
                      parallax_stream_t stream) {
    if (!x || !W_R || !rho) return PARALLAX_ERR_NULL;
    if (B < 1 || T < 1 || H < 1 || (d != 64 && d != 128) || d_model < 64 || d_model % 64 != 0 || (H * d) % 256 != 0)
        return PARALLAX_ERR_SHAPE;
    if ((long long)B * T > (1ll << 31) - 1 || (long long)d_model * H * d > (1ll << 40)) return PARALLAX_ERR_SHAPE;
    if (!aligned16(x) || !aligned16(W_R) || !aligned16(rho)) return PARALLAX_ERR_ALIGN;
    if (dtype != PARALLAX_BF16) return PARALLAX_ERR_DTYPE;
    DevState *s = nullptr;
    int st = get_state(&s);
    if (st) return st;
    if ((st = ensure_encoder())) return st;
    CUtensorMap tx, tw;
    const uint64_t dx[2] = {(uint64_t)d_model, (uint64_t)B * T};
    const uint32_t bx[2] = {64, 128};
    const uint64_t dw[2] = {(uint64_t)H * d, (uint64_t)d_model};
    const uint32_t bw[2] = {64, 64};
    if ((st = encode(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, 2, dx, bx, 2))) return st;
    if ((st = encode(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W_R, 2, dw, bw, 2))) return st;
    return status_of(launch_rho_proj(tx, tw, rho, B, T, d_model, H, d, s->sms, make_ctl(s),
                                     static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
