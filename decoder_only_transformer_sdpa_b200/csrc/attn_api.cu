// attn_api.cu -- the extern "C" entry points of libattn.so (declared in
// include/attn.h): argument validation, workspace carving and dispatch to the
// kernels.  Nothing here computes attention; every step runs in a kernel.
#include "../../include/attn.h"
#include "internal.h"

#include <math.h>
#include <mutex>

#define ATTN_API extern "C" __attribute__((visibility("default")))

namespace attn {
namespace {

// Device-side error word.  Kernels receive its address as an argument (one
// address per device, looked up once) and set it when a bounded wait runs out.
__device__ int g_device_error;

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int *g_err_addr[kMaxDevices];
int g_cc_major[kMaxDevices];  // 0 = not yet queried

thread_local int t_last_launches = 0;
thread_local cudaEvent_t t_prof_start = nullptr, t_prof_end = nullptr;

// Takes the armed profiling events (if any) for the call being made.
LaunchInfo take_launch_info() {
    LaunchInfo li;
    li.main_start = t_prof_start;
    li.main_end = t_prof_end;
    t_prof_start = t_prof_end = nullptr;
    return li;
}

int current_device(int &dev) {
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_DEVICE;
    return ATTN_OK;
}

// Checks the current device is sm_100 and returns its error-word address.
int device_setup(int **err_addr) {
    int dev;
    int st = current_device(dev);
    if (st != ATTN_OK) return st;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_cc_major[dev] == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return ATTN_ERR_CUDA;
        if (major != 10 || minor != 0) {
            g_cc_major[dev] = -1;
        } else {
            void *p = nullptr;
            if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return ATTN_ERR_CUDA;
            g_err_addr[dev] = static_cast<int *>(p);
            g_cc_major[dev] = major;
        }
    }
    if (g_cc_major[dev] < 0) return ATTN_ERR_DEVICE;
    if (err_addr) *err_addr = g_err_addr[dev];
    return ATTN_OK;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_shape(int B, int H, int T, int D, int dmax) {
    if (B < 1 || H < 1 || T < 1) return ATTN_ERR_SHAPE;
    if (D < 1 || D > dmax) return ATTN_ERR_UNSUPPORTED_D;
    const long double n = (long double)B * H * T * D;
    if (n > (long double)(1ll << 40)) return ATTN_ERR_SHAPE;
    if ((long long)B * H > 0x7fffffffLL / 8) return ATTN_ERR_SHAPE;
    return ATTN_OK;
}

int check_scale(float scale) {
    return (isfinite(scale) && scale > 0.f) ? ATTN_OK : ATTN_ERR_SCALE;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int finish(cudaError_t e, const LaunchInfo &li) {
    if (e != cudaSuccess) {
        cudaGetLastError();  // clear a sticky launch error of this call
        return ATTN_ERR_CUDA;
    }
    t_last_launches = li.kernels;
    return ATTN_OK;
}

bool bf16_d_supported(int D) { return D == 32 || D == 64 || D == 128; }
bool decode_d_supported(int D) { return D == 32 || D == 64; }

}  // namespace
}  // namespace attn

using namespace attn;

ATTN_API const char *attn_status_string(int status) {
    switch (status) {
        case ATTN_OK: return "ok";
        case ATTN_ERR_NULL: return "a required pointer is NULL";
        case ATTN_ERR_SHAPE: return "invalid shape (B, H, T must be >= 1; size overflow)";
        case ATTN_ERR_UNSUPPORTED_D: return "unsupported head_dim";
        case ATTN_ERR_ALIGN: return "pointer misaligned (bf16: 16 bytes, float32: 4 bytes)";
        case ATTN_ERR_CUDA: return "CUDA error";
        case ATTN_ERR_TIMEOUT: return "a bounded in-kernel wait timed out";
        case ATTN_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case ATTN_ERR_DEVICE: return "current device is not sm_100 (B200 class)";
        case ATTN_ERR_SCALE: return "scale must be finite and positive";
        case ATTN_ERR_OPTION: return "unsupported attn_options value";
        case ATTN_ERR_DEVICE_CHECK: return "a device-side bounds check failed (debug build)";
        default: return "unknown status";
    }
}

ATTN_API int attn_version(void) { return 1; }

ATTN_API int attn_profile_next_call(cudaEvent_t start, cudaEvent_t end) {
    if ((start == nullptr) != (end == nullptr)) return ATTN_ERR_NULL;
    t_prof_start = start;
    t_prof_end = end;
    return ATTN_OK;
}

ATTN_API int attn_last_launch_count(void) { return t_last_launches; }

namespace {

// A [B,H,T,D] bf16 view is usable by TMA when its batch, head and token
// strides are positive multiples of 8 elements (16 bytes) below 2^39.
bool strides_ok(const attn_strides &x) {
    auto ok = [](int64_t v) { return v > 0 && v % 8 == 0 && v < (1ll << 39); };
    return ok(x.b) && ok(x.h) && ok(x.t);
}

TStrides to_tstrides(const attn_strides &x) { return TStrides{x.b, x.h, x.t}; }

// The options of one call, as the kernels take them.
struct Opts {
    int causal = 1;
    bool dropout = false;
    DropoutParams drop{};
    uint8_t *mask = nullptr;  // a kept dropout mask (dropout only), not yet checked
    size_t mask_bytes = 0;
};

// Reads the options (NULL = the decoder's defaults: causal, no dropout).
int read_options(const attn_options *opts, Opts &out) {
    out = Opts{};
    if (!opts) return ATTN_OK;
    if (opts->causal != 0 && opts->causal != 1) return ATTN_ERR_OPTION;
    if (opts->reserved != 0) return ATTN_ERR_OPTION;
    const double p = opts->dropout_p;
    if (!(p >= 0.0 && p < 1.0)) return ATTN_ERR_OPTION;  // also rejects NaN
    const double t = floor(p * 65536.0 + 0.5);
    if (t >= 65536.0) return ATTN_ERR_OPTION;
    out.causal = opts->causal;
    if (t > 0.0) {  // threshold 0 keeps every weight with scale 1: no dropout
        out.dropout = true;
        out.drop.k0 = (uint32_t)opts->dropout_seed;
        out.drop.k1 = (uint32_t)(opts->dropout_seed >> 32);
        out.drop.thr = (uint32_t)t;
        out.drop.offset = opts->dropout_offset;
        out.drop.keep_scale = (float)(65536.0 / (65536.0 - t));
        out.mask = static_cast<uint8_t *>(opts->dropout_mask);
        out.mask_bytes = opts->dropout_mask_bytes;
    }
    return ATTN_OK;
}

size_t mask_bytes_for(int B, int H, int T) {
    if (B < 1 || H < 1 || T < 1) return 0;
    const size_t tp = ((size_t)T + 127) / 128 * 128;
    const size_t heads = (size_t)B * (size_t)H;
    if (heads > (SIZE_MAX / tp) / (tp / 8)) return 0;
    return heads * (tp / 8) * tp;
}

// Hands a kept dropout mask to the kernels once its size is checked against
// the shape (bf16 path; the float32 path draws the mask every time).
int attach_mask(Opts &op, int B, int H, int T) {
    if (!op.dropout || !op.mask) return ATTN_OK;
    const size_t need = mask_bytes_for(B, H, T);
    if (need == 0 || op.mask_bytes < need) return ATTN_ERR_OPTION;
    if (!aligned(op.mask, 16)) return ATTN_ERR_ALIGN;
    op.drop.mask = op.mask;
    op.drop.mask_ld = (uint32_t)(((size_t)T + 127) / 128 * 128);
    return ATTN_OK;
}

Shape make_shape(int B, int H, int T, int D, float scale, const Opts &op) {
    Shape s{B, H, T, D, scale};
    s.causal = op.causal;
    s.dropout = op.dropout;
    s.drop = op.drop;
    return s;
}

int fwd_strides(const attn_strides *strides, const Shape &s, FwdStrides &str) {
    if (!strides) {
        const TStrides c = contiguous_strides(s);
        str = FwdStrides{c, c, c, c};
        return ATTN_OK;
    }
    for (int i = 0; i < 4; ++i)
        if (!strides_ok(strides[i])) return ATTN_ERR_ALIGN;
    str = FwdStrides{to_tstrides(strides[0]), to_tstrides(strides[1]), to_tstrides(strides[2]),
                     to_tstrides(strides[3])};
    return ATTN_OK;
}

int bwd_strides(const attn_strides *strides, const Shape &s, BwdStrides &str) {
    if (!strides) {
        const TStrides c = contiguous_strides(s);
        str = BwdStrides{c, c, c, c, c, c, c, c};
        return ATTN_OK;
    }
    for (int i = 0; i < 8; ++i)
        if (!strides_ok(strides[i])) return ATTN_ERR_ALIGN;
    TStrides *dst[8] = {&str.q, &str.k, &str.v, &str.o, &str.dO, &str.dq, &str.dk, &str.dv};
    for (int i = 0; i < 8; ++i) *dst[i] = to_tstrides(strides[i]);
    return ATTN_OK;
}

int fwd_impl(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H, int T,
             int D, float scale, Opts op, const FwdStrides &str, cudaStream_t stream,
             LaunchInfo &li) {
    if (!q || !k || !v || !o || !lse) return ATTN_ERR_NULL;
    int st = check_shape(B, H, T, D, 128);
    if (st != ATTN_OK) return st;
    if (!bf16_d_supported(D)) return ATTN_ERR_UNSUPPORTED_D;
    if ((st = check_scale(scale)) != ATTN_OK) return st;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
        return ATTN_ERR_ALIGN;
    if ((st = attach_mask(op, B, H, T)) != ATTN_OK) return st;
    int *err = nullptr;
    if ((st = device_setup(&err)) != ATTN_OK) return st;
    const Shape sh = make_shape(B, H, T, D, scale, op);
    if (sh.drop.mask) {
        // A lent mask buffer: draw the keep bits into it first; the forward
        // (and later the backward) load them.
        const cudaError_t em = draw_dropout_mask(sh, err, stream, li);
        if (em != cudaSuccess) return finish(em, li);
    }
    cudaError_t e = sm100_fwd(static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k),
                              static_cast<const __nv_bfloat16 *>(v), static_cast<__nv_bfloat16 *>(o), lse,
                              sh, str, err, stream, li);
    return finish(e, li);
}

// Pointer, shape, head_dim, scale and alignment checks of the bf16 backward,
// in the order its status codes are reported.
int bwd_args(const void *q, const void *k, const void *v, const void *o, const float *lse,
             const void *dO, void *dq, void *dk, void *dv, int B, int H, int T, int D, float scale) {
    if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return ATTN_ERR_NULL;
    int st = check_shape(B, H, T, D, 128);
    if (st != ATTN_OK) return st;
    if (!bf16_d_supported(D)) return ATTN_ERR_UNSUPPORTED_D;
    if ((st = check_scale(scale)) != ATTN_OK) return st;
    const void *ptrs[] = {q, k, v, o, dO, dq, dk, dv};
    for (const void *p : ptrs)
        if (!aligned(p, 16)) return ATTN_ERR_ALIGN;
    if (!aligned(lse, 4)) return ATTN_ERR_ALIGN;
    return ATTN_OK;
}

int bwd_impl(const void *q, const void *k, const void *v, const void *o, const float *lse,
             const void *dO, void *dq, void *dk, void *dv, int B, int H, int T, int D, float scale,
             Opts op, const BwdStrides &str, void *workspace, size_t workspace_bytes,
             cudaStream_t stream, LaunchInfo &li) {
    int st = bwd_args(q, k, v, o, lse, dO, dq, dk, dv, B, H, T, D, scale);
    if (st != ATTN_OK) return st;
    if ((st = attach_mask(op, B, H, T)) != ATTN_OK) return st;
    const size_t need = attn_bwd_workspace_bytes(B, H, T, D);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return ATTN_ERR_WORKSPACE;
    int *err = nullptr;
    if ((st = device_setup(&err)) != ATTN_OK) return st;
    const BwdWorkspace wl = bwd_workspace_layout(B, H, T, D);
    char *ws = static_cast<char *>(workspace);
    float *dq_acc = reinterpret_cast<float *>(ws + wl.dq_acc);
    float *lse2 = reinterpret_cast<float *>(ws + wl.lse2);
    float *delta = reinterpret_cast<float *>(ws + wl.delta);
    cudaError_t e = sm100_bwd(
        static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k),
        static_cast<const __nv_bfloat16 *>(v), static_cast<const __nv_bfloat16 *>(o), lse,
        static_cast<const __nv_bfloat16 *>(dO), static_cast<__nv_bfloat16 *>(dq),
        static_cast<__nv_bfloat16 *>(dk), static_cast<__nv_bfloat16 *>(dv), dq_acc, lse2, delta,
        make_shape(B, H, T, D, scale, op), str, err, stream, li);
    return finish(e, li);
}

}  // namespace

ATTN_API int attn_fwd_ex(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                         int H, int T, int D, float scale, const attn_strides *strides,
                         const attn_options *opts, cudaStream_t stream) {
    LaunchInfo li = take_launch_info();
    Opts op;
    int st;
    if ((st = read_options(opts, op)) != ATTN_OK) return st;
    FwdStrides str;
    if ((st = fwd_strides(strides, Shape{B, H, T, D, scale}, str)) != ATTN_OK) return st;
    return fwd_impl(q, k, v, o, lse, B, H, T, D, scale, op, str, stream, li);
}

ATTN_API int attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                      int H, int T, int D, float scale, cudaStream_t stream) {
    return attn_fwd_ex(q, k, v, o, lse, B, H, T, D, scale, nullptr, nullptr, stream);
}

ATTN_API int attn_fwd_strided(const void *q, const void *k, const void *v, void *o, float *lse,
                              int B, int H, int T, int D, float scale, const attn_strides *strides,
                              cudaStream_t stream) {
    if (!strides) {
        take_launch_info();  // the arming is consumed by this call
        return ATTN_ERR_NULL;
    }
    return attn_fwd_ex(q, k, v, o, lse, B, H, T, D, scale, strides, nullptr, stream);
}

ATTN_API int attn_decode(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                         int H, int Tq, int Tk, int D, float scale, const attn_strides *strides,
                         cudaStream_t stream) {
    LaunchInfo li = take_launch_info();
    if (!q || !k || !v || !o || !lse) return ATTN_ERR_NULL;
    int st = check_shape(B, H, Tk, D, 128);
    if (st != ATTN_OK) return st;
    if (Tq < 1 || Tq > ATTN_DECODE_MAX_QUERIES || Tq > Tk) return ATTN_ERR_SHAPE;
    if (!decode_d_supported(D)) return ATTN_ERR_UNSUPPORTED_D;
    if ((st = check_scale(scale)) != ATTN_OK) return st;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
        return ATTN_ERR_ALIGN;
    FwdStrides str;
    if (strides) {
        for (int i = 0; i < 4; ++i)
            if (!strides_ok(strides[i])) return ATTN_ERR_ALIGN;
        str = FwdStrides{to_tstrides(strides[0]), to_tstrides(strides[1]), to_tstrides(strides[2]),
                         to_tstrides(strides[3])};
    } else {
        const TStrides kv = contiguous_strides(Shape{B, H, Tk, D, scale});
        const TStrides qo = contiguous_strides(Shape{B, H, Tq, D, scale});
        str = FwdStrides{qo, kv, kv, qo};
    }
    int *err = nullptr;
    if ((st = device_setup(&err)) != ATTN_OK) return st;
    cudaError_t e = sm100_decode(static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k),
                                 static_cast<const __nv_bfloat16 *>(v), static_cast<__nv_bfloat16 *>(o), lse,
                                 DecodeShape{B, H, Tq, Tk, D, scale}, str, err, stream, li);
    return finish(e, li);
}

// Workspace of the bf16 backward: dQ float32 accumulator, padded lse, Delta.
ATTN_API size_t attn_bwd_workspace_bytes(int B, int H, int T, int D) {
    if (check_shape(B, H, T, D, 128) != ATTN_OK || !bf16_d_supported(D)) return 0;
    return bwd_workspace_layout(B, H, T, D).total;
}

ATTN_API int attn_bwd_ex(const void *q, const void *k, const void *v, const void *o,
                         const float *lse, const void *dO, void *dq, void *dk, void *dv, int B,
                         int H, int T, int D, float scale, const attn_strides *strides,
                         const attn_options *opts, void *workspace, size_t workspace_bytes,
                         cudaStream_t stream) {
    LaunchInfo li = take_launch_info();
    Opts op;
    int st;
    if ((st = read_options(opts, op)) != ATTN_OK) return st;
    BwdStrides str;
    if ((st = bwd_strides(strides, Shape{B, H, T, D, scale}, str)) != ATTN_OK) return st;
    return bwd_impl(q, k, v, o, lse, dO, dq, dk, dv, B, H, T, D, scale, op, str, workspace,
                    workspace_bytes, stream, li);
}

ATTN_API int attn_bwd(const void *q, const void *k, const void *v, const void *o, const float *lse,
                      const void *dO, void *dq, void *dk, void *dv, int B, int H, int T, int D,
                      float scale, void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    return attn_bwd_ex(q, k, v, o, lse, dO, dq, dk, dv, B, H, T, D, scale, nullptr, nullptr,
                       workspace, workspace_bytes, stream);
}

ATTN_API int attn_bwd_strided(const void *q, const void *k, const void *v, const void *o,
                              const float *lse, const void *dO, void *dq, void *dk, void *dv, int B,
                              int H, int T, int D, float scale, const attn_strides *strides,
                              void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    if (!strides) {
        take_launch_info();
        return ATTN_ERR_NULL;
    }
    return attn_bwd_ex(q, k, v, o, lse, dO, dq, dk, dv, B, H, T, D, scale, strides, nullptr,
                       workspace, workspace_bytes, stream);
}

ATTN_API int attn_fwd_f32_ex(const float *q, const float *k, const float *v, float *o, float *lse,
                             int B, int H, int T, int D, float scale, const attn_options *opts,
                             cudaStream_t stream) {
    LaunchInfo li = take_launch_info();
    Opts op;
    int st0;
    if ((st0 = read_options(opts, op)) != ATTN_OK) return st0;
    if (!q || !k || !v || !o || !lse) return ATTN_ERR_NULL;
    int st = check_shape(B, H, T, D, 128);
    if (st != ATTN_OK) return st;
    if ((st = check_scale(scale)) != ATTN_OK) return st;
    if (!aligned(q, 4) || !aligned(k, 4) || !aligned(v, 4) || !aligned(o, 4) || !aligned(lse, 4))
        return ATTN_ERR_ALIGN;
    if ((st = device_setup(nullptr)) != ATTN_OK) return st;
    cudaError_t e = simt_fwd<float>(q, k, v, o, lse, make_shape(B, H, T, D, scale, op), stream, li);
    return finish(e, li);
}

ATTN_API int attn_fwd_f32(const float *q, const float *k, const float *v, float *o, float *lse,
                          int B, int H, int T, int D, float scale, cudaStream_t stream) {
    return attn_fwd_f32_ex(q, k, v, o, lse, B, H, T, D, scale, nullptr, stream);
}

ATTN_API size_t attn_dropout_mask_bytes(int B, int H, int T) { return mask_bytes_for(B, H, T); }

ATTN_API size_t attn_bwd_f32_workspace_bytes(int B, int H, int T, int D) {
    if (check_shape(B, H, T, D, 128) != ATTN_OK) return 0;
    return round_up((size_t)B * H * T * sizeof(float), 256);
}

ATTN_API int attn_bwd_f32_ex(const float *q, const float *k, const float *v, const float *o,
                             const float *lse, const float *dO, float *dq, float *dk, float *dv,
                             int B, int H, int T, int D, float scale, const attn_options *opts,
                             void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    LaunchInfo li = take_launch_info();
    Opts op;
    int st0;
    if ((st0 = read_options(opts, op)) != ATTN_OK) return st0;
    if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return ATTN_ERR_NULL;
    int st = check_shape(B, H, T, D, 128);
    if (st != ATTN_OK) return st;
    if ((st = check_scale(scale)) != ATTN_OK) return st;
    const void *ptrs[] = {q, k, v, o, lse, dO, dq, dk, dv};
    for (const void *p : ptrs)
        if (!aligned(p, 4)) return ATTN_ERR_ALIGN;
    const size_t need = attn_bwd_f32_workspace_bytes(B, H, T, D);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return ATTN_ERR_WORKSPACE;
    if ((st = device_setup(nullptr)) != ATTN_OK) return st;
    cudaError_t e = simt_bwd<float>(q, k, v, o, lse, dO, dq, dk, dv, static_cast<float *>(workspace),
                                    make_shape(B, H, T, D, scale, op), stream, li);
    return finish(e, li);
}

ATTN_API int attn_bwd_f32(const float *q, const float *k, const float *v, const float *o,
                          const float *lse, const float *dO, float *dq, float *dk, float *dv, int B,
                          int H, int T, int D, float scale, void *workspace, size_t workspace_bytes,
                          cudaStream_t stream) {
    return attn_bwd_f32_ex(q, k, v, o, lse, dO, dq, dk, dv, B, H, T, D, scale, nullptr, workspace,
                           workspace_bytes, stream);
}

ATTN_API int attn_device_error(cudaStream_t stream) {
    int *err = nullptr;
    int st = device_setup(&err);
    if (st != ATTN_OK) return st;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return ATTN_ERR_CUDA;
    int h = 0;
    if (cudaMemcpy(&h, err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return ATTN_ERR_CUDA;
    if (h != 0) {
        const int zero = 0;
        if (cudaMemcpy(err, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
            return ATTN_ERR_CUDA;
        if (h == kErrBounds) return ATTN_ERR_DEVICE_CHECK;
        return h == kErrLayout ? ATTN_ERR_CUDA : ATTN_ERR_TIMEOUT;
    }
    return ATTN_OK;
}

ATTN_API int attn_selftest_wait_timeout(uint32_t polls, cudaStream_t stream) {
    if (polls < 1 || polls > (1u << 22)) return ATTN_ERR_SHAPE;
    int *err = nullptr;
    int st = device_setup(&err);
    if (st != ATTN_OK) return st;
    return selftest_wait_timeout(polls, err, stream) == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

ATTN_API int attn_selftest_device_check(cudaStream_t stream) {
    int *err = nullptr;
    int st = device_setup(&err);
    if (st != ATTN_OK) return st;
    return selftest_failed_check(err, stream) == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

namespace attn {
int bwd_arg_check(const void *q, const void *k, const void *v, const void *o, const float *lse,
                  const void *dO, void *dq, void *dk, void *dv, int B, int H, int T, int D,
                  float scale) {
    return bwd_args(q, k, v, o, lse, dO, dq, dk, dv, B, H, T, D, scale);
}

int device_check() { return device_setup(nullptr); }

void *tensor_map_encoder() {
    static void *fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = p;
    });
    return fn;
}
}  // namespace attn
