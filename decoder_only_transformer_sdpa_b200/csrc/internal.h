// internal.h -- declarations shared by the library's translation units (not
// part of the public ABI; every symbol here has hidden visibility).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

#include "philox.cuh"

namespace attn {

// Upper bound on the polls of any in-kernel wait (mbarrier or flag).  A wait
// that runs out sets the device error word to kErrTimeout and the kernel
// leaves by its normal exit path.  A poll costs from ~20 ns up to ~1 us
// (try_wait may suspend the thread briefly), so a stuck wait ends after
// roughly 0.1 s to a few seconds; legitimate waits last microseconds.
constexpr uint32_t kWaitLimit = 1u << 22;
constexpr int kErrTimeout = 1;
// The debug build (-DATTN_DEVICE_CHECKS) checks tile coordinates, TMEM column
// ranges and shared-memory offsets inside the kernels; a failed check records
// kErrBounds in the device error word and the kernel carries on (nothing
// traps).  The release build compiles the checks away.
constexpr int kErrBounds = 3;
// A kernel whose tile layout leaves less alignment padding than its dynamic
// shared-memory base needs records kErrLayout and leaves before touching
// shared memory.
constexpr int kErrLayout = 4;
#ifdef ATTN_DEVICE_CHECKS
#define ATTN_DCHECK(cond, err)                           \
    do {                                                 \
        if (!(cond)) atomicExch((err), ::attn::kErrBounds); \
    } while (0)
#else
#define ATTN_DCHECK(cond, err) \
    do {                       \
    } while (0)
#endif

struct Shape {
    int B, H, T, D;
    float scale;
    int causal = 1;        // 1: key j visible to query i iff j <= i; 0: all keys visible
    bool dropout = false;  // attention dropout on the weights (drop.thr > 0)
    DropoutParams drop{};
};

// Element strides of a [B, H, T, D] view (the d stride is 1).  Contiguous
// tensors have {H*T*D, T*D, D}; q/k/v viewed inside a [B, T, 3*H*D] c_attn
// output have {T*3*H*D, D, 3*H*D}.
struct TStrides {
    long long b, h, t;
};
inline TStrides contiguous_strides(const Shape &s) {
    return TStrides{(long long)s.H * s.T * s.D, (long long)s.T * s.D, (long long)s.D};
}
struct FwdStrides {
    TStrides q, k, v, o;
};
struct BwdStrides {
    TStrides q, k, v, o, dO, dq, dk, dv;
};

// Builds a 4-D TMA map over a bf16 [B, H, T, D] view with the given element
// strides: dimensions (D, T, H, B), box (min(D, 64), 128, 1, 1), swizzle
// matching the box row (128 B at D >= 64, 64 B at D = 32); D = 128 tiles load
// as two 64-column slabs.
cudaError_t make_map_bf16(void *map, const void *ptr, const Shape &s, const TStrides &st);

// Per-call bookkeeping: kernels enqueued, and the optional event pair to
// record around the call's main kernel (see attn_profile_next_call).
struct LaunchInfo {
    int kernels = 0;
    cudaEvent_t main_start = nullptr;
    cudaEvent_t main_end = nullptr;
};

// Launches `kernel` with programmatic stream serialisation: its CTAs may be
// scheduled, and run their prologue (barrier init, TMEM allocation), while the
// previous grid in the stream drains.  Every kernel launched this way calls
// grid_dep_wait() before touching global memory.
template <typename... Params, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...);
}

// Raises `kernel`'s dynamic shared-memory limit to `bytes` on device `dev`
// once per call site: the attribute lasts for the process, so later calls on
// a device whose bit is set in `done` skip the runtime call.
inline cudaError_t set_max_smem_once(const void *kernel, size_t bytes, int dev,
                                     std::atomic<unsigned long long> &done) {
    const unsigned long long bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
    if (bit && (done.load(std::memory_order_relaxed) & bit)) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_relaxed);
    return e;
}

// Records li.main_start / li.main_end (when armed) around a main kernel.
inline cudaError_t mark_main_start(const LaunchInfo &li, cudaStream_t st) {
    return li.main_start ? cudaEventRecord(li.main_start, st) : cudaSuccess;
}
inline cudaError_t mark_main_end(const LaunchInfo &li, cudaStream_t st) {
    return li.main_end ? cudaEventRecord(li.main_end, st) : cudaSuccess;
}

// ---- decode: the Tq newest queries against the keys/values of Tk tokens
constexpr int kMaxDecodeQueries = 16;
struct DecodeShape {
    int B, H, Tq, Tk, D;
    float scale;
};
// bf16, D in {32, 64}; strides of q, k, v, o (k, v over Tk tokens; q, o over Tq).
cudaError_t sm100_decode(const __nv_bfloat16 *q, const __nv_bfloat16 *k, const __nv_bfloat16 *v,
                         __nv_bfloat16 *o, float *lse, const DecodeShape &s, const FwdStrides &str,
                         int *err, cudaStream_t st, LaunchInfo &li);

// ---- SIMT kernels (float32 math on CUDA cores), element type float or bf16
template <typename T>
cudaError_t simt_fwd(const T *q, const T *k, const T *v, T *o, float *lse, Shape s,
                     cudaStream_t st, LaunchInfo &li);
template <typename T>
cudaError_t simt_bwd(const T *q, const T *k, const T *v, const T *o, const float *lse,
                     const T *dO, T *dq, T *dk, T *dv, float *delta, Shape s,
                     cudaStream_t st, LaunchInfo &li);

// ---- tcgen05 / TMA kernels for bf16, D in {32, 64, 128}
cudaError_t sm100_fwd(const __nv_bfloat16 *q, const __nv_bfloat16 *k, const __nv_bfloat16 *v,
                      __nv_bfloat16 *o, float *lse, Shape s, const FwdStrides &str, int *err,
                      cudaStream_t st, LaunchInfo &li);
cudaError_t sm100_bwd(const __nv_bfloat16 *q, const __nv_bfloat16 *k, const __nv_bfloat16 *v,
                      const __nv_bfloat16 *o, const float *lse, const __nv_bfloat16 *dO,
                      __nv_bfloat16 *dq, __nv_bfloat16 *dk, __nv_bfloat16 *dv,
                      float *dq_acc, float *lse2, float *delta, Shape s, const BwdStrides &str,
                      int *err, cudaStream_t st, LaunchInfo &li);

// Draws the keep bytes of every tile the bf16 kernels visit into s.drop.mask
// (laid out as philox.cuh describes); launched ahead of the forward when the
// caller lends a mask buffer.
cudaError_t draw_dropout_mask(const Shape &s, int *err, cudaStream_t st, LaunchInfo &li);

// The backward main kernel at D = 128 (prep and post kernels run around it in
// sm100_bwd).
cudaError_t sm100_bwd128_main(const __nv_bfloat16 *q, const __nv_bfloat16 *k,
                              const __nv_bfloat16 *v, const __nv_bfloat16 *dO, __nv_bfloat16 *dk,
                              __nv_bfloat16 *dv, float *dq_acc, const float *lse2,
                              const float *delta, const Shape &s, const BwdStrides &str, int *err,
                              cudaStream_t st, LaunchInfo &li);

// Workspace layout of the bf16 backward (offsets in bytes, each 256-aligned):
// float32 dQ accumulator [B*H*T*D], then log2-scaled lse and Delta, each
// [B*H][T padded to a multiple of 128].
struct BwdWorkspace {
    size_t dq_acc, lse2, delta, total;
};
inline BwdWorkspace bwd_workspace_layout(int B, int H, int T, int D) {
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    const size_t rows = (size_t)B * H * T;
    const size_t prows = (size_t)B * H * (size_t)((T + 127) / 128 * 128);
    BwdWorkspace w;
    w.dq_acc = 0;
    w.lse2 = up(rows * D * sizeof(float));
    w.delta = w.lse2 + up(prows * sizeof(float));
    w.total = w.delta + up(prows * sizeof(float));
    return w;
}

// Launches one thread that waits on an mbarrier nobody arrives at, polling at
// most `polls` times, so the timeout path can be exercised without a fault.
cudaError_t selftest_wait_timeout(uint32_t polls, int *err, cudaStream_t st);
// Runs one device-side bounds check that cannot hold (recorded by the debug
// build, compiled away by the release build).
cudaError_t selftest_failed_check(int *err, cudaStream_t st);

// The argument checks attn_bwd runs before it looks at its workspace
// (pointers, shape, head_dim, scale, alignment, in that order): ATTN_OK or the
// status attn_bwd returns for these arguments.
int bwd_arg_check(const void *q, const void *k, const void *v, const void *o, const float *lse,
                  const void *dO, void *dq, void *dk, void *dv, int B, int H, int T, int D,
                  float scale);
// The device check attn_bwd runs after its workspace check: ATTN_OK on an
// sm_100 device, ATTN_ERR_DEVICE on another, ATTN_ERR_CUDA when the runtime
// cannot say.
int device_check();

// Driver entry point for cuTensorMapEncodeTiled, resolved once at run time
// through the runtime (so the library does not link libcuda directly).
void *tensor_map_encoder();

}  // namespace attn
