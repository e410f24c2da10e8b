// attn_bwd_noalloc.cu -- attn_bwd_noalloc: the bf16 backward for callers that
// cannot allocate device memory themselves.
//
// Some callers of this library have no way to obtain scratch memory: plain C
// hosts with no device allocator of their own, plug-ins inside a framework
// that owns every byte of device memory through its own pool and forbids
// cudaMalloc, and latency-critical loops where a cudaMalloc (which can
// synchronise the device) is not acceptable.  For them this entry point runs
// the same backward as attn_bwd, with its scratch (the float32 dQ accumulator,
// the padded lse and Delta) taken from a fixed array compiled into the
// library instead of a caller-supplied workspace.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds its ATTN_NOALLOC_SCRATCH_BYTES until the process exits.  All
// calls on a device share it and it keeps the last call's contents; the
// backward clears what must start at zero (the dQ accumulator) on every call.
// Calls that overlap on the GPU (different streams, or different host
// threads, on the same device) race on the array and must be serialised by
// the caller.
#include "../../include/attn.h"
#include "internal.h"

#include <mutex>

#define ATTN_API extern "C" __attribute__((visibility("default")))

namespace attn {
namespace {

static_assert(ATTN_NOALLOC_SCRATCH_BYTES % 256 == 0, "scratch size must keep 256-byte alignment");

static __device__ __align__(256) unsigned char g_noalloc_scratch[ATTN_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxDevices];

// Device address of the scratch array on the current device.  In host code
// the array's name only stands for it; the address must be looked up once per
// device, with that device current, before any kernel can be given it.
int scratch_on_current_device(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();  // leave no stale error for a later launch check to find
            return ATTN_ERR_CUDA;
        }
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return ATTN_OK;
}

}  // namespace
}  // namespace attn

ATTN_API int attn_bwd_noalloc(const void *q, const void *k, const void *v, const void *o,
                              const float *lse, const void *dO, void *dq, void *dk, void *dv,
                              int B, int H, int T, int D, float scale, cudaStream_t stream) {
    // The statuses and their order are attn_bwd's: argument errors, then the
    // scratch size (attn_bwd's workspace check), then the device; the scratch
    // address is looked up only on a supported device.
    int st = attn::bwd_arg_check(q, k, v, o, lse, dO, dq, dk, dv, B, H, T, D, scale);
    if (st != ATTN_OK) return st;
    const size_t need = attn_bwd_workspace_bytes(B, H, T, D);
    if (need == 0 || need > (size_t)ATTN_NOALLOC_SCRATCH_BYTES) return ATTN_ERR_WORKSPACE;
    if ((st = attn::device_check()) != ATTN_OK) return st;
    void *scratch = nullptr;
    if ((st = attn::scratch_on_current_device(&scratch)) != ATTN_OK) return st;
    return attn_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, T, D, scale, scratch,
                    (size_t)ATTN_NOALLOC_SCRATCH_BYTES, stream);
}
