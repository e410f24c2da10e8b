// selftest.cu -- exercises the kernels' error paths without a fault:
//  * the bounded wait: a single thread waits on a fresh mbarrier that no one
//    arrives at, gives up after a given number of polls and records the
//    timeout in the device error word, exactly as the attention kernels do
//    when a wait runs out;
//  * the debug build's bounds checks: one check that cannot hold, which the
//    debug build records like any failed check (and the release build
//    compiles away).  Nothing faults or hangs.
#include "internal.h"
#include "sm100.cuh"

namespace attn {
namespace {

__global__ void wait_timeout_kernel(uint32_t polls, int *err) {
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    sm100::mbar_init(&bar, 1);
    sm100::fence_mbar_init();
    for (uint32_t i = 0; i < polls; ++i)
        if (sm100::mbar_try_wait(&bar, 0)) return;  // never completes
    atomicExch(err, kErrTimeout);
}

__global__ void failed_check_kernel(int *err) {
    ATTN_DCHECK(threadIdx.x >= blockDim.x, err);  // never holds; touches no memory
}

}  // namespace

cudaError_t selftest_wait_timeout(uint32_t polls, int *err, cudaStream_t st) {
    wait_timeout_kernel<<<1, 32, 0, st>>>(polls, err);
    return cudaGetLastError();
}

cudaError_t selftest_failed_check(int *err, cudaStream_t st) {
    failed_check_kernel<<<1, 32, 0, st>>>(err);
    return cudaGetLastError();
}

}  // namespace attn
