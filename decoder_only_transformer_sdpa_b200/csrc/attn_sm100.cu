// attn_sm100.cu -- bf16 backward entry (provisional: CUDA-core kernels while
// the tensor-core backward is brought up).
#include "internal.h"

namespace attn {

cudaError_t sm100_bwd(const __nv_bfloat16 *q, const __nv_bfloat16 *k, const __nv_bfloat16 *v,
                      const __nv_bfloat16 *o, const float *lse, const __nv_bfloat16 *dO,
                      __nv_bfloat16 *dq, __nv_bfloat16 *dk, __nv_bfloat16 *dv, float *dq_acc,
                      float *delta, Shape s, int *err, cudaStream_t st, LaunchInfo &li) {
    (void)err;
    (void)dq_acc;
    return simt_bwd<__nv_bfloat16>(q, k, v, o, lse, dO, dq, dk, dv, delta, s, st, li);
}

}  // namespace attn
