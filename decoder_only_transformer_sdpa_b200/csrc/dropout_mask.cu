// dropout_mask.cu -- draws the kept attention-dropout mask ahead of the
// forward.
//
// When the caller lends a mask buffer (attn_options.dropout_mask), the keep
// bits are drawn once, here, by a full-occupancy kernel that does nothing else,
// and the tcgen05 forward and backward both load them.  Drawing them inside the
// forward instead more than doubles the instructions its softmax warps issue
// (the generator takes about ten per weight), and with two CTAs per SM and a
// full register file no other warp can take that work over.  Here the
// generator runs with every warp slot of the SM filled, and the forward only
// adds a 16-byte load per row and key tile.
//
// The bits are those of philox.cuh (Philox4x32-10, counter (i, key group, bh,
// offset), key = seed), laid out as philox.cuh describes; only the tiles the
// kernels visit are drawn: every (query tile, key tile) pair without the
// causal mask, the pairs with key tile <= query tile under it.
#include "internal.h"
#include "sm100.cuh"

namespace attn {
namespace {

using namespace sm100;

constexpr int kRows = 128;   // query rows of a tile: one per thread
constexpr int kGroups = 16;  // 8-key groups of a 128-key tile: one keep byte each

// One block per (head, query tile, key tile); thread r draws the 16 keep bytes
// of query row (query tile) * 128 + r against the key tile and stores them
// with one 16-byte store.
template <bool Causal>
__global__ void __launch_bounds__(kRows) mask_kernel(const DropoutParams dp, int ntiles, int *err) {
    const long long blk = blockIdx.x;
    const int j = (int)(blk % ntiles);
    const int qt = (int)((blk / ntiles) % ntiles);
    const uint32_t bh = (uint32_t)(blk / ((long long)ntiles * ntiles));
    grid_dep_wait();
    grid_dep_launch();
    if (Causal && j > qt) return;  // above the diagonal: never visited
    const uint32_t ti = (uint32_t)(qt * kRows + (int)threadIdx.x);
    ATTN_DCHECK(ti < dp.mask_ld && (uint32_t)(j + 1) * kGroups <= (dp.mask_ld >> 3), err);
    uint32_t w[kGroups / 4];
#pragma unroll
    for (int q = 0; q < kGroups / 4; ++q) {
        uint32_t x = 0u;
#pragma unroll
        for (int e = 0; e < 4; ++e)
            x |= philox::keep_byte(dp, ti, (uint32_t)(j * kGroups + 4 * q + e), bh) << (8 * e);
        w[q] = x;
    }
    *reinterpret_cast<uint4 *>(dp.mask + philox::mask_at(dp, bh, (uint32_t)(j * kGroups), ti)) =
        make_uint4(w[0], w[1], w[2], w[3]);
}

}  // namespace

cudaError_t draw_dropout_mask(const Shape &s, int *err, cudaStream_t st, LaunchInfo &li) {
    if (!s.dropout || !s.drop.mask) return cudaErrorInvalidValue;
    const int ntiles = (s.T + kRows - 1) / kRows;
    if (s.drop.mask_ld != (uint32_t)ntiles * kRows) return cudaErrorInvalidValue;
    const long long blocks = (long long)s.B * s.H * ntiles * ntiles;
    if (blocks < 1 || blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const cudaError_t e =
        s.causal ? launch_pdl(mask_kernel<true>, dim3((unsigned)blocks), dim3(kRows), 0, st, s.drop, ntiles, err)
                 : launch_pdl(mask_kernel<false>, dim3((unsigned)blocks), dim3(kRows), 0, st, s.drop, ntiles, err);
    if (e == cudaSuccess) li.kernels += 1;
    return e;
}

}  // namespace attn
