// attn_bwd_sm100.cu -- causal attention backward on B200 tensor cores (and
// the same attention without the mask).
//
// The pages define the forward only ("How Andrej Karpathy built GPT from 200
// lines of code", sections "Self-Attention: the mathematical trick" [55:20]
// and "Implementing the attention heads (Query, Key, Value)" [1:06:16]-
// [1:17:18]); the backward is its exact derivative for L = sum(O * dO):
//
//   P_ij  = exp(scale q_i.k_j - lse_i)          (recomputed from the saved lse)
//   dV_j  = sum_{i>=j} P_ij dO_i
//   dP_ij = dO_i . v_j,   Delta_i = dO_i . O_i
//   dS_ij = P_ij (dP_ij - Delta_i)
//   dK_j  = scale sum_{i>=j} dS_ij q_i,   dQ_i = scale sum_{j<=i} dS_ij k_j
//
// Three launches on the caller's stream:
//   prep   -Delta_i and -lse_i * log2(e) into tile-padded float32 arrays
//          (negated, so that the main kernels add them: pad rows get 0 and
//          -inf and contribute exactly 0), and the float32 dQ accumulator
//          zeroed;
//   main   one CTA per (128-row key tile j, head), looping over the query
//          tiles i >= j (all query tiles without the mask, where keys past T
//          are zero rows of K and V and so add nothing to dQ); dK_j and dV_j
//          accumulate in TMEM, the partial
//          dQ_i = dS_ij K_j is added into the float32 accumulator by TMA
//          reduce-add;
//   post   dQ = scale * accumulator, rounded to bf16.
//
// Main kernel, sixteen warps in four warpgroups:
//   warp 0      TMA producer: K_j (and V_j) once; Q_i, dO_i (and lse_i,
//               Delta_i) per tile into a 2-stage ring (a stage is released
//               after dK_i, since dQ_i reads neither Q nor dO); without the
//               causal mask and dropout the ring has 3 stages (BwdSmem)
//   warp 1      tcgen05 issuer of S^T and dP^T, TMEM owner
//   warp 2      in the 3-stage layout, V_j and lse_i, Delta_i (their own
//               2-slot ring); idle otherwise
//   warp 3      tcgen05 issuer of dV, dK and dQ
//   warps 4..11 softmax gradient, two warps per TMEM lane quadrant (one per
//               64-query half): per key row (TMEM lane) P^T = exp2(S^T - lse),
//               dS^T = P^T (dP^T - Delta), in packed float32 pairs (two queries
//               per instruction); only the diagonal tile runs the causal test;
//               P^T to TMEM (bf16), dS^T to shared memory (bf16, double
//               buffered)
//   warps 12..15 dQ drain: TMEM -> swizzled shared staging -> TMA reduce-add;
//               at the end of each item the dK and dV epilogue, so that the
//               softmax-gradient warps go straight on to the next item
// The block launches with 512 x 128 registers (the whole register file);
// setmaxnreg then gives the first warpgroup 56, the drain warpgroup 104 and
// the two softmax-gradient warpgroups 176 each (56 + 104 + 2 x 176 = 4 x 128),
// so the elementwise warps keep their 32-element chunks in flight without
// spilling.  The launch checks the build has exactly 128 registers per thread.
//
// Per query tile the score issuer runs S^T = K Q^T and dP^T = V dO^T (M = key
// rows); once the softmax gradient of that tile is ready, the gradient issuer
// runs dV += P^T dO (A from TMEM), dK += dS^T Q and dQ_i = dS K (A read
// MN-major from the same shared dS^T tile).  The next tile's S^T / dP^T are
// issued as soon as the current ones have been read out of TMEM, so they
// overlap the elementwise work; across items the score issuer runs ahead into
// the next item's K/V buffer while the gradients of the last tile are still
// being issued.
//
// With attention dropout (Drop) the keep bit of (query i, key j) is the one
// the forward drew (philox.cuh): the eight lanes holding keys 8g .. 8g+7 each
// load (from a kept mask) or draw the bits of four queries for all eight keys
// and trade them in a three-stage shuffle butterfly; P^T in TMEM keeps only the kept weights (dV is scaled by the keep
// scale at the end), and the kernel forms dS^T / keep_scale =
// P^T (M dP^T - Delta / keep_scale) with Delta / keep_scale from the prep
// kernel, so the keep scale enters once per output element (dK here, dQ in
// the post kernel) instead of once per weight.
//
// TMEM columns: S^T [0,128), dP^T [128,256), dV [256,256+D), dK [256+D,256+2D),
// dQ [256+2D, 256+3D), P^T (bf16 pairs) [256+3D, 256+3D+64).
#include "internal.h"
#include "sm100.cuh"

#include <cudaTypedefs.h>
#include <cstddef>
#include <type_traits>

namespace attn {
namespace {

using namespace sm100;

constexpr int kBT = 128;          // rows per tile (keys and queries)
constexpr int kThreads = 512;     // 16 warps (four warpgroups)
constexpr int kEwThreads = 256;   // softmax-gradient threads (warps 4..11)
constexpr int kEwWarp0 = 4;       // first softmax-gradient warp
constexpr int kDrainWarp0 = 12;   // first dQ-drain warp
constexpr int kRegsLaunch = 128;  // registers per thread at launch
constexpr int kRegsIssue = 56;    // producer / MMA warpgroup after the hand-over
constexpr int kRegsEw = 176;      // softmax-gradient warpgroups
constexpr int kRegsDrain = 104;   // drain warpgroup
static_assert(kRegsIssue + kRegsDrain + 2 * kRegsEw == 4 * kRegsLaunch, "the register split must add up");
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

// Two layouts.  Under the causal mask (short items, 4.5 query tiles on
// average at T = 1024), and with dropout (whose longer softmax-gradient work
// sets the tile period): a 2-stage Q / dO / lse / Delta ring and K, V double
// buffered across items.  Without the mask and without dropout (every item
// runs over all query tiles, and the ring's reload sits on the tile period):
// a 3-stage Q / dO ring, paid for by a single V buffer (its last reader is the
// item's last dP^T) and by lse / Delta in a 2-slot ring of their own, loaded
// with V by warp 2.
template <int D, bool R3>
struct BwdSmem {
    static constexpr int kTileBytes = kBT * D * 2;
    static constexpr int kQS = R3 ? 3 : 2;    // Q / dO stages
    static constexpr int kLS = R3 ? 2 : kQS;  // lse / Delta slots (the Q / dO stages without R3)
    static constexpr int kVB = R3 ? 1 : 2;    // V buffers
    alignas(1024) __nv_bfloat16 q[kQS][kBT * D];
    alignas(1024) __nv_bfloat16 dO[kQS][kBT * D];
    alignas(1024) __nv_bfloat16 k[2][kBT * D];   // double buffered across work items
    alignas(1024) __nv_bfloat16 v[kVB][kBT * D];
    // dS^T, [buffer][query half][key row][64 queries], 128-byte swizzled rows
    alignas(1024) __nv_bfloat16 ds[2][2][kBT * 64];
    // dQ staging for the TMA reduce: one 32-column box [row][32 floats], swizzled
    alignas(1024) float stage[kBT * 32];
    alignas(16) float lse2[kLS][kBT];
    alignas(16) float delta[kLS][kBT];
    uint64_t kv_full[2], kv_empty[2], qdo_full[kQS], qdo_empty[kQS];
    uint64_t v_full, v_empty, ld_full[kLS], ld_empty[kLS];  // the R3 layout's V and lse / Delta
    uint64_t sdp_full, sdp_free, p_ready[2], ds_ready[2], p_free, ds_free[2];
    uint64_t dq_full, dq_free, acc_done, acc_free, drain;
    uint32_t tmem_slot;
    int abort;
};

// Bytes of a layout in use (without the tail padding to its alignment).
template <int D, bool R3>
struct SmemUsed {
    using S = BwdSmem<D, R3>;
    static constexpr size_t value = offsetof(S, abort) + sizeof(int);
};
template <int D, bool R3>
constexpr size_t kSmemUsed = SmemUsed<D, R3>::value;

// ------------------------------------------------------------------ prep

// One thread per (tile-padded row, 16-byte chunk of the row): D/8 threads per
// row read O and dO with coalesced 16-byte loads, Delta_i is reduced across
// them with shuffles, and the same threads zero their part of the dQ
// accumulator row.  Grid: x over blocks of 256 / (D/8) tokens, y over heads
// (striding when there are more heads than grid rows), so a thread finds its
// token and head without integer division.
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16 *__restrict__ o,
                                                       const __nv_bfloat16 *__restrict__ dO,
                                                       const float *__restrict__ lse,
                                                       float *__restrict__ lse2,
                                                       float *__restrict__ delta,
                                                       float *__restrict__ dq_acc, float dscale, int T,
                                                       int Tpad, int BH, int H, TStrides so, TStrides sdo) {
    constexpr int kTpr = D / 8;           // threads per row (a power of two dividing 32)
    constexpr int kRows = 256 / kTpr;     // rows per block
    grid_dep_wait();
    grid_dep_launch();
    const int c = (int)threadIdx.x % kTpr;
    const int t = (int)blockIdx.x * kRows + (int)threadIdx.x / kTpr;
    if (t >= Tpad) return;  // whole rows leave together: the shuffle groups stay complete
    const bool live = t < T;
    for (int bh = (int)blockIdx.y; bh < BH; bh += (int)gridDim.y) {
        const size_t row = (size_t)bh * T + t;
        float acc = 0.f;
        if (live) {
            const long long hb = bh / H, hh = bh % H;
            const uint4 a = reinterpret_cast<const uint4 *>(o + hb * so.b + hh * so.h + (long long)t * so.t)[c];
            const uint4 g = reinterpret_cast<const uint4 *>(dO + hb * sdo.b + hh * sdo.h + (long long)t * sdo.t)[c];
            const __nv_bfloat162 *a2 = reinterpret_cast<const __nv_bfloat162 *>(&a);
            const __nv_bfloat162 *g2 = reinterpret_cast<const __nv_bfloat162 *>(&g);
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const float2 fa = __bfloat1622float2(a2[x]), fg = __bfloat1622float2(g2[x]);
                acc = fmaf(fa.x, fg.x, acc);
                acc = fmaf(fa.y, fg.y, acc);
            }
            float4 *z = reinterpret_cast<float4 *>(dq_acc + row * D + 8 * c);
            z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
            z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int off = kTpr / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (c == 0) {
            const size_t prow = (size_t)bh * Tpad + t;
            delta[prow] = live ? -(acc * dscale) : 0.f;
            lse2[prow] = live ? -(lse[row] * kLog2e) : -INFINITY;
        }
    }
}

// ------------------------------------------------------------------ post

// dQ = scale * accumulator: 8 elements per thread (two 16-byte loads, one
// 16-byte store into the strided dQ view).  Grid as the prep kernel's: x over
// blocks of 256 / (D/8) tokens, y over heads.
template <int D>
__global__ void __launch_bounds__(256) bwd_post_kernel(const float4 *__restrict__ acc,
                                                       __nv_bfloat16 *__restrict__ dq, float scale,
                                                       int T, int BH, int H, TStrides sdq) {
    constexpr int kCpr = D / 8;           // 8-element chunks per row
    constexpr int kRows = 256 / kCpr;
    grid_dep_wait();
    grid_dep_launch();
    const int c = (int)threadIdx.x % kCpr;
    const int t = (int)blockIdx.x * kRows + (int)threadIdx.x / kCpr;
    if (t >= T) return;
    for (int bh = (int)blockIdx.y; bh < BH; bh += (int)gridDim.y) {
        const size_t i = ((size_t)bh * T + t) * kCpr + c;
        const float4 a = acc[2 * i], b = acc[2 * i + 1];
        uint4 r;
        r.x = pack_bf16x2(a.x * scale, a.y * scale);
        r.y = pack_bf16x2(a.z * scale, a.w * scale);
        r.z = pack_bf16x2(b.x * scale, b.y * scale);
        r.w = pack_bf16x2(b.z * scale, b.w * scale);
        const long long hb = bh / H, hh = bh % H;
        *reinterpret_cast<uint4 *>(dq + hb * sdq.b + hh * sdq.h + (long long)t * sdq.t + 8 * c) = r;
    }
}

// With dropout the main kernels compute dS / keep_scale (the keep scale is
// taken out of the per-weight arithmetic): the prep kernel stores
// -Delta / keep_scale, and dK and dQ take keep_scale in their output scale.
inline float delta_scale(const Shape &s) { return s.dropout ? 1.f / s.drop.keep_scale : 1.f; }
inline float dq_scale(const Shape &s) { return s.dropout ? s.scale * s.drop.keep_scale : s.scale; }

// The (token blocks, heads) grid of the prep and post kernels.
template <int D>
dim3 rows_grid(int rows, int BH) {
    constexpr int kRows = 256 / (D / 8);
    return dim3((unsigned)((rows + kRows - 1) / kRows), (unsigned)(BH < 65535 ? BH : 65535));
}

// ------------------------------------------------------------------ main

// The n-th work item of CTA c in a grid of G CTAs over W items ordered
// heaviest first (snake order: c, 2G - 1 - c, 2G + c, ...), or -1.
__device__ __forceinline__ int item_of(int c, int n, int G, int W) {
    const long long w = (long long)n * G + ((n & 1) ? (G - 1 - c) : c);
    return w < W ? (int)w : -1;
}

template <int D, bool Causal, bool Drop>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                    const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                    const __grid_constant__ CUtensorMap tdq, const float *__restrict__ lse2,
                    const float *__restrict__ delta, __nv_bfloat16 *__restrict__ dk,
                    __nv_bfloat16 *__restrict__ dv, const TStrides sdk, const TStrides sdv,
                    int T, int Tpad, int H, int BH, int nt, float scale_log2, float scale,
                    const DropoutParams dp, int *err) {
    constexpr bool R3 = !Causal && !Drop;
    using Smem = BwdSmem<D, R3>;
    constexpr int kQStages = Smem::kQS, kLStages = Smem::kLS;
    constexpr int kRowBytes = D * 2;
    constexpr uint32_t kSwz = (D == 64) ? kSwizzle128B : kSwizzle64B;
    constexpr uint32_t kAtom = 8 * kRowBytes;
    constexpr uint32_t kHalf = kBT * 64 * 2;  // bytes of one 64-query half of dS^T
    extern __shared__ uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                         ~uintptr_t(1023));
    volatile int *abort = &sm.abort;
    if constexpr (R3) {
        // The launch allocates only the padding the layout leaves below the
        // per-block limit: a base that needs more leaves before touching
        // shared memory and reports it.
        uint32_t dyn;
        asm volatile("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
        const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
        if (pad + (uint32_t)kSmemUsed<D, R3> > dyn) {
            if (threadIdx.x == 0) atomicExch(err, kErrLayout);
            return;
        }
    }

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = (int)gridDim.x, cta = (int)blockIdx.x;
    const int W = nt * BH;  // work items; item w is key tile w / BH (tile 0 heaviest) of head w % BH

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sm.kv_full[s], 1);
            mbar_init(&sm.kv_empty[s], 2);  // one commit from each tcgen05 stream
        }
        for (int s = 0; s < kQStages; ++s) {
            mbar_init(&sm.qdo_full[s], 1);
            mbar_init(&sm.qdo_empty[s], 1);
        }
        if constexpr (R3) {
            mbar_init(&sm.v_full, 1);
            mbar_init(&sm.v_empty, 1);  // the score stream, after the item's last dP^T
            for (int s = 0; s < kLStages; ++s) {
                mbar_init(&sm.ld_full[s], 1);
                mbar_init(&sm.ld_empty[s], kEwThreads);
            }
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sm.p_ready[s], kEwThreads);
            mbar_init(&sm.ds_ready[s], kEwThreads);
            mbar_init(&sm.ds_free[s], 1);
        }
        mbar_init(&sm.sdp_full, 1);
        mbar_init(&sm.sdp_free, kEwThreads);
        mbar_init(&sm.p_free, 1);
        mbar_init(&sm.dq_full, 1);
        mbar_init(&sm.dq_free, kBT);
        mbar_init(&sm.acc_done, 1);
        mbar_init(&sm.acc_free, kBT);  // the drain warpgroup
        mbar_init(&sm.drain, 2);  // both tcgen05 streams
        sm.abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(&sm.tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    grid_dep_wait();
    grid_dep_launch();
    const uint32_t tmem = sm.tmem_slot;
    ATTN_DCHECK(tmem == 0u, err);  // all 512 columns, from lane 0 column 0
    const uint32_t tS = tmem, tdP = tmem + 128;
    const uint32_t tdV = tmem + 256, tdK = tmem + 256 + D, tdQ = tmem + 256 + 2 * D;
    const uint32_t tP = tmem + 256 + 3 * D;

    if (warp < kEwWarp0) {
    // ==================================================== first warpgroup
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsIssue));
    if (warp == 0) {
        // ------------------------------------------------ TMA producer (whole warp,
        // one elected lane issues): per item, K and V into buffer n & 1 (once
        // the MMAs of item n - 2 released it), then Q, dO, lse, Delta of its
        // query tiles through the ring (g counts the CTA's tiles).
        if (lane == 0) {
            prefetch_tensormap(&tq);
            prefetch_tensormap(&tk);
            prefetch_tensormap(&tv);
            prefetch_tensormap(&tdo);
        }
        __syncwarp();
        int g = 0, n_items = 0;
        bool ok = true;
        for (int n = 0; ok; ++n) {
            const int w = item_of(cta, n, G, W);
            if (w < 0) break;
            const int kt = w / BH, bh = w % BH, hh = bh % H, bb = bh / H;
            const int q_first = Causal ? kt : 0;
            const int kb = n & 1;
            ATTN_DCHECK(kt >= 0 && kt < nt && bh >= 0 && bh < BH && kt * kBT < T, err);
            if (n >= 2 && !(ok = mbar_wait_warp(&sm.kv_empty[kb], (uint32_t)((n >> 1) - 1) & 1u, err, abort)))
                break;
            if constexpr (R3) {  // V comes from warp 2
                mbar_arrive_expect_tx_e(&sm.kv_full[kb], Smem::kTileBytes);
                tma_load_4d_e(sm.k[kb], &tk, &sm.kv_full[kb], 0, kt * kBT, hh, bb);
            } else {
                mbar_arrive_expect_tx_e(&sm.kv_full[kb], 2 * Smem::kTileBytes);
                tma_load_4d_e(sm.k[kb], &tk, &sm.kv_full[kb], 0, kt * kBT, hh, bb);
                tma_load_4d_e(sm.v[kb], &tv, &sm.kv_full[kb], 0, kt * kBT, hh, bb);
            }
            n_items = n + 1;
            for (int i = q_first; i < nt; ++i, ++g) {
                const int st = g % kQStages;
                if (!(ok = mbar_wait_warp(&sm.qdo_empty[st], (uint32_t)((g / kQStages) & 1) ^ 1u, err, abort))) break;
                mbar_arrive_expect_tx_e(&sm.qdo_full[st], 2 * Smem::kTileBytes + (R3 ? 0 : 2 * kBT * 4));
                tma_load_4d_e(sm.q[st], &tq, &sm.qdo_full[st], 0, i * kBT, hh, bb);
                tma_load_4d_e(sm.dO[st], &tdo, &sm.qdo_full[st], 0, i * kBT, hh, bb);
                if constexpr (!R3) {  // lse and Delta travel with the stage
                    const size_t prow = (size_t)bh * Tpad + (size_t)i * kBT;
                    ATTN_DCHECK(prow + kBT <= (size_t)BH * Tpad && i * kBT < T, err);
                    bulk_load_e(sm.lse2[st], lse2 + prow, kBT * 4, &sm.qdo_full[st]);
                    bulk_load_e(sm.delta[st], delta + prow, kBT * 4, &sm.qdo_full[st]);
                }
            }
        }
        // The last loads issued have landed before the CTA leaves.
        for (int x = (g > kQStages ? g - kQStages : 0); x < g; ++x)
            for (uint32_t m = 0; m < kWaitLimit && !mbar_try_wait(&sm.qdo_full[x % kQStages], (uint32_t)(x / kQStages) & 1u); ++m) {}
        for (int n = (n_items > 2 ? n_items - 2 : 0); n < n_items; ++n)
            for (uint32_t m = 0; m < kWaitLimit && !mbar_try_wait(&sm.kv_full[n & 1], (uint32_t)(n >> 1) & 1u); ++m) {}
    } else if (warp == 2) {
        if constexpr (R3) {
            // ------------------------------------------------ second loader (R3
            // layout): V of each item (single buffer, once the score stream is
            // done with the previous item) and the lse / Delta rows of each
            // tile into their 2-slot ring (once the softmax-gradient warps are
            // done with the tile two back), so the Q / dO producer never waits
            // on either.
            if (lane == 0) prefetch_tensormap(&tv);
            __syncwarp();
            int g = 0, n_v = 0;
            bool ok = true;
            for (int n = 0; ok; ++n) {
                const int w = item_of(cta, n, G, W);
                if (w < 0) break;
                const int kt = w / BH, bh = w % BH;
                if (n >= 1 && !(ok = mbar_wait_warp(&sm.v_empty, (uint32_t)(n - 1) & 1u, err, abort))) break;
                mbar_arrive_expect_tx_e(&sm.v_full, Smem::kTileBytes);
                tma_load_4d_e(sm.v[0], &tv, &sm.v_full, 0, kt * kBT, bh % H, bh / H);
                n_v = n + 1;
                for (int i = Causal ? kt : 0; i < nt; ++i, ++g) {  // the item's query tiles
                    const int sl = g % kLStages;
                    if (g >= kLStages &&
                        !(ok = mbar_wait_warp(&sm.ld_empty[sl], (uint32_t)(g / kLStages - 1) & 1u, err, abort)))
                        break;
                    const size_t prow = (size_t)bh * Tpad + (size_t)i * kBT;
                    ATTN_DCHECK(prow + kBT <= (size_t)BH * Tpad && i * kBT < T, err);
                    mbar_arrive_expect_tx_e(&sm.ld_full[sl], 2 * kBT * 4);
                    bulk_load_e(sm.lse2[sl], lse2 + prow, kBT * 4, &sm.ld_full[sl]);
                    bulk_load_e(sm.delta[sl], delta + prow, kBT * 4, &sm.ld_full[sl]);
                }
            }
            // The last loads issued have landed before the CTA leaves.
            for (int x = (g > kLStages ? g - kLStages : 0); x < g; ++x)
                mbar_wait_drain(&sm.ld_full[x % kLStages], (uint32_t)(x / kLStages) & 1u);
            if (n_v > 0) mbar_wait_drain(&sm.v_full, (uint32_t)(n_v - 1) & 1u);
        }
    } else if (warp == 1 || warp == 3) {
        // ------------------------------------------------ tcgen05 issuers (whole
        // warp, one elected lane issues).  Two independent streams share the
        // tensor core, so that each warp's waits and bookkeeping overlap the
        // other's MMAs: warp 1 issues S^T / dP^T of every tile, warp 3 the
        // gradients dV, dK, dQ.  They touch disjoint TMEM regions, and each
        // barrier is committed by the stream whose MMAs it tracks (a commit
        // covers only its own thread's MMAs); the K/V buffer of an item is
        // released once both streams have committed.
        constexpr uint32_t idS = idesc_bf16(kBT, kBT, 0, 0);  // S^T, dP^T: both K-major
        constexpr uint32_t idKV = idesc_bf16(kBT, D, 0, 1);   // dV, dK: A K-major/TMEM, B MN-major
        constexpr uint32_t idQ = idesc_bf16(kBT, D, 1, 1);    // dQ: A (dS) and B (K) MN-major
        bool ok = true;
        int g = 0;  // the CTA's tiles so far
        for (int n = 0; ok; ++n) {
            const int w = item_of(cta, n, G, W);
            if (w < 0) break;
            const int kt = w / BH;
            const int n_q = nt - (Causal ? kt : 0);
            const int kb = n & 1;
            if (warp == 1) {
                // ---- score stream
                if (!(ok = mbar_wait_warp(&sm.kv_full[kb], (uint32_t)(n >> 1) & 1u, err, abort))) break;
                if (R3 && !(ok = mbar_wait_warp(&sm.v_full, (uint32_t)n & 1u, err, abort))) break;
                // K and V as K-major operands.
                const uint64_t kd_k = smem_desc(smem_u32(sm.k[kb]), 16, kAtom, kSwz);
                const uint64_t vd_k = smem_desc(smem_u32(sm.v[R3 ? 0 : kb]), 16, kAtom, kSwz);
                for (int idx = 0; idx < n_q; ++idx, ++g) {
                    const int st = g % kQStages;
                    if (!(ok = mbar_wait_warp(&sm.qdo_full[st], (uint32_t)(g / kQStages) & 1u, err, abort))) break;
                    if (g >= 1 && !(ok = mbar_wait_warp(&sm.sdp_free, (uint32_t)(g - 1) & 1u, err, abort))) break;
                    tc_fence_after();
                    // S^T = K Q^T and dP^T = V dO^T: D / 16 MMAs each, all
                    // operands K-major (32 bytes per step).
                    const uint64_t qd = smem_desc(smem_u32(sm.q[st]), 16, kAtom, kSwz);
                    const uint64_t dod = smem_desc(smem_u32(sm.dO[st]), 16, kAtom, kSwz);
                    if constexpr (D == 64) {
                        mma_ss_x4<2, 2>(tS, kd_k, qd, idS, 0u);
                        mma_ss_x4<2, 2>(tdP, vd_k, dod, idS, 0u);
                    } else {
                        mma_ss_x2<2, 2>(tS, kd_k, qd, idS, 0u);
                        mma_ss_x2<2, 2>(tdP, vd_k, dod, idS, 0u);
                    }
                    mma_commit_e(&sm.sdp_full);
                }
                if (!ok) break;
                if constexpr (R3) mma_commit_e(&sm.v_empty);  // the item's reads of V
                mma_commit_e(&sm.kv_empty[kb]);  // this stream's reads of the item's K (and V)
            } else {
                // ---- gradient stream.  K needs no wait of its own: the first
                // tile's dS^T exists only after that tile's S^T, which waited
                // for K and V.
                const uint64_t kd_mn = smem_desc(smem_u32(sm.k[kb]), kBT * kRowBytes, kAtom, kSwz);
                for (int p = 0; p < n_q; ++p, ++g) {
                    const int st = g % kQStages, b = g & 1;
                    // MN-major views (16 rows = kRowBytes 16-byte units per K step).
                    const uint64_t qd_mn = smem_desc(smem_u32(sm.q[st]), kBT * kRowBytes, kAtom, kSwz);
                    const uint64_t dod_mn = smem_desc(smem_u32(sm.dO[st]), kBT * kRowBytes, kAtom, kSwz);
                    const uint32_t ds_addr = smem_u32(sm.ds[b][0]);
                    // dS^T read K-major for dK (32 bytes per step within a 64-query
                    // half, the second half kHalf further) and MN-major for dQ (16
                    // key rows of 128 bytes per step, the two query halves kHalf
                    // apart).
                    const uint64_t dsd_k = smem_desc(ds_addr, 16, 1024, kSwizzle128B);
                    const uint64_t dsd_mn = smem_desc(ds_addr, kHalf, 1024, kSwizzle128B);
                    if (!(ok = mbar_wait_warp(&sm.p_ready[b], (uint32_t)(g >> 1) & 1u, err, abort))) break;
                    // The item's first dV / dK overwrite the accumulators: the
                    // previous item's epilogue must have read them.
                    if (p == 0 && n >= 1 &&
                        !(ok = mbar_wait_warp(&sm.acc_free, (uint32_t)(n - 1) & 1u, err, abort)))
                        break;
                    tc_fence_after();
                    // dV += P^T dO: 8 MMAs of K = 16 queries, A from TMEM.
                    mma_ts_x4<kRowBytes>(tdV, tP, dod_mn, idKV, p > 0 ? 1u : 0u);
                    mma_ts_x4<kRowBytes>(tdV, tP + 32, dod_mn + 4 * kRowBytes, idKV, 1u);
                    mma_commit_e(&sm.p_free);
                    if (!(ok = mbar_wait_warp(&sm.ds_ready[b], (uint32_t)(g >> 1) & 1u, err, abort))) break;
                    tc_fence_after();
                    // dK += dS^T Q: 8 MMAs of K = 16 queries.
                    mma_ss_x4<2, kRowBytes>(tdK, dsd_k, qd_mn, idKV, p > 0 ? 1u : 0u);
                    mma_ss_x4<2, kRowBytes>(tdK, dsd_k + (kHalf >> 4), qd_mn + 4 * kRowBytes, idKV, 1u);
                    // Q, dO, lse, Delta of this tile are consumed (its S^T / dP^T
                    // completed before its dS^T existed).
                    mma_commit_e(&sm.qdo_empty[st]);
                    if (g >= 1 && !(ok = mbar_wait_warp(&sm.dq_free, (uint32_t)(g - 1) & 1u, err, abort))) break;
                    tc_fence_after();
                    // dQ_i = dS K: 8 MMAs of K = 16 keys, both operands MN-major.
                    mma_ss_x4<128, kRowBytes>(tdQ, dsd_mn, kd_mn, idQ, 0u);
                    mma_ss_x4<128, kRowBytes>(tdQ, dsd_mn + 4 * 128, kd_mn + 4 * kRowBytes, idQ, 1u);
                    mma_commit_e(&sm.dq_full);
                    mma_commit_e(&sm.ds_free[b]);
                }
                if (!ok) break;
                mma_commit_e(&sm.acc_done);      // this item's dK, dV are complete
                mma_commit_e(&sm.kv_empty[kb]);  // and this stream's reads of its K
            }
        }
        mma_commit_e(&sm.drain);
        mbar_wait_drain(&sm.drain, 0);
    }
    } else if (warp < kDrainWarp0) {
    // ==================================================== softmax-gradient warpgroups
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsEw));
    {
        // ------------------------------------------------ softmax gradient
        const int quad = warp & 3;
        const int half = (warp - kEwWarp0) >> 2;        // query columns [64 half, 64 half + 64)
        const int kr = quad * 32 + lane;                // key row within the tile (TMEM lane)
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const uint32_t sw = (uint32_t)(kr & 7);
        bool ok = true;
        int g0 = 0;  // the CTA's tiles before this item
        for (int n = 0; ok; ++n) {
        const int w = item_of(cta, n, G, W);
        if (w < 0) break;
        const int kt = w / BH, bh = w % BH;
        const int q_first = Causal ? kt : 0;
        const int n_q = nt - q_first;
        for (int idx = 0; idx < n_q; ++idx) {
            const int g = g0 + idx;
            const int st = g % kQStages, b = g & 1;
            const int sl = R3 ? g % kLStages : st;  // lse / Delta slot
            // With a kept dropout mask, this tile's keep bytes are loaded
            // before the wait for S^T, so their latency overlaps it: byte r of
            // kept[c] is keys 8 jg .. +7 of query ib + 8 r (as drawn below).
            uint32_t kept[2] = {0u, 0u};
            if constexpr (Drop) {
                if (dp.mask) {
                    const uint32_t jg = (uint32_t)((kt * kBT + quad * 32 + (lane & ~7)) >> 3);
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const uint32_t ib = (uint32_t)((q_first + idx) * kBT + 64 * half + 32 * c) + (lane & 7);
#pragma unroll
                        for (int r = 0; r < 4; ++r)
                            kept[c] |= (uint32_t)__ldg(dp.mask + philox::mask_at(dp, (uint32_t)bh, jg, ib + 8u * r))
                                       << (8 * r);
                    }
                }
            }
            ok = (!R3 || mbar_wait_warp(&sm.ld_full[sl], (uint32_t)(g / kLStages) & 1u, err, abort)) &&
                 mbar_wait_warp(&sm.sdp_full, (uint32_t)g & 1u, err, abort);
            if (!ok) break;
            tc_fence_after();
            const bool diag = Causal && (idx == 0);
            const uint32_t lse_addr = smem_u32(sm.lse2[sl]), dl_addr = smem_u32(sm.delta[sl]);
            const uint32_t ds_row = smem_u32(sm.ds[b][half]) + (uint32_t)kr * 128;
            ATTN_DCHECK(kr < kBT && (kr + 1) * 128 <= (int)sizeof(sm.ds[0][0]), err);
#pragma unroll
            for (int c = 0; c < 2; ++c) {  // 32 query columns per chunk
                const int q0 = 64 * half + 32 * c;
                uint32_t rs[32], rp[32];
                tmem_ld32(tS + lane_off + q0, rs);
                tmem_ld32(tdP + lane_off + q0, rp);
                tmem_wait_ld();
                reg_fence32(rs);
                reg_fence32(rp);
                if (c == 1) {  // this warp's S^T and dP^T columns are read: the next tile may overwrite them
                    tc_fence_before();
                    mbar_arrive(&sm.sdp_free);
                }
                // keep bit of query q0 + x for this thread's key: bit x of keepm
                uint32_t keepm = 0xFFFFFFFFu;
                if constexpr (Drop) {
                    const uint32_t sub = (uint32_t)(lane & 7);
                    const uint32_t jg = (uint32_t)((kt * kBT + quad * 32 + (lane & ~7)) >> 3);
                    const uint32_t ib = (uint32_t)((q_first + idx) * kBT + q0) + sub;
                    uint32_t wbits = kept[c];  // byte r: keys 8 jg .. +7 of query ib + 8 r
                    if (!dp.mask) {
#pragma unroll
                        for (int r = 0; r < 4; ++r)
                            wbits |= philox::keep_byte_lanes(dp, ib + 8u * r, jg, (uint32_t)bh) << (8 * r);
                    }
                    keepm = philox::transpose_keep_bits(wbits, lane);
                }
                uint32_t pw[16], dw[16];
                const uint64_t sc2 = f2pack(scale_log2, scale_log2);
                // lse2 and delta hold -lse * log2(e) and -Delta' (prep kernel)
                auto elementwise = [&](auto diag_c) {
                    constexpr bool kDiag = decltype(diag_c)::value;
#pragma unroll
                    for (int x = 0; x < 32; x += 4) {
                        const float4 l4 = ld_shared_f4(lse_addr + (q0 + x) * 4);
                        const float4 d4 = ld_shared_f4(dl_addr + (q0 + x) * 4);
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int e = x + 2 * h;
                            const uint64_t nl = h ? f2pack(l4.z, l4.w) : f2pack(l4.x, l4.y);
                            const uint64_t nd = h ? f2pack(d4.z, d4.w) : f2pack(d4.x, d4.y);
                            const float2 t = f2unpack(
                                ffma2(f2pack(__uint_as_float(rs[e]), __uint_as_float(rs[e + 1])), sc2, nl));
                            float p0 = ex2(t.x), p1 = ex2(t.y);
                            if constexpr (kDiag) {  // query before key: masked
                                if (q0 + e < kr) p0 = 0.f;
                                if (q0 + e + 1 < kr) p1 = 0.f;
                            }
                            const uint64_t rp2 = f2pack(__uint_as_float(rp[e]), __uint_as_float(rp[e + 1]));
                            float2 dd;
                            if constexpr (Drop) {
                                // kept weight p~ = keep ? p : 0; dS / keep_scale = p~ dP - p Delta'
                                const float k0 = (keepm >> e) & 1u ? p0 : 0.f;
                                const float k1 = (keepm >> (e + 1)) & 1u ? p1 : 0.f;
                                dd = f2unpack(ffma2(f2pack(p0, p1), nd, fmul2(f2pack(k0, k1), rp2)));
                                pw[e / 2] = pack_bf16x2(k0, k1);
                            } else {
                                dd = f2unpack(fmul2(f2pack(p0, p1), fadd2(rp2, nd)));
                                pw[e / 2] = pack_bf16x2(p0, p1);
                            }
                            dw[e / 2] = pack_bf16x2(dd.x, dd.y);
                        }
                    }
                };
                if (diag)
                    elementwise(std::true_type{});
                else
                    elementwise(std::false_type{});
                if (c == 0) {
                    // P^T in TMEM is free once dV of the previous tile completed;
                    // this dS^T buffer once dK/dQ of two tiles ago completed.
                    bool wt = true;
                    if (g >= 1) wt = mbar_wait(&sm.p_free, (uint32_t)(g - 1) & 1u, err, abort);
                    wt = wt && mbar_wait(&sm.ds_free[b], (uint32_t)((g >> 1) & 1) ^ 1u, err, abort);
                    ok = __all_sync(0xffffffffu, wt);
                    if (!ok) break;
                    tc_fence_after();
                }
                tmem_st16(tP + lane_off + q0 / 2, pw);
#pragma unroll
                for (int u = 0; u < 4; ++u) {  // four 16-byte chunks = 32 queries
                    const uint32_t g = 4 * c + u;          // 8-query group within this half
                    st_shared_v4(ds_row + ((g ^ sw) << 4), dw[4 * u], dw[4 * u + 1], dw[4 * u + 2],
                                 dw[4 * u + 3]);
                }
            }
            if (!ok) break;
            if constexpr (R3) mbar_arrive(&sm.ld_empty[sl]);  // this tile's lse / Delta are read
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&sm.p_ready[b]);
            mbar_arrive(&sm.ds_ready[b]);
        }
        g0 += n_q;
        }
    }
    } else {
    // ==================================================== drain warpgroup
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsDrain));
    {
        // ------------------------------------------------ dQ drain
        const int quad = warp & 3;
        const int qr = quad * 32 + lane;                // query row within the tile
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const bool leader = (warp == kDrainWarp0 && lane == 0);
        const uint32_t sw = (uint32_t)(qr & 7);
        int g = 0;
        bool ok = true;
        for (int n = 0; ok; ++n) {
        const int w = item_of(cta, n, G, W);
        if (w < 0) break;
        const int kt = w / BH, bh = w % BH;
        const int q_first = Causal ? kt : 0;
        for (int idx = 0; idx < nt - q_first; ++idx, ++g) {
            ok = __all_sync(0xffffffffu, mbar_wait(&sm.dq_full, (uint32_t)g & 1u, err, abort));
            if (!ok) break;
            tc_fence_after();
            uint32_t r[D / 32][32];
#pragma unroll
            for (int h = 0; h < D / 32; ++h) tmem_ld32(tdQ + lane_off + 32 * h, r[h]);
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < D / 32; ++h) reg_fence32(r[h]);
            tc_fence_before();
            mbar_arrive(&sm.dq_free);
#pragma unroll
            for (int h = 0; h < D / 32; ++h) {
                if (leader) bulk_wait_read_all();  // the previous reduce has read the staging box
                named_bar_sync(1, 128);
                const uint32_t row = smem_u32(sm.stage) + (uint32_t)qr * 128;
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    st_shared_v4(row + ((u ^ sw) << 4), r[h][4 * u], r[h][4 * u + 1], r[h][4 * u + 2],
                                 r[h][4 * u + 3]);
                fence_proxy_async_smem();
                named_bar_sync(1, 128);
                if (leader) {
                    ATTN_DCHECK((q_first + idx) * kBT < T && bh < BH, err);
                    tma_reduce_add_3d(&tdq, sm.stage, 32 * h, (q_first + idx) * kBT, bh);
                    bulk_commit();
                }
            }
        }
        if (!ok) break;
        // ---- epilogue of the item: dK (times scale) and dV (times the keep
        // scale) leave TMEM as bf16 rows (TMEM lane = key row); then the
        // accumulators are free for the next item's first dV / dK MMAs
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.acc_done, (uint32_t)n & 1u, err, abort));
        if (!ok) break;
        tc_fence_after();
        {
            const int hh = bh % H, bb = bh / H;
            const int t = kt * kBT + qr;
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                const uint32_t src = which == 0 ? tdK : tdV;
                const float mul = Drop ? (which == 0 ? scale : 1.f) * dp.keep_scale : (which == 0 ? scale : 1.f);
                const TStrides so = which == 0 ? sdk : sdv;
                __nv_bfloat16 *out = (which == 0 ? dk : dv) + (long long)bb * so.b +
                                     (long long)hh * so.h + (long long)t * so.t;
                uint32_t r[D / 32][32];
#pragma unroll
                for (int h = 0; h < D / 32; ++h) tmem_ld32(src + lane_off + 32 * h, r[h]);
                tmem_wait_ld();
#pragma unroll
                for (int h = 0; h < D / 32; ++h) reg_fence32(r[h]);
                if (t < T) {
#pragma unroll
                    for (int h = 0; h < D / 32; ++h) {
                        uint4 *dst = reinterpret_cast<uint4 *>(out + 32 * h);
#pragma unroll
                        for (int x = 0; x < 4; ++x) {
                            uint4 w4;
                            w4.x = pack_bf16x2(__uint_as_float(r[h][8 * x + 0]) * mul, __uint_as_float(r[h][8 * x + 1]) * mul);
                            w4.y = pack_bf16x2(__uint_as_float(r[h][8 * x + 2]) * mul, __uint_as_float(r[h][8 * x + 3]) * mul);
                            w4.z = pack_bf16x2(__uint_as_float(r[h][8 * x + 4]) * mul, __uint_as_float(r[h][8 * x + 5]) * mul);
                            w4.w = pack_bf16x2(__uint_as_float(r[h][8 * x + 6]) * mul, __uint_as_float(r[h][8 * x + 7]) * mul);
                            dst[x] = w4;
                        }
                    }
                }
            }
        }
        tc_fence_before();
        mbar_arrive(&sm.acc_free);
        }
        if (leader) bulk_wait_all();
    }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Encodes a [BH, T, D] tensor (bf16 or float32) as a 3-D TMA map.
cudaError_t make_map(CUtensorMap *map, const void *ptr, int BH, int T, int D, bool f32, int box_x) {
    auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
    if (!enc) return cudaErrorInitializationError;
    const int es = f32 ? 4 : 2;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)T, (cuuint64_t)BH};
    const cuuint64_t strides[2] = {(cuuint64_t)D * es, (cuuint64_t)T * D * es};
    const cuuint32_t box[3] = {(cuuint32_t)box_x, (cuuint32_t)kBT, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapSwizzle swz = (box_x * es == 128) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    const CUresult r = enc(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                           const_cast<void *>(ptr), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int D, bool Causal, bool Drop>
cudaError_t launch_bwd(const __nv_bfloat16 *q, const __nv_bfloat16 *k, const __nv_bfloat16 *v,
                       const __nv_bfloat16 *o, const float *lse, const __nv_bfloat16 *dO,
                       __nv_bfloat16 *dq, __nv_bfloat16 *dk, __nv_bfloat16 *dv, float *dq_acc,
                       float *lse2, float *delta, Shape s, const BwdStrides &str,
                       int *err, cudaStream_t st, LaunchInfo &li) {
    const int BH = s.B * s.H;
    const int nt = (s.T + kBT - 1) / kBT;
    const int Tpad = nt * kBT;
    const long long items = (long long)nt * BH;
    int dev = 0, sms = 0;
    cudaError_t e0;
    if ((e0 = cudaGetDevice(&dev)) != cudaSuccess) return e0;
    if ((e0 = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e0;
    // Persistent grid: one CTA per SM over the (key tile, head) items.
    const long long blocks = items < sms ? items : sms;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    CUtensorMap mq, mk, mv, mdo, mdq;
    cudaError_t e;
    if ((e = make_map_bf16(&mq, q, s, str.q)) != cudaSuccess) return e;
    if ((e = make_map_bf16(&mk, k, s, str.k)) != cudaSuccess) return e;
    if ((e = make_map_bf16(&mv, v, s, str.v)) != cudaSuccess) return e;
    if ((e = make_map_bf16(&mdo, dO, s, str.dO)) != cudaSuccess) return e;
    if ((e = make_map(&mdq, dq_acc, BH, s.T, D, true, 32)) != cudaSuccess) return e;

    if ((e = launch_pdl(bwd_prep_kernel<D>, rows_grid<D>(Tpad, BH), dim3(256), 0, st, o, dO, lse, lse2,
                        delta, dq_acc, delta_scale(s), s.T, Tpad, BH, s.H, str.o, str.dO)) != cudaSuccess)
        return e;
    li.kernels += 1;

    // The layout plus the padding a 1024-byte alignment of the base may need;
    // the R3 layout caps that at the per-block limit (the kernel checks the
    // base it gets).
    constexpr bool R3 = !Causal && !Drop;
    size_t smem = sizeof(BwdSmem<D, R3>) + 1024;
    if constexpr (R3) {
        int smem_max = 0;
        if ((e = cudaDeviceGetAttribute(&smem_max, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
            return e;
        smem = kSmemUsed<D, R3> + 1023;
        if (smem > (size_t)smem_max) smem = (size_t)smem_max;
        if (kSmemUsed<D, R3> > smem) return cudaErrorInvalidConfiguration;
    }
    {
        // The setmaxnreg hand-over assumes the block holds 512 x 128
        // registers; any other build would make the increases wait forever.
        static int checked = 0;  // 0 unknown, 1 good, -1 bad
        if (checked == 0) {
            cudaFuncAttributes fa;
            if ((e = cudaFuncGetAttributes(&fa, bwd_main_kernel<D, Causal, Drop>)) != cudaSuccess) return e;
            checked = (fa.numRegs == kRegsLaunch) ? 1 : -1;
        }
        if (checked < 0) return cudaErrorInvalidConfiguration;
    }
    static std::atomic<unsigned long long> smem_set{0};
    if ((e = set_max_smem_once(reinterpret_cast<const void *>(bwd_main_kernel<D, Causal, Drop>), smem, dev,
                               smem_set)) != cudaSuccess)
        return e;
    if ((e = mark_main_start(li, st)) != cudaSuccess) return e;
    if ((e = launch_pdl(bwd_main_kernel<D, Causal, Drop>, dim3((unsigned)blocks), dim3(kThreads), smem, st,
                        mq, mk, mv, mdo, mdq, lse2, delta, dk, dv, str.dk, str.dv, s.T, Tpad, s.H, BH,
                        nt, s.scale * kLog2e, s.scale, s.drop, err)) != cudaSuccess)
        return e;
    li.kernels += 1;
    if ((e = mark_main_end(li, st)) != cudaSuccess) return e;

    if ((e = launch_pdl(bwd_post_kernel<D>, rows_grid<D>(s.T, BH), dim3(256), 0, st,
                        reinterpret_cast<const float4 *>(dq_acc), dq, dq_scale(s), s.T, BH, s.H, str.dq)) !=
        cudaSuccess)
        return e;
    li.kernels += 1;
    return cudaSuccess;
}

// head_dim 128: the same prep and post kernels around the D = 128 main kernel
// (attn_bwd128_sm100.cu).
cudaError_t launch_bwd128(const __nv_bfloat16 *q, const __nv_bfloat16 *k, const __nv_bfloat16 *v,
                          const __nv_bfloat16 *o, const float *lse, const __nv_bfloat16 *dO,
                          __nv_bfloat16 *dq, __nv_bfloat16 *dk, __nv_bfloat16 *dv, float *dq_acc,
                          float *lse2, float *delta, Shape s, const BwdStrides &str,
                          int *err, cudaStream_t st, LaunchInfo &li) {
    constexpr int D = 128;
    const int BH = s.B * s.H;
    const int Tpad = (s.T + kBT - 1) / kBT * kBT;
    cudaError_t e;
    if ((e = launch_pdl(bwd_prep_kernel<D>, rows_grid<D>(Tpad, BH), dim3(256), 0, st, o, dO, lse, lse2,
                        delta, dq_acc, delta_scale(s), s.T, Tpad, BH, s.H, str.o, str.dO)) != cudaSuccess)
        return e;
    li.kernels += 1;
    if ((e = sm100_bwd128_main(q, k, v, dO, dk, dv, dq_acc, lse2, delta, s, str, err, st, li)) !=
        cudaSuccess)
        return e;
    if ((e = launch_pdl(bwd_post_kernel<D>, rows_grid<D>(s.T, BH), dim3(256), 0, st,
                        reinterpret_cast<const float4 *>(dq_acc), dq, dq_scale(s), s.T, BH, s.H, str.dq)) !=
        cudaSuccess)
        return e;
    li.kernels += 1;
    return cudaSuccess;
}

}  // namespace

cudaError_t sm100_bwd(const __nv_bfloat16 *q, const __nv_bfloat16 *k, const __nv_bfloat16 *v,
                      const __nv_bfloat16 *o, const float *lse, const __nv_bfloat16 *dO,
                      __nv_bfloat16 *dq, __nv_bfloat16 *dk, __nv_bfloat16 *dv, float *dq_acc,
                      float *lse2, float *delta, Shape s, const BwdStrides &str,
                      int *err, cudaStream_t st, LaunchInfo &li) {
#define ATTN_BWD_CASE(DD, C, R)                                                                    \
    if (s.D == DD && (s.causal != 0) == C && s.dropout == R)                                       \
        return launch_bwd<DD, C, R>(q, k, v, o, lse, dO, dq, dk, dv, dq_acc, lse2, delta, s, str, err, \
                                    st, li);
    ATTN_BWD_CASE(64, true, false)
    ATTN_BWD_CASE(64, false, false)
    ATTN_BWD_CASE(64, true, true)
    ATTN_BWD_CASE(64, false, true)
    ATTN_BWD_CASE(32, true, false)
    ATTN_BWD_CASE(32, false, false)
    ATTN_BWD_CASE(32, true, true)
    ATTN_BWD_CASE(32, false, true)
#undef ATTN_BWD_CASE
    if (s.D == 128)
        return launch_bwd128(q, k, v, o, lse, dO, dq, dk, dv, dq_acc, lse2, delta, s, str, err, st, li);
    return cudaErrorInvalidValue;
}

}  // namespace attn
