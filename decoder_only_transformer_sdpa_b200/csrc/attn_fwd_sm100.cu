// attn_fwd_sm100.cu -- causal attention forward on B200 tensor cores (and the
// same attention without the mask).
//
// Computes, per head, O = softmax(scale * Q K^T with the upper triangle at
// -inf) V and the natural-log row log-sum-exp ("How Andrej Karpathy built GPT
// from 200 lines of code": section "Implementing the attention heads (Query,
// Key, Value)" [1:06:16]-[1:17:18] for the scaled query-key affinities and
// the value aggregation; section "Self-Attention: the mathematical trick"
// [55:20] for the -inf upper triangle and the softmax).
//
// Persistent kernel: two CTAs per SM at D <= 64 (256 TMEM columns, ~97 KB
// shared memory and <= 168 registers each), so one CTA's softmax overlaps the
// other's MMAs and both keep the exp unit busy; one CTA per SM at D = 128
// (320 TMEM columns, 192 KB of tiles).  Rows of D = 128 are kept as two
// 64-column slabs with the 128-byte swizzle; the S MMAs run over both slabs
// and the PV MMA's N = 128 spans them.  Work items are (128-row query tile,
// head) pairs ordered heaviest first (most key tiles under the causal mask);
// CTA c takes items c, 2G-1-c, 2G+c, ... (a snake over rounds of G = grid size
// items), which balances the causal work as well as greedy longest-first.
// Barrier phases run on across items, so the next item's Q and K/V tiles
// stream in and its first S MMA issues while the current item drains.
// Eight warps in two warpgroups:
//   warp 0      TMA producer: Q of each item into a 2-buffer ring, K_j / V_j
//               tiles into a 2-stage ring (at D <= 64, K one tile ahead of V)
//   warp 1      tcgen05 issuer of S = Q K_j^T into TMEM; owns the TMEM
//               allocation.  S of the next tile is issued as soon as the
//               softmax has read the current one.
//   warp 2      at D = 128 without dropout, the O store stream: stores each
//               item's O / l, staged by the softmax warps in the item's Q
//               buffer, with TMA and hands the buffer back to the producer
//               once the store has read it; otherwise idle, and the first
//               softmax thread does this
//   warp 3      tcgen05 issuer of O += P_j V_j with P_j read from TMEM
//   warps 4..7  softmax: one query row per thread (TMEM lane), online max and
//               sum in registers, P_j written to TMEM as bf16, lazy rescale of
//               the O accumulator, final O / l and lse per item.  At D = 128
//               without dropout an item's epilogue runs inside the next
//               item's first tile, after its exponentials, so the item's last
//               PV completes behind them instead of stalling the warps at the
//               item boundary.  O / l is staged in the item's Q buffer, no
//               longer read by then.
// At D <= 64 (two CTAs per SM, 128 registers per thread at launch) the first
// warpgroup hands registers to the softmax warpgroup with setmaxnreg: 48 and
// 208 per thread, 128 x 48 + 128 x 208 = the block's 256 x 128; the launch
// checks that the kernel was built with exactly 128 registers per thread.
// Key tiles wholly above the diagonal are never loaded; only the diagonal
// tile applies the element mask.  The score matrix never leaves the SM.
// Without the mask (Causal = false) every query tile runs over all key tiles
// and only the last key tile masks the keys past T.  With dropout (Drop) each
// softmax thread takes its row's 16 keep bytes of a key tile before waiting for
// the tile's S: one 16-byte load from the kept mask when the caller lent one
// (drawn beforehand by dropout_mask.cu), else drawn here from Philox4x32-10,
// eight keys per call (philox.cuh).  The row sum l takes every weight, P_j in
// TMEM only the kept ones, and the final O is scaled by keep_scale / l.
//
// TMEM columns: S [0,128), P (bf16 pairs) [128,192), O [192, 192+D).
#include "internal.h"
#include "sm100.cuh"

#include <cudaTypedefs.h>

namespace attn {
namespace {

using namespace sm100;

constexpr int kBM = 128;          // query rows per CTA (= TMEM lanes)
constexpr int kBN = 128;          // key rows per tile
constexpr int kStages = 2;        // K/V ring depth
constexpr int kThreads = 256;     // 8 warps (two warpgroups)
constexpr int kSoftmaxWarp0 = 4;  // first softmax warp (the second warpgroup)
constexpr int kRegsLaunch = 128;  // registers per thread at launch (D <= 64)
constexpr int kRegsLow = 48;      // first warpgroup after the hand-over
constexpr int kRegsHigh = 208;    // softmax warpgroup after the hand-over
static_assert(kRegsLow + kRegsHigh == 2 * kRegsLaunch, "the register split must add up");
// TMEM columns: 256 at D <= 64, 512 (of which 320 used) at D = 128
template <int D>
__host__ __device__ constexpr uint32_t tmem_cols() { return D > 64 ? 512u : 256u; }
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O when max grows > 2^8

template <int D>
struct FwdSmem {
    static constexpr int kTileBytes = kBN * D * 2;
    alignas(1024) __nv_bfloat16 q[2][kBM * D];
    alignas(1024) __nv_bfloat16 k[kStages][kBN * D];
    alignas(1024) __nv_bfloat16 v[kStages][kBN * D];
    uint64_t q_full[2], q_empty[2];
    uint64_t k_full[kStages], v_full[kStages], k_empty[kStages], v_empty[kStages];
    uint64_t s_full, s_free, p_full;
    uint64_t o_done, o_final, o_free, o_staged, drain;
    uint32_t tmem_slot;
    int abort;
};

// Stores a 4-D tile from shared memory through a tensor map (rows past the
// map's extent are not written); one thread issues, bulk-group tracked.
__device__ __forceinline__ void tma_store_4d(const CUtensorMap *map, const void *src, int c0, int c1,
                                             int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group"
        " [%0, {%1, %2, %3, %4}], [%5];" ::"l"(reinterpret_cast<uint64_t>(map)),
        "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(src))
        : "memory");
}

// The bf16-pair mask of keys e0 and e0 + 1 (e0 even, < 32) of a word W of keep
// bits, given sh[t] = W << t: the sign bit of byte b of sh[t] is bit 8b + 7 - t
// of W, and prmt with a sign-replicating selector copies a byte's sign bit over
// a whole byte; the low half takes key e0, the high half key e0 + 1.
__device__ __forceinline__ uint32_t keep_pair_mask(const uint32_t (&sh)[8], int e0) {
    const int b = e0 >> 3;
    const uint32_t sel = (uint32_t)(8 + b) * 0x0011u | (uint32_t)(12 + b) * 0x1100u;
    uint32_t m;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(m) : "r"(sh[7 - (e0 & 7)]), "r"(sh[6 - (e0 & 7)]), "r"(sel));
    return m;
}

// The n-th work item of CTA c in a grid of G CTAs over W items (snake order),
// or -1 when the CTA has no n-th item.
__device__ __forceinline__ int item_of(int c, int n, int G, int W) {
    const long long w = (long long)n * G + ((n & 1) ? (G - 1 - c) : c);
    return w < W ? (int)w : -1;
}

template <int D, bool Causal, bool Drop>
__global__ void __launch_bounds__(kThreads, D > 64 ? 1 : 2)
    fwd_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
               const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap to,
               float *__restrict__ lse, int T, int H, int BH, int ntiles,
               float scale_log2, const DropoutParams dp, int *err) {
    using Smem = FwdSmem<D>;
    constexpr int kSlabCols = D > 64 ? 64 : D;            // columns per swizzle slab
    constexpr int kSlabs = D / kSlabCols;                 // 1, or 2 at D = 128
    constexpr int kRowBytes = kSlabCols * 2;              // 128 (D >= 64) or 64 (D = 32)
    constexpr uint32_t kSwz = (kRowBytes == 128) ? kSwizzle128B : kSwizzle64B;
    constexpr uint32_t kAtom = 8 * kRowBytes;             // 8-row swizzle atom
    constexpr uint32_t kSlabBytes = 128 * kRowBytes;      // one 128-row slab
    constexpr uint32_t kTmemCols = tmem_cols<D>();
    // With one CTA per SM (D = 128) nothing else fills the item boundary, so an
    // item's epilogue moves into the next item's first tile and warp 2 issues
    // its O store; with two CTAs per SM the other CTA's softmax fills the
    // boundary, and the epilogue stays at the end of the item (measured: the
    // deferred form is slower there).  Not with dropout, whose generator state
    // leaves no registers for the deferred epilogue's.
    constexpr bool kDeferEpilogue = D > 64 && !Drop;
    extern __shared__ uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                         ~uintptr_t(1023));
    volatile int *abort = &sm.abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = (int)gridDim.x, cta = (int)blockIdx.x;
    const int W = ntiles * BH;  // work items; item w is query tile ntiles-1-w/BH of head w%BH

    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.q_full[b], 1);
            mbar_init(&sm.q_empty[b], 1);  // the O store's issuer, once the store has read the buffer
        }
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.k_full[s], 1);
            mbar_init(&sm.v_full[s], 1);
            mbar_init(&sm.k_empty[s], 1);
            mbar_init(&sm.v_empty[s], 1);
        }
        mbar_init(&sm.s_full, 1);
        mbar_init(&sm.s_free, kBM);
        mbar_init(&sm.p_full, kBM);
        mbar_init(&sm.o_done, 1);
        mbar_init(&sm.o_final, 1);
        mbar_init(&sm.o_free, kBM);
        mbar_init(&sm.o_staged, kBM);
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
    ATTN_DCHECK((tmem >> 16) == 0u && (tmem & 0xFFFFu) + kTmemCols <= 512u, err);  // lane 0, within TMEM
    const uint32_t tS = tmem;
    const uint32_t tP = tmem + 128;
    const uint32_t tO = tmem + 192;
    if (warp < kSoftmaxWarp0) {
    // ==================================================== first warpgroup
    if constexpr (D <= 64) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
    if (warp == 0) {
        // ------------------------------------------------ TMA producer (whole warp,
        // one elected lane issues)
        if (lane == 0) {
            prefetch_tensormap(&tq);
            prefetch_tensormap(&tk);
            prefetch_tensormap(&tv);
        }
        __syncwarp();
        if constexpr (D <= 64) {
            // K runs one tile ahead of V: K_{g+1} is issued before V_g, so that
            // the wait for V_g's ring slot (freed by PV_{g-2}) never holds up
            // the K load the next S needs.
            int gt = 0;  // K tiles loaded so far (the K/V ring position)
            int gv = 0;  // V tiles loaded so far
            int nq = 0;  // Q tiles loaded so far
            int pv_j = 0, pv_hh = 0, pv_bb = 0;  // the V tile gv (pending while gv < gt)
            bool ok = true;
            auto load_v = [&]() -> bool {
                const int s = gv % kStages;
                const uint32_t ph = (uint32_t)(gv / kStages) & 1u;
                if (!mbar_wait_warp(&sm.v_empty[s], ph ^ 1u, err, abort)) return false;
                mbar_arrive_expect_tx_e(&sm.v_full[s], Smem::kTileBytes);
#pragma unroll
                for (int sl = 0; sl < kSlabs; ++sl)
                    tma_load_4d_e(reinterpret_cast<uint8_t *>(sm.v[s]) + sl * kSlabBytes, &tv,
                                  &sm.v_full[s], sl * kSlabCols, pv_j * kBN, pv_hh, pv_bb);
                ++gv;
                return true;
            };
            for (int n = 0; ok; ++n) {
                const int w = item_of(cta, n, G, W);
                if (w < 0) break;
                const int qt = ntiles - 1 - w / BH, bh = w % BH;
                const int hh = bh % H, bb = bh / H;
                const int qb = n & 1;
                ATTN_DCHECK(qt >= 0 && qt < ntiles && bh >= 0 && bh < BH, err);
                if (!(ok = mbar_wait_warp(&sm.q_empty[qb], (uint32_t)((n >> 1) & 1) ^ 1u, err, abort))) break;
                mbar_arrive_expect_tx_e(&sm.q_full[qb], Smem::kTileBytes);
#pragma unroll
                for (int sl = 0; sl < kSlabs; ++sl)
                    tma_load_4d_e(reinterpret_cast<uint8_t *>(sm.q[qb]) + sl * kSlabBytes, &tq,
                                  &sm.q_full[qb], sl * kSlabCols, qt * kBM, hh, bb);
                nq = n + 1;
                const int nk = Causal ? qt + 1 : ntiles;  // key tiles this item reads
                for (int j = 0; j < nk; ++j, ++gt) {
                    ATTN_DCHECK(j * kBN < T, err);  // the key tile holds at least one key
                    const int s = gt % kStages;
                    const uint32_t ph = (uint32_t)(gt / kStages) & 1u;
                    if (!(ok = mbar_wait_warp(&sm.k_empty[s], ph ^ 1u, err, abort))) break;
                    mbar_arrive_expect_tx_e(&sm.k_full[s], Smem::kTileBytes);
#pragma unroll
                    for (int sl = 0; sl < kSlabs; ++sl)
                        tma_load_4d_e(reinterpret_cast<uint8_t *>(sm.k[s]) + sl * kSlabBytes, &tk,
                                      &sm.k_full[s], sl * kSlabCols, j * kBN, hh, bb);
                    if (gv < gt && !(ok = load_v())) break;  // the previous tile's V
                    pv_j = j;
                    pv_hh = hh;
                    pv_bb = bb;
                }
            }
            if (ok && gv < gt) ok = load_v();  // the last V (K ahead)
            // Drain: the last loads this warp issued have landed before exit (on the
            // normal path the consumers waited on all of them already).
            for (int g = (gt > kStages ? gt - kStages : 0); g < gt; ++g)
                mbar_wait_drain(&sm.k_full[g % kStages], (uint32_t)(g / kStages) & 1u);
            for (int g = (gv > kStages ? gv - kStages : 0); g < gv; ++g)
                mbar_wait_drain(&sm.v_full[g % kStages], (uint32_t)(g / kStages) & 1u);
            for (int n = (nq > 2 ? nq - 2 : 0); n < nq; ++n)
                mbar_wait_drain(&sm.q_full[n & 1], (uint32_t)(n >> 1) & 1u);
        } else {
            // At D = 128 (one CTA per SM) K_j and V_j go in order: measured
            // faster there than K ahead.
            int gt = 0;  // key tiles loaded so far (the K/V ring position)
            int nq = 0;  // Q tiles loaded so far
            bool ok = true;
            for (int n = 0; ok; ++n) {
                const int w = item_of(cta, n, G, W);
                if (w < 0) break;
                const int qt = ntiles - 1 - w / BH, bh = w % BH;
                const int hh = bh % H, bb = bh / H;
                const int qb = n & 1;
                ATTN_DCHECK(qt >= 0 && qt < ntiles && bh >= 0 && bh < BH, err);
                if (!(ok = mbar_wait_warp(&sm.q_empty[qb], (uint32_t)((n >> 1) & 1) ^ 1u, err, abort))) break;
                mbar_arrive_expect_tx_e(&sm.q_full[qb], Smem::kTileBytes);
#pragma unroll
                for (int sl = 0; sl < kSlabs; ++sl)
                    tma_load_4d_e(reinterpret_cast<uint8_t *>(sm.q[qb]) + sl * kSlabBytes, &tq,
                                  &sm.q_full[qb], sl * kSlabCols, qt * kBM, hh, bb);
                nq = n + 1;
                const int nk = Causal ? qt + 1 : ntiles;  // key tiles this item reads
                for (int j = 0; j < nk; ++j, ++gt) {
                    ATTN_DCHECK(j * kBN < T, err);  // the key tile holds at least one key
                    const int s = gt % kStages;
                    const uint32_t ph = (uint32_t)(gt / kStages) & 1u;
                    if (!(ok = mbar_wait_warp(&sm.k_empty[s], ph ^ 1u, err, abort))) break;
                    mbar_arrive_expect_tx_e(&sm.k_full[s], Smem::kTileBytes);
#pragma unroll
                    for (int sl = 0; sl < kSlabs; ++sl)
                        tma_load_4d_e(reinterpret_cast<uint8_t *>(sm.k[s]) + sl * kSlabBytes, &tk,
                                      &sm.k_full[s], sl * kSlabCols, j * kBN, hh, bb);
                    if (!(ok = mbar_wait_warp(&sm.v_empty[s], ph ^ 1u, err, abort))) {
                        // K of this tile is in flight: let it land before leaving.
                        for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(&sm.k_full[s], ph); ++i) {}
                        break;
                    }
                    mbar_arrive_expect_tx_e(&sm.v_full[s], Smem::kTileBytes);
#pragma unroll
                    for (int sl = 0; sl < kSlabs; ++sl)
                        tma_load_4d_e(reinterpret_cast<uint8_t *>(sm.v[s]) + sl * kSlabBytes, &tv,
                                      &sm.v_full[s], sl * kSlabCols, j * kBN, hh, bb);
                }
            }
            // Drain: the last loads this warp issued have landed before exit (on the
            // normal path the consumers waited on all of them already).
            for (int g = (gt > kStages ? gt - kStages : 0); g < gt; ++g) {
                const int s = g % kStages;
                const uint32_t ph = (uint32_t)(g / kStages) & 1u;
                for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(&sm.k_full[s], ph); ++i) {}
                for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(&sm.v_full[s], ph); ++i) {}
            }
            for (int n = (nq > 2 ? nq - 2 : 0); n < nq; ++n)
                for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(&sm.q_full[n & 1], (uint32_t)(n >> 1) & 1u); ++i) {}
        }
    } else if (kDeferEpilogue && warp == 2) {
        // ------------------------------------------------ O store stream: once
        // the softmax warps have staged an item's O / l in its Q buffer, one
        // lane stores it with the tensor map and, when the store has read the
        // buffer, hands it back to the producer.
        bool ok = true;
        for (int n = 0; ok; ++n) {
            const int w = item_of(cta, n, G, W);
            if (w < 0) break;
            const int qt = ntiles - 1 - w / BH, bh = w % BH;
            if (!(ok = mbar_wait_warp(&sm.o_staged, (uint32_t)n & 1u, err, abort))) break;
            if (lane == 0) {
                const uint8_t *qbuf = reinterpret_cast<const uint8_t *>(sm.q[n & 1]);
#pragma unroll
                for (int sl = 0; sl < kSlabs; ++sl)
                    tma_store_4d(&to, qbuf + sl * kSlabBytes, sl * kSlabCols, qt * kBM, bh % H, bh / H);
                bulk_commit();
                bulk_wait_read_all();
                mbar_arrive(&sm.q_empty[n & 1]);
            }
            __syncwarp();
        }
        if (lane == 0) bulk_wait_all();  // the O stores have completed
    } else if (warp == 1 || warp == 3) {
        // ------------------------------------------------ tcgen05 issuers (whole
        // warp, one elected lane issues).  Two independent streams share the
        // tensor core so that each warp's waits overlap the other's MMAs: warp
        // 1 issues S_g = Q K_g^T for every key tile (S_{g+1} is in flight while
        // the softmax of g runs, also across items), warp 3 issues O += P_g V_g
        // once the softmax has written P_g.  Each barrier is committed by the
        // stream whose MMAs it tracks.
        constexpr uint32_t idS = idesc_bf16(kBM, kBN, 0, 0);  // Q, K both K-major
        constexpr uint32_t idO = idesc_bf16(kBM, D, 0, 1);    // P from TMEM, V MN-major
        bool ok = true;
        int gt = 0;
        for (int n = 0; ok; ++n) {
            const int w = item_of(cta, n, G, W);
            if (w < 0) break;
            const int qt = ntiles - 1 - w / BH;
            const int qb = n & 1;
            const int nk = Causal ? qt + 1 : ntiles;
            if (warp == 1) {
                // ---- score stream
                if (!(ok = mbar_wait_warp(&sm.q_full[qb], (uint32_t)(n >> 1) & 1u, err, abort))) break;
                const uint64_t qd = smem_desc(smem_u32(sm.q[qb]), 16, kAtom, kSwz);
                for (int j = 0; j < nk; ++j, ++gt) {
                    // S_g = Q K_j^T, once the softmax has read S_{g-1} out of TMEM.
                    const int s = gt % kStages;
                    if (!(ok = mbar_wait_warp(&sm.k_full[s], (uint32_t)(gt / kStages) & 1u, err, abort))) break;
                    if (gt >= 1 && !(ok = mbar_wait_warp(&sm.s_free, (uint32_t)(gt - 1) & 1u, err, abort))) break;
                    tc_fence_after();
                    // D / 16 MMAs of K = 16: Q and K both K-major (32 bytes per step).
                    const uint64_t kd = smem_desc(smem_u32(sm.k[s]), 16, kAtom, kSwz);
                    if constexpr (D == 128) {
                        mma_ss_x4<2, 2>(tS, qd, kd, idS, 0u);
                        mma_ss_x4<2, 2>(tS, qd + (kSlabBytes >> 4), kd + (kSlabBytes >> 4), idS, 1u);
                    } else if constexpr (D == 64) {
                        mma_ss_x4<2, 2>(tS, qd, kd, idS, 0u);
                    } else {
                        mma_ss_x2<2, 2>(tS, qd, kd, idS, 0u);
                    }
                    mma_commit_e(&sm.s_full);
                    mma_commit_e(&sm.k_empty[s]);
                    // (this item's Q buffer is released by the softmax warps,
                    // which stage the item's O in it for the TMA store)
                }
            } else {
                // ---- PV stream
                for (int j = 0; j < nk; ++j, ++gt) {
                    const int s = gt % kStages;
                    if (!(ok = mbar_wait_warp(&sm.p_full, (uint32_t)gt & 1u, err, abort))) break;
                    if (!(ok = mbar_wait_warp(&sm.v_full[s], (uint32_t)(gt / kStages) & 1u, err, abort))) break;
                    // The first PV of an item overwrites O: the previous item's O
                    // must have been read out by the softmax warps.
                    if (j == 0 && n >= 1 &&
                        !(ok = mbar_wait_warp(&sm.o_free, (uint32_t)(n - 1) & 1u, err, abort)))
                        break;
                    tc_fence_after();
                    // 8 MMAs of K = 16 keys: P from TMEM (8 columns per step), V
                    // MN-major (16 rows = kRowBytes 16-byte units per step).
                    // (The LBO is the slab stride: N = 128 spans two slabs at D = 128.)
                    const uint64_t vd = smem_desc(smem_u32(sm.v[s]), kSlabBytes, kAtom, kSwz);
                    mma_ts_x4<kRowBytes>(tO, tP, vd, idO, j > 0 ? 1u : 0u);
                    mma_ts_x4<kRowBytes>(tO, tP + 32, vd + 4 * kRowBytes, idO, 1u);
                    mma_commit_e(&sm.o_done);  // PV complete: O stable, P region free
                    mma_commit_e(&sm.v_empty[s]);
                    if (j == nk - 1) mma_commit_e(&sm.o_final);
                }
            }
        }
        // All MMAs of both streams are complete once `drain` fires.
        mma_commit_e(&sm.drain);
        mbar_wait_drain(&sm.drain, 0);
    }
    } else {
    // ==================================================== softmax warpgroup
    if constexpr (D <= 64) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
    {
        const int quad = warp & 3;                 // TMEM lanes 32*quad .. +31
        const int row = quad * 32 + lane;          // row within the query tile
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        // Epilogue of item pn (row max pm in log2 units, row sum pl): once its
        // last PV has completed, O / l goes as bf16 into the item's Q buffer
        // (every S MMA of the item has completed by then) in the swizzled
        // layout of a TMA tile, for warp 2 to store; O's TMEM is released as
        // soon as it is in registers; the row's lse goes to global memory.
        auto epilogue = [&](int pn, float pm, float pl, int pqt, int pbh) -> bool {
            if (!mbar_wait_warp(&sm.o_final, (uint32_t)pn & 1u, err, abort)) return false;
            tc_fence_after();
            const float inv = (Drop ? dp.keep_scale : 1.f) / pl;
            uint8_t *qbuf = reinterpret_cast<uint8_t *>(sm.q[pn & 1]);
            const uint32_t swz = kRowBytes == 128 ? (uint32_t)(row & 7) : (uint32_t)((row >> 1) & 3);
            constexpr int kPerRound = D > 64 ? 2 : D / 32;  // 32-column TMEM loads in flight at once
#pragma unroll
            for (int h0 = 0; h0 < D / 32; h0 += kPerRound) {
                uint32_t r[kPerRound][32];
#pragma unroll
                for (int h = 0; h < kPerRound; ++h) tmem_ld32(tO + lane_off + 32 * (h0 + h), r[h]);
                tmem_wait_ld();
#pragma unroll
                for (int h = 0; h < kPerRound; ++h) reg_fence32(r[h]);
                if (h0 + kPerRound == D / 32) {
                    tc_fence_before();
                    mbar_arrive(&sm.o_free);
                }
#pragma unroll
                for (int h = 0; h < kPerRound; ++h) {
                    const int col0 = 32 * (h0 + h);  // first column of this load
                    const int sl = col0 / kSlabCols;
                    const uint32_t base = smem_u32(qbuf + sl * kSlabBytes) + (uint32_t)row * kRowBytes;
                    ATTN_DCHECK(sl * kSlabBytes + (row + 1) * kRowBytes <= (int)sizeof(sm.q[0]), err);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {  // 16-byte chunks of 8 columns
                        const uint32_t chunk = (uint32_t)((col0 % kSlabCols) / 8 + c);
                        const uint32_t *v = &r[h][8 * c];
                        st_shared_v4(base + ((chunk ^ swz) << 4),
                                     pack_bf16x2(__uint_as_float(v[0]) * inv, __uint_as_float(v[1]) * inv),
                                     pack_bf16x2(__uint_as_float(v[2]) * inv, __uint_as_float(v[3]) * inv),
                                     pack_bf16x2(__uint_as_float(v[4]) * inv, __uint_as_float(v[5]) * inv),
                                     pack_bf16x2(__uint_as_float(v[6]) * inv, __uint_as_float(v[7]) * inv));
                    }
                }
            }
            fence_proxy_async_smem();
            if constexpr (kDeferEpilogue) {
                mbar_arrive(&sm.o_staged);
            } else {
                named_bar_sync(1, kBM);
                if (warp == kSoftmaxWarp0 && lane == 0) {
#pragma unroll
                    for (int sl = 0; sl < kSlabs; ++sl)
                        tma_store_4d(&to, qbuf + sl * kSlabBytes, sl * kSlabCols, pqt * kBM, pbh % H, pbh / H);
                    bulk_commit();
                    // Once the store has read the tile, the buffer takes item pn + 2's Q.
                    bulk_wait_read_all();
                    mbar_arrive(&sm.q_empty[pn & 1]);
                }
            }
            const int t = pqt * kBM + row;
            ATTN_DCHECK(pbh >= 0 && pbh < BH && row < kBM, err);
            if (t < T) lse[(size_t)pbh * T + t] = (pm + log2f(pl)) * 0.69314718055994531f;
            return true;
        };
        int gt = 0;  // global key-tile counter (barrier phases)
        int pn = -1, pqt = 0, pbh = 0;  // the item whose epilogue is still to run
        float pm = 0.f, pl = 1.f;
        bool ok = true;
        for (int n = 0; ok; ++n) {
            const int w = item_of(cta, n, G, W);
            if (w < 0) break;
            const int qt = ntiles - 1 - w / BH, bh = w % BH;
            float m_used = -INFINITY, l = 0.f;
            const int nk = Causal ? qt + 1 : ntiles;
            for (int j = 0; j < nk; ++j, ++gt) {
                // This row's keep bits against key tile j (Drop), four 8-key
                // groups (bytes) per word, ready before S is: loaded from the
                // kept mask, or drawn here, eight keys per generator call.
                [[maybe_unused]] uint32_t kwv[kBN / 32];
                if constexpr (Drop) {
                    const uint32_t ti = (uint32_t)(qt * kBM + row);
                    if (dp.mask) {
                        ATTN_DCHECK(ti < dp.mask_ld && (uint32_t)(j + 1) * kBN <= dp.mask_ld, err);
                        const uint4 mw = __ldg(reinterpret_cast<const uint4 *>(
                            dp.mask + philox::mask_at(dp, (uint32_t)bh, (uint32_t)(j * (kBN / 8)), ti)));
                        kwv[0] = mw.x;
                        kwv[1] = mw.y;
                        kwv[2] = mw.z;
                        kwv[3] = mw.w;
                    } else {
#pragma unroll
                        for (int q = 0; q < kBN / 32; ++q) {
                            uint32_t w4 = 0u;
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                w4 |= philox::keep_byte(dp, ti, (uint32_t)(j * (kBN / 8) + 4 * q + e),
                                                        (uint32_t)bh)
                                      << (8 * e);
                            kwv[q] = w4;
                        }
                    }
                }
                ok = mbar_wait_warp(&sm.s_full, (uint32_t)gt & 1u, err, abort);
                if (!ok) break;
                tc_fence_after();
                float s[kBN];
                {
                    // All four 32-column loads in flight before one wait.
                    uint32_t r0[32], r1[32], r2[32], r3[32];
                    tmem_ld32(tS + lane_off + 0, r0);
                    tmem_ld32(tS + lane_off + 32, r1);
                    tmem_ld32(tS + lane_off + 64, r2);
                    tmem_ld32(tS + lane_off + 96, r3);
                    tmem_wait_ld();
                    reg_fence32(r0);
                    reg_fence32(r1);
                    reg_fence32(r2);
                    reg_fence32(r3);
                    tc_fence_before();
                    mbar_arrive(&sm.s_free);  // S is in registers: the next S may overwrite it
#pragma unroll
                    for (int x = 0; x < 32; ++x) {
                        s[x] = __uint_as_float(r0[x]);
                        s[32 + x] = __uint_as_float(r1[x]);
                        s[64 + x] = __uint_as_float(r2[x]);
                        s[96 + x] = __uint_as_float(r3[x]);
                    }
                }
                if constexpr (Causal) {
                    if (j == qt) {  // diagonal tile: key column c is visible to row r iff c <= r
#pragma unroll
                        for (int c = 0; c < kBN; ++c)
                            if (c > row) s[c] = -INFINITY;
                    }
                } else {
                    const int lim = T - j * kBN;  // keys past T (zero-filled rows) are masked
                    if (lim < kBN) {
#pragma unroll
                        for (int c = 0; c < kBN; ++c)
                            if (c >= lim) s[c] = -INFINITY;
                    }
                }
                // Row max as eight independent chains (short dependency depth).
                float mc[8];
#pragma unroll
                for (int x = 0; x < 8; ++x) mc[x] = s[x];
#pragma unroll
                for (int c = 8; c < kBN; c += 8)
#pragma unroll
                    for (int x = 0; x < 8; ++x) mc[x] = fmaxf(mc[x], s[c + x]);
                const float mx = fmaxf(fmaxf(fmaxf(mc[0], mc[1]), fmaxf(mc[2], mc[3])),
                                       fmaxf(fmaxf(mc[4], mc[5]), fmaxf(mc[6], mc[7])));
                const float mxs = mx * scale_log2;
                // Each row moves its own running max only when its scores exceed
                // it by more than the threshold; the warp merely decides whether
                // the TMEM round trip of O is needed (rows that keep their max
                // scale by exactly 1).  A row's arithmetic thus depends on its
                // own scores alone.
                const bool need = mxs > m_used + kRescaleThreshold;
                bool pv_done = (gt == 0);  // the previous PV is complete: O stable, P free
                if (__any_sync(0xffffffffu, need)) {
                    const float m_new = need ? mxs : m_used;
                    const float alpha = ex2(m_used - m_new);
                    if (j > 0) {
                        ok = mbar_wait_warp(&sm.o_done, (uint32_t)(gt - 1) & 1u, err, abort);
                        if (!ok) break;
                        pv_done = true;
                        tc_fence_after();
#pragma unroll
                        for (int c = 0; c < D; c += 16) {
                            uint32_t r[16];
                            tmem_ld16(tO + lane_off + c, r);
                            tmem_wait_ld();
                            reg_fence16(r);
#pragma unroll
                            for (int x = 0; x < 16; ++x) r[x] = __float_as_uint(__uint_as_float(r[x]) * alpha);
                            tmem_st16(tO + lane_off + c, r);
                        }
                    }
                    l *= alpha;
                    m_used = m_new;
                }
                const float neg_m = -m_used;
                // All exponentials first (packed bf16 pairs), then wait for the
                // previous PV to release the P region: the wait sits at the end
                // of the tile, where the previous PV has had the most time.
                // Exponent arguments and the two running row sums (even and odd
                // keys) are float32 pairs, one packed instruction per key pair.
                uint32_t pk[kBN / 2];
                const uint64_t sc2 = f2pack(scale_log2, scale_log2), nm2 = f2pack(neg_m, neg_m);
                uint64_t l2 = f2pack(0.f, 0.f);
                if constexpr (Drop) {
                    // Word q of keep bits covers keys 32q .. 32q+31 (bit e = key
                    // 32q + e); its left shifts by 0..7 put every key's bit in the
                    // sign position of some byte, so a byte permute turns the two
                    // bits of a key pair into the pair's bf16 mask.
#pragma unroll
                    for (int q = 0; q < kBN / 32; ++q) {
                        uint32_t sh[8];
#pragma unroll
                        for (int t = 0; t < 8; ++t) sh[t] = kwv[q] << t;
#pragma unroll
                        for (int y = 0; y < 16; ++y) {
                            const int x = 16 * q + y;
                            const float2 t = f2unpack(ffma2(f2pack(s[2 * x], s[2 * x + 1]), sc2, nm2));
                            const float p0 = ex2(t.x);
                            const float p1 = ex2(t.y);
                            l2 = fadd2(l2, f2pack(p0, p1));
                            pk[x] = pack_bf16x2(p0, p1) & keep_pair_mask(sh, 2 * y);
                        }
                    }
                } else {
#pragma unroll
                    for (int x = 0; x < kBN / 2; ++x) {
                        const float2 t = f2unpack(ffma2(f2pack(s[2 * x], s[2 * x + 1]), sc2, nm2));
                        const float p0 = ex2(t.x);
                        const float p1 = ex2(t.y);
                        l2 = fadd2(l2, f2pack(p0, p1));
                        pk[x] = pack_bf16x2(p0, p1);
                    }
                }
                const float2 lab = f2unpack(l2);
                l += lab.x + lab.y;
                if (kDeferEpilogue && j == 0 && pn >= 0) {
                    // The previous item's epilogue, off the item boundary: its
                    // last PV has had this tile's exponentials to complete (its
                    // completion also frees the P region).
                    if (!(ok = epilogue(pn, pm, pl, pqt, pbh))) break;
                    pn = -1;
                } else if (!pv_done) {
                    ok = mbar_wait_warp(&sm.o_done, (uint32_t)(gt - 1) & 1u, err, abort);
                    if (!ok) break;
                    tc_fence_after();
                }
#pragma unroll
                for (int c = 0; c < kBN / 2; c += 16)
                    tmem_st16(tP + lane_off + c, *reinterpret_cast<uint32_t (*)[16]>(&pk[c]));
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&sm.p_full);
            }
            if (!ok) break;
            if constexpr (kDeferEpilogue) {
                pn = n;
                pqt = qt;
                pbh = bh;
                pm = m_used;
                pl = l;
            } else if (!(ok = epilogue(n, m_used, l, qt, bh))) {
                break;
            }
        }
        if (kDeferEpilogue && ok && pn >= 0) epilogue(pn, pm, pl, pqt, pbh);  // the CTA's last item
        // The O stores issued by the first softmax thread have completed.
        if (!kDeferEpilogue && warp == kSoftmaxWarp0 && lane == 0) bulk_wait_all();
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

}  // namespace

cudaError_t make_map_bf16(void *map, const void *ptr, const Shape &s, const TStrides &st) {
    auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
    if (!enc) return cudaErrorInitializationError;
    const cuuint64_t dims[4] = {(cuuint64_t)s.D, (cuuint64_t)s.T, (cuuint64_t)s.H, (cuuint64_t)s.B};
    const cuuint64_t strides[3] = {(cuuint64_t)st.t * 2, (cuuint64_t)st.h * 2, (cuuint64_t)st.b * 2};
    // Box: one 128-row slab of at most 64 columns (128 bytes, the swizzle span);
    // D = 128 rows load as two slabs.
    const cuuint32_t box_x = s.D > 64 ? 64 : (cuuint32_t)s.D;
    const cuuint32_t box[4] = {box_x, 128, 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = enc(static_cast<CUtensorMap *>(map), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                           const_cast<void *>(ptr), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE,
                           box_x * 2 == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

namespace {

template <int D, bool Causal, bool Drop>
cudaError_t launch_fwd(const __nv_bfloat16 *q, const __nv_bfloat16 *k, const __nv_bfloat16 *v,
                       __nv_bfloat16 *o, float *lse, Shape s, const FwdStrides &str, int *err,
                       cudaStream_t st, LaunchInfo &li) {
    const int BH = s.B * s.H;
    const int ntiles = (s.T + kBM - 1) / kBM;
    const long long items = (long long)ntiles * BH;
    if (items > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    int dev = 0, sms = 0;
    cudaError_t e0;
    if ((e0 = cudaGetDevice(&dev)) != cudaSuccess) return e0;
    if ((e0 = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e0;
    // Persistent grid: two CTAs per SM (one at D = 128), never more CTAs than
    // work items.
    const long long per_sm = D > 64 ? 1 : 2;
    const long long grid = items < per_sm * sms ? items : per_sm * sms;
    CUtensorMap mq, mk, mv, mo;
    cudaError_t e;
    if ((e = make_map_bf16(&mq, q, s, str.q)) != cudaSuccess) return e;
    if ((e = make_map_bf16(&mk, k, s, str.k)) != cudaSuccess) return e;
    if ((e = make_map_bf16(&mv, v, s, str.v)) != cudaSuccess) return e;
    if ((e = make_map_bf16(&mo, o, s, str.o)) != cudaSuccess) return e;
    const size_t smem = sizeof(FwdSmem<D>) + 1024;
    static std::atomic<unsigned long long> smem_set{0};
    if ((e = set_max_smem_once(reinterpret_cast<const void *>(fwd_kernel<D, Causal, Drop>), smem, dev,
                               smem_set)) != cudaSuccess)
        return e;
    if constexpr (D <= 64) {
        // The setmaxnreg hand-over assumes the block holds 256 x 128
        // registers; any other build would make the increase wait forever.
        static int checked = 0;  // 0 unknown, 1 good, -1 bad
        if (checked == 0) {
            cudaFuncAttributes fa;
            if ((e = cudaFuncGetAttributes(&fa, fwd_kernel<D, Causal, Drop>)) != cudaSuccess) return e;
            checked = (fa.numRegs == kRegsLaunch) ? 1 : -1;
        }
        if (checked < 0) return cudaErrorInvalidConfiguration;
    }
    const float scale_log2 = s.scale * 1.4426950408889634f;
    if ((e = mark_main_start(li, st)) != cudaSuccess) return e;
    if ((e = launch_pdl(fwd_kernel<D, Causal, Drop>, dim3((unsigned)grid), dim3(kThreads), smem, st,
                        mq, mk, mv, mo, lse, s.T, s.H, BH, ntiles, scale_log2, s.drop, err)) !=
        cudaSuccess)
        return e;
    li.kernels += 1;
    return mark_main_end(li, st);
}

}  // namespace

cudaError_t sm100_fwd(const __nv_bfloat16 *q, const __nv_bfloat16 *k, const __nv_bfloat16 *v,
                      __nv_bfloat16 *o, float *lse, Shape s, const FwdStrides &str, int *err,
                      cudaStream_t st, LaunchInfo &li) {
#define ATTN_FWD_CASE(DD, C, R)                                    \
    if (s.D == DD && (s.causal != 0) == C && s.dropout == R)       \
        return launch_fwd<DD, C, R>(q, k, v, o, lse, s, str, err, st, li);
    ATTN_FWD_CASE(128, true, false)
    ATTN_FWD_CASE(128, false, false)
    ATTN_FWD_CASE(128, true, true)
    ATTN_FWD_CASE(128, false, true)
    ATTN_FWD_CASE(64, true, false)
    ATTN_FWD_CASE(64, false, false)
    ATTN_FWD_CASE(64, true, true)
    ATTN_FWD_CASE(64, false, true)
    ATTN_FWD_CASE(32, true, false)
    ATTN_FWD_CASE(32, false, false)
    ATTN_FWD_CASE(32, true, true)
    ATTN_FWD_CASE(32, false, true)
#undef ATTN_FWD_CASE
    return cudaErrorInvalidValue;
}

}  // namespace attn
