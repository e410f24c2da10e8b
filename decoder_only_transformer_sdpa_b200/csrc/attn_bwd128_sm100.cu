// attn_bwd128_sm100.cu -- the backward main kernel at head_dim 128.
//
// Same derivative as attn_bwd_sm100.cu (the exact gradient of the forward of
// "How Andrej Karpathy built GPT from 200 lines of code", sections
// "Self-Attention: the mathematical trick" [55:20] and "Implementing the
// attention heads (Query, Key, Value)" [1:06:16]-[1:17:18], for the loss
// L = sum(O * dO)), with a TMEM plan that fits D = 128: S^T, dP^T, dK and dV
// at 128 columns each would fill all 512, so
//   * the query side is walked in 64-row sub-tiles (S^T, dP^T: 64 columns);
//   * dQ is computed transposed, dQ_i^T = K^T dS^T (M = D = 128 rows of
//     TMEM, N = 64 queries), with K read MN-major from the same shared tile
//     the S^T MMA reads K-major;
//   * the drain warps transpose dQ^T through a swizzled shared staging tile
//     and add it into the float32 accumulator with TMA reduce-add.
//
// One CTA per (128-row key tile, head), 15 warps:
//   warp 0      TMA producer: K_j, V_j once (two 64-column slabs each); Q_i,
//               dO_i (64 rows, two slabs each), lse_i, Delta_i per sub-tile
//               into a 2-stage ring
//   warp 1      tcgen05 issuer of S^T and dP^T, TMEM owner
//   warps 2..9  softmax gradient: two warps per TMEM lane quadrant (32 key
//               rows), one per 32-query half of the sub-tile; P^T to TMEM
//               (bf16), dS^T to shared memory (bf16, double buffered)
//   warps 10..13 dQ drain: TMEM lane d holds column d of dQ^T
//   warp 14     tcgen05 issuer of dV, dK and dQ^T (a second stream, so that
//               each issuer's waits overlap the other's MMAs)
//
// TMEM columns: S^T [0,64), dP^T [64,128), dV [128,256), dK [256,384),
// dQ^T [384,448), P^T (bf16 pairs) [448,480).
#include "internal.h"
#include "sm100.cuh"

#include <cudaTypedefs.h>
#include <type_traits>

namespace attn {
namespace {

using namespace sm100;

constexpr int D = 128;
constexpr int kBK = 128;          // key rows per CTA
constexpr int kBQ = 64;           // query rows per sub-tile
constexpr int kThreads = 480;     // 15 warps
constexpr int kEwThreads = 256;   // softmax-gradient threads (warps 2..9)
constexpr int kQStages = 2;       // Q / dO / lse / Delta ring depth
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kAtom = 1024;  // 8 rows of 128 bytes (128-byte swizzle)
constexpr uint32_t kKSlab = kBK * 128;  // one 64-column slab of K or V: 16 KB
constexpr uint32_t kQSlab = kBQ * 128;  // one 64-column slab of Q or dO: 8 KB

struct Smem128 {
    alignas(1024) __nv_bfloat16 k[2][kBK * 64];             // [slab][key][64 cols]
    alignas(1024) __nv_bfloat16 v[2][kBK * 64];
    alignas(1024) __nv_bfloat16 q[kQStages][2][kBQ * 64];   // [stage][slab][query][64 cols]
    alignas(1024) __nv_bfloat16 dO[kQStages][2][kBQ * 64];
    alignas(1024) __nv_bfloat16 ds[2][kBK * kBQ];           // dS^T [buffer][key][64 queries]
    alignas(1024) float stage[4][kBQ * 32];                 // dQ [d block][query][32 d], swizzled
    alignas(16) float lse2[kQStages][kBQ];
    alignas(16) float delta[kQStages][kBQ];
    uint64_t kv_full, qdo_full[kQStages], qdo_empty[kQStages];
    uint64_t sdp_full, sdp_free, p_ready[2], ds_ready[2], p_free, ds_free[2];
    uint64_t dq_full, dq_free, acc_done, drain;
    uint32_t tmem_slot;
    int abort;
};

template <bool Causal, bool Drop>
__global__ void __launch_bounds__(kThreads, 1)
    bwd128_main_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                       const __grid_constant__ CUtensorMap tdq, const float *__restrict__ lse2,
                       const float *__restrict__ delta, __nv_bfloat16 *__restrict__ dk,
                       __nv_bfloat16 *__restrict__ dv, const TStrides sdk, const TStrides sdv,
                       int T, int Tpad, int H, int BH, int nqt, float scale_log2, float scale,
                       const DropoutParams dp, int *err) {
    extern __shared__ uint8_t smem_raw[];
    Smem128 &sm = *reinterpret_cast<Smem128 *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    volatile int *abort = &sm.abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kt = (int)(blockIdx.x / BH);  // key tile; tile 0 sees the most query sub-tiles
    const int bh = (int)(blockIdx.x % BH);
    const int hh = bh % H, bb = bh / H;
    // Query sub-tiles: from the first one that reaches this key tile's
    // diagonal (causal) or 0, to the last.
    const int q_first = Causal ? (kt * kBK) / kBQ : 0;
    const int n_q = nqt - q_first;

    if (threadIdx.x == 0) {
        mbar_init(&sm.kv_full, 1);
        for (int s = 0; s < kQStages; ++s) {
            mbar_init(&sm.qdo_full[s], 1);
            mbar_init(&sm.qdo_empty[s], 1);
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
        mbar_init(&sm.dq_free, 128);
        mbar_init(&sm.acc_done, 1);
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
    const uint32_t tS = tmem, tdP = tmem + 64, tdV = tmem + 128, tdK = tmem + 256;
    const uint32_t tdQ = tmem + 384, tP = tmem + 448;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tensormap(&tq);
            prefetch_tensormap(&tk);
            prefetch_tensormap(&tv);
            prefetch_tensormap(&tdo);
        }
        __syncwarp();
        mbar_arrive_expect_tx_e(&sm.kv_full, 2 * 2 * kKSlab);
        for (int sl = 0; sl < 2; ++sl) {
            tma_load_4d_e(sm.k[sl], &tk, &sm.kv_full, 64 * sl, kt * kBK, hh, bb);
            tma_load_4d_e(sm.v[sl], &tv, &sm.kv_full, 64 * sl, kt * kBK, hh, bb);
        }
        int issued = 0;
        for (int idx = 0; idx < n_q; ++idx) {
            const int st = idx % kQStages;
            const int i = q_first + idx;
            if (!mbar_wait_warp(&sm.qdo_empty[st], (uint32_t)((idx / kQStages) & 1) ^ 1u, err, abort)) break;
            mbar_arrive_expect_tx_e(&sm.qdo_full[st], 2 * 2 * kQSlab + 2 * kBQ * 4);
            for (int sl = 0; sl < 2; ++sl) {
                tma_load_4d_e(sm.q[st][sl], &tq, &sm.qdo_full[st], 64 * sl, i * kBQ, hh, bb);
                tma_load_4d_e(sm.dO[st][sl], &tdo, &sm.qdo_full[st], 64 * sl, i * kBQ, hh, bb);
            }
            const size_t prow = (size_t)bh * Tpad + (size_t)i * kBQ;
            ATTN_DCHECK(kt * kBK < T && prow + kBQ <= (size_t)BH * Tpad && i * kBQ < T, err);
            bulk_load_e(sm.lse2[st], lse2 + prow, kBQ * 4, &sm.qdo_full[st]);
            bulk_load_e(sm.delta[st], delta + prow, kBQ * 4, &sm.qdo_full[st]);
            issued = idx + 1;
        }
        for (int idx = (issued > kQStages ? issued - kQStages : 0); idx < issued; ++idx)
            for (uint32_t n = 0; n < kWaitLimit && !mbar_try_wait(&sm.qdo_full[idx % kQStages], (uint32_t)(idx / kQStages) & 1u); ++n) {}
        mbar_wait_warp(&sm.kv_full, 0, err, abort);
    } else if (warp == 1 || warp == 14) {
        // ------------------------------------------------ tcgen05 issuers: warp 1
        // the scores, warp 14 the gradients.  They touch disjoint TMEM, and each
        // barrier is committed by the stream whose MMAs it tracks (a commit
        // covers only its own thread's MMAs).
        constexpr uint32_t idS = idesc_bf16(kBK, kBQ, 0, 0);  // S^T, dP^T: M = 128 keys, N = 64 queries
        constexpr uint32_t idKV = idesc_bf16(kBK, D, 0, 1);   // dV, dK: N = 128 columns (B MN-major)
        constexpr uint32_t idQ = idesc_bf16(D, kBQ, 1, 1);    // dQ^T: M = 128 columns, both MN-major
        bool ok = true;
        if (warp == 1) {
            // K and V K-major (A of S^T / dP^T; 32 bytes per K step, second slab
            // kKSlab further).
            const uint64_t kd_k = smem_desc(smem_u32(sm.k[0]), 16, kAtom, kSwizzle128B);
            const uint64_t vd_k = smem_desc(smem_u32(sm.v[0]), 16, kAtom, kSwizzle128B);
            ok = mbar_wait_warp(&sm.kv_full, 0, err, abort);
            for (int idx = 0; ok && idx < n_q; ++idx) {
                const int st = idx % kQStages;
                if (!(ok = mbar_wait_warp(&sm.qdo_full[st], (uint32_t)(idx / kQStages) & 1u, err, abort))) break;
                if (idx >= 1 && !(ok = mbar_wait_warp(&sm.sdp_free, (uint32_t)(idx - 1) & 1u, err, abort))) break;
                tc_fence_after();
                const uint64_t qd = smem_desc(smem_u32(sm.q[st][0]), 16, kAtom, kSwizzle128B);
                const uint64_t dod = smem_desc(smem_u32(sm.dO[st][0]), 16, kAtom, kSwizzle128B);
                // S^T = K Q^T and dP^T = V dO^T over D = 128: 8 MMAs each.
                mma_ss_x4<2, 2>(tS, kd_k, qd, idS, 0u);
                mma_ss_x4<2, 2>(tS, kd_k + (kKSlab >> 4), qd + (kQSlab >> 4), idS, 1u);
                mma_ss_x4<2, 2>(tdP, vd_k, dod, idS, 0u);
                mma_ss_x4<2, 2>(tdP, vd_k + (kKSlab >> 4), dod + (kQSlab >> 4), idS, 1u);
                mma_commit_e(&sm.sdp_full);
            }
        } else {
            // K MN-major as the A of dQ^T (M = 128 spans the two slabs: LBO =
            // slab stride; 16 keys = 2048 bytes per K step).  It needs no wait
            // of its own: the first dS^T exists only after the first S^T, which
            // waited for K and V.
            const uint64_t kd_mn = smem_desc(smem_u32(sm.k[0]), kKSlab, kAtom, kSwizzle128B);
            for (int p = 0; ok && p < n_q; ++p) {
                const int st = p % kQStages, b = p & 1;
                // Q and dO MN-major as B of dK / dV (N = 128 spans two slabs:
                // LBO = slab stride; 16 queries = 2048 bytes per K step).
                const uint64_t qd_mn = smem_desc(smem_u32(sm.q[st][0]), kQSlab, kAtom, kSwizzle128B);
                const uint64_t dod_mn = smem_desc(smem_u32(sm.dO[st][0]), kQSlab, kAtom, kSwizzle128B);
                const uint32_t ds_addr = smem_u32(sm.ds[b]);
                // dS^T [key][64 queries]: K-major A of dK (32 bytes per 16
                // queries) and MN-major B of dQ^T (2048 bytes per 16 keys).
                const uint64_t dsd_k = smem_desc(ds_addr, 16, kAtom, kSwizzle128B);
                const uint64_t dsd_mn = smem_desc(ds_addr, kKSlab, kAtom, kSwizzle128B);
                if (!(ok = mbar_wait_warp(&sm.p_ready[b], (uint32_t)(p >> 1) & 1u, err, abort))) break;
                tc_fence_after();
                // dV += P^T dO: 4 MMAs of K = 16 queries, A from TMEM.
                mma_ts_x4<128>(tdV, tP, dod_mn, idKV, p > 0 ? 1u : 0u);
                mma_commit_e(&sm.p_free);
                if (!(ok = mbar_wait_warp(&sm.ds_ready[b], (uint32_t)(p >> 1) & 1u, err, abort))) break;
                tc_fence_after();
                // dK += dS^T Q: 4 MMAs of K = 16 queries.
                mma_ss_x4<2, 128>(tdK, dsd_k, qd_mn, idKV, p > 0 ? 1u : 0u);
                // Q, dO, lse, Delta of this sub-tile are consumed (its S^T /
                // dP^T completed before its dS^T existed).
                mma_commit_e(&sm.qdo_empty[st]);
                if (p >= 1 && !(ok = mbar_wait_warp(&sm.dq_free, (uint32_t)(p - 1) & 1u, err, abort))) break;
                tc_fence_after();
                // dQ^T = K^T dS^T: 8 MMAs of K = 16 keys.
                mma_ss_x4<128, 128>(tdQ, kd_mn, dsd_mn, idQ, 0u);
                mma_ss_x4<128, 128>(tdQ, kd_mn + 4 * 128, dsd_mn + 4 * 128, idQ, 1u);
                mma_commit_e(&sm.dq_full);
                mma_commit_e(&sm.ds_free[b]);
            }
            mma_commit_e(&sm.acc_done);
        }
        mma_commit_e(&sm.drain);
        mbar_wait_drain(&sm.drain, 0);
    } else if (warp < 10) {
        // ------------------------------------------------ softmax gradient
        const int quad = warp & 3;
        const int half = (warp - 2) >> 2;               // queries [32 half, 32 half + 32)
        const int kr = quad * 32 + lane;                // key row (TMEM lane)
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const uint32_t sw = (uint32_t)(kr & 7);
        const int q0 = 32 * half;
        bool ok = true;
        for (int idx = 0; idx < n_q; ++idx) {
            const int st = idx % kQStages, b = idx & 1;
            const int i = q_first + idx;
            // With a kept dropout mask, this sub-tile's keep bytes are loaded
            // before the wait for S^T (byte r: keys 8 jg .. +7 of query ib + 8 r).
            uint32_t kept = 0u;
            if constexpr (Drop) {
                if (dp.mask) {
                    const uint32_t jg = (uint32_t)((kt * kBK + quad * 32 + (lane & ~7)) >> 3);
                    const uint32_t ib = (uint32_t)(i * kBQ + q0) + (lane & 7);
#pragma unroll
                    for (int r = 0; r < 4; ++r)
                        kept |= (uint32_t)__ldg(dp.mask + philox::mask_at(dp, (uint32_t)bh, jg, ib + 8u * r))
                                << (8 * r);
                }
            }
            ok = mbar_wait_warp(&sm.sdp_full, (uint32_t)idx & 1u, err, abort);
            if (!ok) break;
            tc_fence_after();
            // causal: the sub-tiles that reach into this key tile mask queries before keys
            const bool diag = Causal && (i * kBQ < kt * kBK + kBK);
            const int qg0 = i * kBQ + q0 - kt * kBK;    // first query minus the tile's first key
            const uint32_t lse_addr = smem_u32(sm.lse2[st]), dl_addr = smem_u32(sm.delta[st]);
            uint32_t rs[32], rp[32];
            tmem_ld32(tS + lane_off + q0, rs);
            tmem_ld32(tdP + lane_off + q0, rp);
            tmem_wait_ld();
            reg_fence32(rs);
            reg_fence32(rp);
            tc_fence_before();
            mbar_arrive(&sm.sdp_free);  // S^T and dP^T are in registers
            uint32_t keepm = 0xFFFFFFFFu;
            if constexpr (Drop) {
                const uint32_t sub = (uint32_t)(lane & 7);
                const uint32_t jg = (uint32_t)((kt * kBK + quad * 32 + (lane & ~7)) >> 3);
                const uint32_t ib = (uint32_t)(i * kBQ + q0) + sub;
                uint32_t wbits = kept;
                if (!dp.mask) {
#pragma unroll
                    for (int r = 0; r < 4; ++r)
                        wbits |= philox::keep_byte_lanes(dp, ib + 8u * r, jg, (uint32_t)bh) << (8 * r);
                }
                keepm = philox::transpose_keep_bits(wbits, lane);
            }
            uint32_t pw[16], dw[16];
            const uint64_t sc2 = f2pack(scale_log2, scale_log2);
            // lse2 and delta hold -lse * log2(e) and -Delta' (prep kernel); the
            // arithmetic runs on float32 pairs, and only the diagonal sub-tile
            // takes the per-weight causal test.
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
                        const float2 t =
                            f2unpack(ffma2(f2pack(__uint_as_float(rs[e]), __uint_as_float(rs[e + 1])), sc2, nl));
                        float p0 = ex2(t.x), p1 = ex2(t.y);
                        if constexpr (kDiag) {  // query before key: masked
                            if (qg0 + e < kr) p0 = 0.f;
                            if (qg0 + e + 1 < kr) p1 = 0.f;
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
            // P^T in TMEM is free once dV of the previous sub-tile completed;
            // this dS^T buffer once dK / dQ^T of two sub-tiles ago completed.
            bool w = true;
            if (idx >= 1) w = mbar_wait(&sm.p_free, (uint32_t)(idx - 1) & 1u, err, abort);
            w = w && mbar_wait(&sm.ds_free[b], (uint32_t)((idx >> 1) & 1) ^ 1u, err, abort);
            ok = __all_sync(0xffffffffu, w);
            if (!ok) break;
            tc_fence_after();
            tmem_st16(tP + lane_off + q0 / 2, pw);
            const uint32_t ds_row = smem_u32(sm.ds[b]) + (uint32_t)kr * 128;
#pragma unroll
            for (int u = 0; u < 4; ++u) {  // four 16-byte chunks = this half's 32 queries
                const uint32_t g = 4 * half + u;
                st_shared_v4(ds_row + ((g ^ sw) << 4), dw[4 * u], dw[4 * u + 1], dw[4 * u + 2],
                             dw[4 * u + 3]);
            }
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&sm.p_ready[b]);
            mbar_arrive(&sm.ds_ready[b]);
        }
        // ---- epilogue: dK (times scale) from the first half's warps, dV from the second's
        if (ok) ok = mbar_wait_warp(&sm.acc_done, 0, err, abort);
        if (ok) {
            tc_fence_after();
            const int t = kt * kBK + kr;
            const uint32_t src = half == 0 ? tdK : tdV;
            const float mul = Drop ? (half == 0 ? scale : 1.f) * dp.keep_scale : (half == 0 ? scale : 1.f);
            const TStrides so = half == 0 ? sdk : sdv;
            __nv_bfloat16 *out = (half == 0 ? dk : dv) + (long long)bb * so.b + (long long)hh * so.h +
                                 (long long)t * so.t;
#pragma unroll
            for (int c = 0; c < D; c += 32) {
                uint32_t r[32];
                tmem_ld32(src + lane_off + c, r);
                tmem_wait_ld();
                reg_fence32(r);
                if (t < T) {
                    uint4 *dst = reinterpret_cast<uint4 *>(out + c);
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        uint4 w4;
                        w4.x = pack_bf16x2(__uint_as_float(r[8 * x + 0]) * mul, __uint_as_float(r[8 * x + 1]) * mul);
                        w4.y = pack_bf16x2(__uint_as_float(r[8 * x + 2]) * mul, __uint_as_float(r[8 * x + 3]) * mul);
                        w4.z = pack_bf16x2(__uint_as_float(r[8 * x + 4]) * mul, __uint_as_float(r[8 * x + 5]) * mul);
                        w4.w = pack_bf16x2(__uint_as_float(r[8 * x + 6]) * mul, __uint_as_float(r[8 * x + 7]) * mul);
                        dst[x] = w4;
                    }
                }
            }
        }
    } else {
        // ------------------------------------------------ dQ drain: TMEM lane d
        // holds dQ^T[d][0..63]; each warp writes its 32 columns d into one
        // swizzled [64 query][32 d] block, then one thread adds the four
        // blocks into the float32 accumulator.
        const int quad = warp & 3;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const bool leader = (warp == 10 && lane == 0);
        const uint32_t blk = smem_u32(sm.stage[quad]);
        const uint32_t chunk = (uint32_t)(lane >> 2), within = (uint32_t)(lane & 3) * 4;
        for (int idx = 0; idx < n_q; ++idx) {
            const bool ok = __all_sync(0xffffffffu, mbar_wait(&sm.dq_full, (uint32_t)idx & 1u, err, abort));
            if (!ok) break;
            tc_fence_after();
            uint32_t r[2][32];
            tmem_ld32(tdQ + lane_off, r[0]);
            tmem_ld32(tdQ + lane_off + 32, r[1]);
            tmem_wait_ld();
            reg_fence32(r[0]);
            reg_fence32(r[1]);
            tc_fence_before();
            mbar_arrive(&sm.dq_free);
            if (leader) bulk_wait_read_all();  // the previous reduce has read the staging blocks
            named_bar_sync(1, 128);
#pragma unroll
            for (int qq = 0; qq < kBQ; ++qq) {
                const uint32_t addr = blk + (uint32_t)qq * 128 + ((chunk ^ (uint32_t)(qq & 7)) << 4) + within;
                asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(r[qq >> 5][qq & 31]) : "memory");
            }
            fence_proxy_async_smem();
            named_bar_sync(1, 128);
            if (leader) {
                ATTN_DCHECK((q_first + idx) * kBQ < T, err);
                for (int db = 0; db < 4; ++db)
                    tma_reduce_add_3d(&tdq, sm.stage[db], 32 * db, (q_first + idx) * kBQ, bh);
                bulk_commit();
            }
        }
        if (leader) bulk_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// 4-D bf16 map over (D, T, H, B) with a box of 64 columns x `rows` rows,
// 128-byte swizzle.
cudaError_t make_map_rows(CUtensorMap *map, const void *ptr, const Shape &s, const TStrides &st,
                          int rows) {
    auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
    if (!enc) return cudaErrorInitializationError;
    const cuuint64_t dims[4] = {(cuuint64_t)s.D, (cuuint64_t)s.T, (cuuint64_t)s.H, (cuuint64_t)s.B};
    const cuuint64_t strides[3] = {(cuuint64_t)st.t * 2, (cuuint64_t)st.h * 2, (cuuint64_t)st.b * 2};
    const cuuint32_t box[4] = {64, (cuuint32_t)rows, 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(ptr), dims,
                           strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// The float32 dQ accumulator [BH, T, 128] as a 3-D map, box 32 x 64, 128-byte swizzle.
cudaError_t make_map_dq(CUtensorMap *map, float *ptr, int BH, int T) {
    auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
    if (!enc) return cudaErrorInitializationError;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)T, (cuuint64_t)BH};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)T * D * 4};
    const cuuint32_t box[3] = {32, (cuuint32_t)kBQ, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, ptr, dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <bool Causal, bool Drop>
cudaError_t launch128(const __nv_bfloat16 *q, const __nv_bfloat16 *k, const __nv_bfloat16 *v,
                      const __nv_bfloat16 *dO, __nv_bfloat16 *dk, __nv_bfloat16 *dv, float *dq_acc,
                      const float *lse2, const float *delta, const Shape &s, const BwdStrides &str,
                      int *err, cudaStream_t st, LaunchInfo &li) {
    const int BH = s.B * s.H;
    const int nkt = (s.T + kBK - 1) / kBK;
    const int nqt = (s.T + kBQ - 1) / kBQ;
    const int Tpad = nkt * kBK;
    const long long blocks = (long long)nkt * BH;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    CUtensorMap mq, mk, mv, mdo, mdq;
    cudaError_t e;
    if ((e = make_map_rows(&mq, q, s, str.q, kBQ)) != cudaSuccess) return e;
    if ((e = make_map_rows(&mk, k, s, str.k, kBK)) != cudaSuccess) return e;
    if ((e = make_map_rows(&mv, v, s, str.v, kBK)) != cudaSuccess) return e;
    if ((e = make_map_rows(&mdo, dO, s, str.dO, kBQ)) != cudaSuccess) return e;
    if ((e = make_map_dq(&mdq, dq_acc, BH, s.T)) != cudaSuccess) return e;
    const size_t smem = sizeof(Smem128) + 1024;
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    static std::atomic<unsigned long long> smem_set{0};
    if ((e = set_max_smem_once(reinterpret_cast<const void *>(bwd128_main_kernel<Causal, Drop>), smem, dev,
                               smem_set)) != cudaSuccess)
        return e;
    if ((e = mark_main_start(li, st)) != cudaSuccess) return e;
    if ((e = launch_pdl(bwd128_main_kernel<Causal, Drop>, dim3((unsigned)blocks), dim3(kThreads), smem,
                        st, mq, mk, mv, mdo, mdq, lse2, delta, dk, dv, str.dk, str.dv, s.T, Tpad, s.H,
                        BH, nqt, s.scale * kLog2e, s.scale, s.drop, err)) != cudaSuccess)
        return e;
    li.kernels += 1;
    return mark_main_end(li, st);
}

}  // namespace

cudaError_t sm100_bwd128_main(const __nv_bfloat16 *q, const __nv_bfloat16 *k,
                              const __nv_bfloat16 *v, const __nv_bfloat16 *dO, __nv_bfloat16 *dk,
                              __nv_bfloat16 *dv, float *dq_acc, const float *lse2,
                              const float *delta, const Shape &s, const BwdStrides &str, int *err,
                              cudaStream_t st, LaunchInfo &li) {
    if (s.D != D) return cudaErrorInvalidValue;
    if (s.causal)
        return s.dropout ? launch128<true, true>(q, k, v, dO, dk, dv, dq_acc, lse2, delta, s, str, err, st, li)
                         : launch128<true, false>(q, k, v, dO, dk, dv, dq_acc, lse2, delta, s, str, err, st, li);
    return s.dropout ? launch128<false, true>(q, k, v, dO, dk, dv, dq_acc, lse2, delta, s, str, err, st, li)
                     : launch128<false, false>(q, k, v, dO, dk, dv, dq_acc, lse2, delta, s, str, err, st, li);
}

}  // namespace attn
