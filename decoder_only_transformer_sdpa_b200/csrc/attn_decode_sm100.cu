// attn_decode_sm100.cu -- decode-shape attention on B200: the Tq newest
// tokens' queries (Tq <= 16) against the keys and values of all Tk tokens.
//
// Text generation appends one token at a time, and each new token's query
// attends to every earlier token and to itself ("nanoGPT — 架构与原理",
// section 5 "边界与局限": generate recomputes the whole forward per token, with
// no KV cache; "How Andrej Karpathy built GPT from 200 lines of code", section
// "Self-Attention: the mathematical trick" [55:20] for the causal mask).  Kept
// keys and values make one new token cost one row of the causal attention:
// query r (position Tk - Tq + r) sees keys 0 .. Tk - Tq + r.
//
// The work is a stream over the cached K and V (4 * Tk * D bytes per head)
// with a few flops per byte, so the kernel is built to keep HBM busy:
//   * one thread-block cluster of cs <= 8 CTAs per head; CTA c takes the
//     128-key tiles c, c + cs, ... (split over the keys, so ~2 CTAs per SM
//     stream at once even for a handful of heads);
//   * a producer warp brings K and V tiles through a 3-stage TMA ring
//     (full/empty mbarriers), swizzled like the other kernels' tiles, so the
//     row-wise score reads and the column-pair PV reads are free of bank
//     conflicts;
//   * the kernel is compiled per query bucket NQ in {1, 2, 4, 8, 16} (the
//     next power of two >= Tq; padding queries are zero rows whose results
//     are dropped), so every per-query loop is unrolled without branches;
//   * eight consumer warps each own 16 keys of every tile and run scores (two
//     lanes per key row), an online softmax (log2 units) over their keys and
//     P V entirely in registers and shuffles, with no CTA-wide barrier in the
//     tile loop, so the warps' latency chains overlap;
//   * the warps' (max, sum, unnormalised O) merge within the CTA, and the cs
//     CTAs' merge in CTA 0 of the cluster through distributed shared memory,
//     so there is no workspace, no atomic and no second launch.
#include "internal.h"
#include "sm100.cuh"

#include <cooperative_groups.h>
#include <cudaTypedefs.h>

namespace attn {
namespace {

using namespace sm100;
namespace cg = cooperative_groups;

constexpr int kTile = 128;         // keys per TMA tile
constexpr int kStages = 3;         // K/V ring depth
constexpr int kWarps = 8;          // consumer warps: warp g owns keys 16 g .. 16 g + 15 of a tile
constexpr int kKeys = kTile / kWarps;
constexpr int kThreads = 32 * (kWarps + 1);  // + one TMA producer warp
constexpr int kMaxCluster = 8;     // portable cluster size
constexpr float kLog2e = 1.4426950408889634f;

// Byte offset of 16-byte chunk c of row t in a TMA tile of D * 2-byte rows
// written with the 128-byte (D = 64) or 64-byte (D = 32) swizzle.
template <int D>
__device__ __forceinline__ uint32_t swz(int t, int c) {
    if constexpr (D == 64)
        return (uint32_t)(t * 128 + ((c ^ (t & 7)) << 4));
    else
        return (uint32_t)(t * 64 + ((c ^ ((t >> 1) & 3)) << 4));
}

template <int D, int NQ>
struct DecSmem {
    static constexpr int kTileBytes = kTile * D * 2;
    // K and V rings (contiguous: after the tiles they hold the warps' partial
    // O, [warp][NQ][D] floats)
    alignas(1024) __nv_bfloat16 k[kStages][kTile * D];
    alignas(1024) __nv_bfloat16 v[kStages][kTile * D];
    // queries times scale * log2(e), zero rows past Tq, as two half rows; the
    // pad puts the halves on different banks (the two lanes of a key read one
    // half each with the same instruction)
    float q[NQ][2][D / 2 + 4];
    float mw[kWarps][NQ], lw[kWarps][NQ];  // per warp: running max (log2 units), sum
    float o[NQ][D];                 // this CTA's unnormalised partial O
    float mc[NQ], lc[NQ];           // this CTA's max and sum (read by CTA 0 of the cluster)
    uint64_t full[kStages], empty[kStages];
    int abort;
};

template <int D, int NQ>
__global__ void __launch_bounds__(kThreads)
    decode_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                  const __nv_bfloat16 *__restrict__ q, const TStrides sq,
                  __nv_bfloat16 *__restrict__ o, const TStrides so, float *__restrict__ lse, int H,
                  int Tq, int Tk, int ntiles, float qscale, int *err) {
    using Smem = DecSmem<D, NQ>;
    constexpr int kChunks = D / 8;            // 16-byte chunks per row
    constexpr int kHalfChunks = kChunks / 2;  // chunks per score lane (two lanes per key)
    constexpr int kPairs = D / 2;             // output column pairs
    constexpr int kSplit = 32 / kPairs;       // PV: lanes sharing a column pair (1 or 2)
    constexpr int kSubKeys = kKeys / kSplit;  // PV: keys per lane
    static_assert(kKeys == 16, "two score lanes per key, 16 keys per warp");
    static_assert(sizeof(float) * kWarps * NQ * D <= 2 * kStages * kTile * D * 2,
                  "warp partials must fit in the K/V rings");
    extern __shared__ uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                         ~uintptr_t(1023));
    volatile int *abort = &sm.abort;
    cg::cluster_group cluster = cg::this_cluster();
    const int cs = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    const int bh = (int)(blockIdx.x / cs);
    const int bb = bh / H, hh = bh % H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // This CTA's tiles: rank, rank + cs, ... (tile 0, which every query sees,
    // is always in CTA 0).
    const int my_tiles = rank < ntiles ? (ntiles - 1 - rank) / cs + 1 : 0;
    ATTN_DCHECK(bb >= 0 && hh >= 0 && hh < H && cs <= kMaxCluster, err);

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], kWarps);
        }
        sm.abort = 0;
        fence_mbar_init();
        prefetch_tensormap(&tk);
        prefetch_tensormap(&tv);
    }
    grid_dep_wait();
    grid_dep_launch();
    if (tid == 0) {
        // The first tiles start streaming before anything else happens.
        for (int n = 0; n < kStages && n < my_tiles; ++n) {
            const int tile = rank + n * cs;
            ATTN_DCHECK(tile >= 0 && tile < ntiles, err);
            mbar_arrive_expect_tx(&sm.full[n], 2 * Smem::kTileBytes);
            tma_load_4d(sm.k[n], &tk, &sm.full[n], 0, tile * kTile, hh, bb);
            tma_load_4d(sm.v[n], &tv, &sm.full[n], 0, tile * kTile, hh, bb);
        }
    }
    // Queries, pre-scaled into log2 units (zero rows past Tq).
    for (int e = tid; e < NQ * kChunks; e += kThreads) {
        const int r = e / kChunks, c = e - r * kChunks;
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        if (r < Tq)
            w = *reinterpret_cast<const uint4 *>(q + (long long)bb * sq.b + (long long)hh * sq.h +
                                                 (long long)r * sq.t + 8 * c);
        const __nv_bfloat162 *w2 = reinterpret_cast<const __nv_bfloat162 *>(&w);
        float *dst = &sm.q[r][(8 * c) / (D / 2)][(8 * c) % (D / 2)];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const float2 f = __bfloat1622float2(w2[x]);
            dst[2 * x] = f.x * qscale;
            dst[2 * x + 1] = f.y * qscale;
        }
    }
    __syncthreads();

    bool ok = true;
    // Consumer state: running max, sum and O of each query over this warp's keys.
    const int cp = lane % kPairs, ks = lane / kPairs;  // PV lanes: column pair, key half
    float m_run[NQ], l_run[NQ], acc[NQ][2];
#pragma unroll
    for (int r = 0; r < NQ; ++r) {
        m_run[r] = -INFINITY;
        l_run[r] = 0.f;
        acc[r][0] = acc[r][1] = 0.f;
    }
    if (warp == kWarps) {
        // ------------------------------------------------ TMA producer
        int issued = my_tiles < kStages ? my_tiles : kStages;  // issued at the start
        if (lane == 0) {
            for (int n = kStages; n < my_tiles; ++n) {
                const int s = n % kStages;
                if (!mbar_wait(&sm.empty[s], (uint32_t)((n / kStages) - 1) & 1u, err, abort)) break;
                const int tile = rank + n * cs;
                ATTN_DCHECK(tile >= 0 && tile < ntiles, err);
                mbar_arrive_expect_tx(&sm.full[s], 2 * Smem::kTileBytes);
                tma_load_4d(sm.k[s], &tk, &sm.full[s], 0, tile * kTile, hh, bb);
                tma_load_4d(sm.v[s], &tv, &sm.full[s], 0, tile * kTile, hh, bb);
                issued = n + 1;
            }
            // The last loads have landed before the ring is reused or left
            // (on the normal path the consumers waited on all of them).
            for (int n = issued > kStages ? issued - kStages : 0; n < issued; ++n)
                for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(&sm.full[n % kStages], (uint32_t)(n / kStages) & 1u); ++i) {}
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ consumer warp: keys
        // 16 warp .. +15 of every tile; scores, online softmax and P V in
        // registers and shuffles
        const int kk = lane >> 1, hf = lane & 1;  // score lanes: key kk, half hf of its row
        for (int n = 0; n < my_tiles; ++n) {
            const int s = n % kStages;
            const int tile = rank + n * cs;
            ATTN_DCHECK(tile >= 0 && tile < ntiles, err);
            if (!(ok = mbar_wait_warp(&sm.full[s], (uint32_t)(n / kStages) & 1u, err, abort))) break;
            const int row = warp * kKeys + kk;  // this lane pair's key row in the tile
            // ---- scores of the warp's 16 keys (two lanes per row)
            float kf[kHalfChunks * 8];
            {
                const uint32_t kbase = smem_u32(sm.k[s]);
#pragma unroll
                for (int i = 0; i < kHalfChunks; ++i) {
                    uint4 w;
                    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(w.x), "=r"(w.y), "=r"(w.z), "=r"(w.w)
                                 : "r"(kbase + swz<D>(row, hf * kHalfChunks + i)));
                    const __nv_bfloat162 *w2 = reinterpret_cast<const __nv_bfloat162 *>(&w);
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        const float2 f = __bfloat1622float2(w2[x]);
                        kf[8 * i + 2 * x] = f.x;
                        kf[8 * i + 2 * x + 1] = f.y;
                    }
                }
            }
            const int j = tile * kTile + row;
            float pw[NQ];
#pragma unroll
            for (int r = 0; r < NQ; ++r) {
                const float *qr = &sm.q[r][hf][0];
                float d0 = 0.f, d1 = 0.f;
#pragma unroll
                for (int x = 0; x < kHalfChunks * 8; x += 2) {
                    d0 = fmaf(qr[x], kf[x], d0);
                    d1 = fmaf(qr[x + 1], kf[x + 1], d1);
                }
                float d = d0 + d1;
                d += __shfl_xor_sync(0xffffffffu, d, 1);
                d = (j <= Tk - Tq + r) ? d : -INFINITY;
                // ---- online softmax over the warp's keys (lane pairs hold
                // copies: the butterflies skip offset 1)
                float mx = d;
#pragma unroll
                for (int off = 2; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                const float m_new = fmaxf(m_run[r], mx);
                const float base = (m_new == -INFINITY) ? 0.f : m_new;  // no visible key yet
                const float pv = ex2(d - base);
                float sum = pv;
#pragma unroll
                for (int off = 2; off < 32; off <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
                const float a = ex2(m_run[r] - base);
                l_run[r] = l_run[r] * a + sum;
                m_run[r] = m_new;
                acc[r][0] *= a;
                acc[r][1] *= a;
                pw[r] = pv;
            }
            // ---- P V: columns 2 cp, 2 cp + 1 over keys ks * kSubKeys .. +kSubKeys - 1
            {
                const uint32_t vbase = smem_u32(sm.v[s]);
#pragma unroll
                for (int t = 0; t < kSubKeys; ++t) {
                    const int key = ks * kSubKeys + t;  // this lane's key of the warp's 16
                    const int vr = warp * kKeys + key;
                    uint32_t w;
                    asm volatile("ld.shared.u32 %0, [%1];"
                                 : "=r"(w)
                                 : "r"(vbase + swz<D>(vr, cp >> 2) + ((cp & 3) << 2)));
                    const float2 vf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w));
#pragma unroll
                    for (int r = 0; r < NQ; ++r) {
                        const float pk = __shfl_sync(0xffffffffu, pw[r], 2 * key);
                        acc[r][0] = fmaf(pk, vf.x, acc[r][0]);
                        acc[r][1] = fmaf(pk, vf.y, acc[r][1]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[s]);  // this warp is done with stage s
        }
        // ---- this warp's (max, sum, partial O) into shared memory; the K/V
        // rings take the partials once every warp is done with every tile
        if (kSplit == 2) {
#pragma unroll
            for (int r = 0; r < NQ; ++r) {
                acc[r][0] += __shfl_xor_sync(0xffffffffu, acc[r][0], 16);
                acc[r][1] += __shfl_xor_sync(0xffffffffu, acc[r][1], 16);
            }
        }
        ok = __all_sync(0xffffffffu, ok);
    }
    __syncthreads();
    if (warp < kWarps) {
        float *part = reinterpret_cast<float *>(&sm.k[0][0]);  // [kWarps][NQ][D]
        if (lane < kPairs) {
#pragma unroll
            for (int r = 0; r < NQ; ++r) {
                part[(warp * NQ + r) * D + 2 * cp] = ok ? acc[r][0] : 0.f;
                part[(warp * NQ + r) * D + 2 * cp + 1] = ok ? acc[r][1] : 0.f;
            }
        }
        if (lane == 0) {
#pragma unroll
            for (int r = 0; r < NQ; ++r) {
                sm.mw[warp][r] = m_run[r];
                sm.lw[warp][r] = ok ? l_run[r] : 0.f;
            }
        }
    }
    __syncthreads();
    // ---- merge the warps into this CTA's (max, sum, partial O)
    {
        const float *part = reinterpret_cast<const float *>(&sm.k[0][0]);
        for (int e = tid; e < NQ * D; e += kThreads) {
            const int r = e / D;
            float mm = -INFINITY;
#pragma unroll
            for (int g = 0; g < kWarps; ++g) mm = fmaxf(mm, sm.mw[g][r]);
            float t = 0.f, L = 0.f;
#pragma unroll
            for (int g = 0; g < kWarps; ++g) {
                const float mg = sm.mw[g][r];
                const float wgt = (mg == -INFINITY) ? 0.f : ex2(mg - mm);
                t = fmaf(wgt, part[(g * NQ + r) * D + (e - r * D)], t);
                L = fmaf(wgt, sm.lw[g][r], L);
            }
            sm.o[r][e - r * D] = t;
            if (e - r * D == 0) {
                sm.mc[r] = mm;
                sm.lc[r] = L;
            }
        }
    }
    // ---- merge the cluster's CTAs in CTA 0 (distributed shared memory)
    cluster.sync();
    if (rank == 0) {
        for (int e = tid; e < Tq * (D / 8); e += kThreads) {
            const int r = e / (D / 8), c = e - r * (D / 8);
            float mx[kMaxCluster];
            float mmax = -INFINITY;
#pragma unroll
            for (int x = 0; x < kMaxCluster; ++x) {
                mx[x] = x < cs ? *cluster.map_shared_rank(&sm.mc[r], x) : -INFINITY;
                mmax = fmaxf(mmax, mx[x]);
            }
            float L = 0.f, out[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int x = 0; x < kMaxCluster; ++x) {
                if (x < cs) {
                    const float wgt = (mx[x] == -INFINITY) ? 0.f : ex2(mx[x] - mmax);
                    L = fmaf(wgt, *cluster.map_shared_rank(&sm.lc[r], x), L);
                    const float4 *ox = reinterpret_cast<const float4 *>(
                        cluster.map_shared_rank(&sm.o[r][8 * c], x));
                    const float4 a = ox[0], b = ox[1];
                    out[0] = fmaf(wgt, a.x, out[0]);
                    out[1] = fmaf(wgt, a.y, out[1]);
                    out[2] = fmaf(wgt, a.z, out[2]);
                    out[3] = fmaf(wgt, a.w, out[3]);
                    out[4] = fmaf(wgt, b.x, out[4]);
                    out[5] = fmaf(wgt, b.y, out[5]);
                    out[6] = fmaf(wgt, b.z, out[6]);
                    out[7] = fmaf(wgt, b.w, out[7]);
                }
            }
            const float inv = 1.f / L;
            uint4 w4;
            w4.x = pack_bf16x2(out[0] * inv, out[1] * inv);
            w4.y = pack_bf16x2(out[2] * inv, out[3] * inv);
            w4.z = pack_bf16x2(out[4] * inv, out[5] * inv);
            w4.w = pack_bf16x2(out[6] * inv, out[7] * inv);
            *reinterpret_cast<uint4 *>(o + (long long)bb * so.b + (long long)hh * so.h +
                                       (long long)r * so.t + 8 * c) = w4;
            if (c == 0) lse[(size_t)bh * Tq + r] = (mmax + log2f(L)) * 0.69314718055994531f;
        }
    }
    cluster.sync();  // the other CTAs keep their shared memory until CTA 0 has read it
}

template <int D, int NQ>
cudaError_t launch_decode(const __nv_bfloat16 *q, const __nv_bfloat16 *k, const __nv_bfloat16 *v,
                          __nv_bfloat16 *o, float *lse, const DecodeShape &s,
                          const FwdStrides &str, int *err, cudaStream_t st, LaunchInfo &li) {
    const int BH = s.B * s.H;
    const int ntiles = (s.Tk + kTile - 1) / kTile;
    int dev = 0, sms = 0;
    cudaError_t e;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    // Cluster size: enough CTAs for ~2 per SM, at most one per tile and 8.
    int cs = (2 * sms) / BH;
    cs = cs < 1 ? 1 : cs;
    cs = cs > kMaxCluster ? kMaxCluster : cs;
    cs = cs > ntiles ? ntiles : cs;
    const long long grid = (long long)BH * cs;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    CUtensorMap mk, mv;
    const Shape kv{s.B, s.H, s.Tk, D, s.scale};
    if ((e = make_map_bf16(&mk, k, kv, str.k)) != cudaSuccess) return e;
    if ((e = make_map_bf16(&mv, v, kv, str.v)) != cudaSuccess) return e;
    const size_t smem = sizeof(DecSmem<D, NQ>) + 1024;
    static std::atomic<unsigned long long> smem_set{0};
    if ((e = set_max_smem_once(reinterpret_cast<const void *>(decode_kernel<D, NQ>), smem, dev, smem_set)) !=
        cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // Programmatic stream serialisation: the kernel's prologue may overlap the
    // previous grid's tail (it calls grid_dep_wait before touching memory).
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const float qscale = s.scale * kLog2e;
    if ((e = mark_main_start(li, st)) != cudaSuccess) return e;
    e = cudaLaunchKernelEx(&cfg, decode_kernel<D, NQ>, mk, mv, q, str.q, o, str.o, lse, s.H, s.Tq,
                           s.Tk, ntiles, qscale, err);
    if (e != cudaSuccess) return e;
    li.kernels += 1;
    return mark_main_end(li, st);
}

}  // namespace

cudaError_t sm100_decode(const __nv_bfloat16 *q, const __nv_bfloat16 *k, const __nv_bfloat16 *v,
                         __nv_bfloat16 *o, float *lse, const DecodeShape &s, const FwdStrides &str,
                         int *err, cudaStream_t st, LaunchInfo &li) {
#define ATTN_DECODE_CASE(DD, NN)                                          \
    if (s.D == DD && s.Tq <= NN)                                         \
        return launch_decode<DD, NN>(q, k, v, o, lse, s, str, err, st, li);
    ATTN_DECODE_CASE(64, 1)
    ATTN_DECODE_CASE(64, 2)
    ATTN_DECODE_CASE(64, 4)
    ATTN_DECODE_CASE(64, 8)
    ATTN_DECODE_CASE(64, 16)
    ATTN_DECODE_CASE(32, 1)
    ATTN_DECODE_CASE(32, 2)
    ATTN_DECODE_CASE(32, 4)
    ATTN_DECODE_CASE(32, 8)
    ATTN_DECODE_CASE(32, 16)
#undef ATTN_DECODE_CASE
    return cudaErrorInvalidValue;
}

}  // namespace attn
