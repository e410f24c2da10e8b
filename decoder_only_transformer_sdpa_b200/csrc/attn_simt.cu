// attn_simt.cu -- causal attention forward and backward on CUDA cores.
//
// This is the float32 path (IEEE expf/logf, fp32 FMAs, no fast-math), used
// for float32 tensors of any head_dim up to 128.  The same templates also
// instantiate for bf16 storage with float32 arithmetic.
//
// Method: "How Andrej Karpathy built GPT from 200 lines of code", sections
// "Self-Attention: the mathematical trick" [55:20] and "Implementing the
// attention heads (Query, Key, Value)" [1:06:16]-[1:17:18]: scores q.k scaled
// by 1/sqrt(head size), future positions masked, softmax, weighted sum of
// values.  Here each thread owns one query row and walks the keys j <= i once
// with a running maximum and running sum (online softmax), so the T x T score
// matrix never exists in memory.  The backward recomputes P_ij from the saved
// lse_i and follows the exact derivative.  With causal = 0 the same kernels
// run every row over all T keys (every key over all T queries).  With drop
// set, attention dropout on the weights uses the keep bits of philox.cuh:
// row sums take every weight, O and dV only the kept ones, scaled by the
// keep scale.
//
// Block = 64 threads = 64 rows of one head; K/V (or Q/dO) tiles of 64 rows
// are staged in shared memory as float32 and shared by the block.
#include "internal.h"

#include <math.h>

namespace attn {
namespace {

constexpr int kRows = 64;

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void from_f(float *p, float x) { *p = x; }
__device__ __forceinline__ void from_f(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

// Tiles are visited heaviest first: under the causal mask row tile t costs t+1
// key tiles, so launching the last tiles first evens out the tail.
__device__ __forceinline__ void tile_and_head(int ntiles, int &tile, long long &bh) {
    const long long b = blockIdx.x;
    bh = b / ntiles;
    tile = ntiles - 1 - (int)(b - bh * ntiles);
}

template <typename T>
__device__ __forceinline__ void stage_rows(float *dst, const T *src, int row0, int nrows_total,
                                           int D) {
    for (int e = threadIdx.x; e < kRows * D; e += blockDim.x) {
        const int r = e / D;
        const int row = row0 + r;
        dst[e] = row < nrows_total ? to_f(src[(size_t)row * D + (e - r * D)]) : 0.f;
    }
}

template <typename T, int DMAX>
__global__ void __launch_bounds__(kRows) fwd_kernel(const T *__restrict__ q, const T *__restrict__ k,
                                                    const T *__restrict__ v, T *__restrict__ o,
                                                    float *__restrict__ lse, int Tn, int D,
                                                    float scale, int causal, int drop,
                                                    DropoutParams dp) {
    extern __shared__ float smem[];
    float *ks = smem;
    float *vs = smem + kRows * D;
    const int ntiles = (Tn + kRows - 1) / kRows;
    int tile;
    long long bh;
    tile_and_head(ntiles, tile, bh);
    const size_t base = (size_t)bh * Tn * D;
    const int i = tile * kRows + threadIdx.x;
    const bool row_ok = i < Tn;

    float qr[DMAX], acc[DMAX];
#pragma unroll
    for (int d = 0; d < DMAX; ++d) {
        qr[d] = (row_ok && d < D) ? to_f(q[base + (size_t)i * D + d]) : 0.f;
        acc[d] = 0.f;
    }
    float m = -INFINITY, l = 0.f;
    const int last_key = causal ? min(tile * kRows + kRows, Tn) - 1 : Tn - 1;
    const int my_last = causal ? i : Tn - 1;
    for (int j0 = 0; j0 <= last_key; j0 += kRows) {
        __syncthreads();
        stage_rows(ks, k + base, j0, Tn, D);
        stage_rows(vs, v + base, j0, Tn, D);
        __syncthreads();
        if (row_ok) {
            const int jend = min(j0 + kRows - 1, my_last);
            uint32_t kb = 0xFFu;  // keep bits of keys (j & ~7) .. +7
            for (int j = j0; j <= jend; ++j) {
                const float *kj = ks + (j - j0) * D;
                const float *vj = vs + (j - j0) * D;
                if (drop && (j & 7) == 0)
                    kb = philox::keep_byte(dp, (uint32_t)i, (uint32_t)j >> 3, (uint32_t)bh);
                float s = 0.f;
#pragma unroll
                for (int d = 0; d < DMAX; ++d)
                    if (d < D) s = fmaf(qr[d], kj[d], s);
                s *= scale;
                const float mn = fmaxf(m, s);
                const float corr = expf(m - mn);
                const float p = expf(s - mn);
                l = fmaf(l, corr, p);
                const float pz = ((kb >> (j & 7)) & 1u) ? p : 0.f;
#pragma unroll
                for (int d = 0; d < DMAX; ++d)
                    if (d < D) acc[d] = fmaf(pz, vj[d], acc[d] * corr);
                m = mn;
            }
        }
    }
    if (row_ok) {
        const float inv = (drop ? dp.keep_scale : 1.f) / l;
#pragma unroll
        for (int d = 0; d < DMAX; ++d)
            if (d < D) from_f(&o[base + (size_t)i * D + d], acc[d] * inv);
        lse[(size_t)bh * Tn + i] = m + logf(l);
    }
}

// Delta_i = <dO_i, O_i> (float32), one thread per row.
template <typename T>
__global__ void delta_kernel(const T *__restrict__ o, const T *__restrict__ dO,
                             float *__restrict__ delta, long long rows, int D) {
    const long long r = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= rows) return;
    float acc = 0.f;
    for (int d = 0; d < D; ++d) acc = fmaf(to_f(dO[r * D + d]), to_f(o[r * D + d]), acc);
    delta[r] = acc;
}

// dQ_i = scale * sum_{j<=i} P_ij (dP_ij - Delta_i) k_j (all j when not
// causal), thread per query row.
template <typename T, int DMAX>
__global__ void __launch_bounds__(kRows) dq_kernel(const T *__restrict__ q, const T *__restrict__ k,
                                                   const T *__restrict__ v, const float *__restrict__ lse,
                                                   const T *__restrict__ dO,
                                                   const float *__restrict__ delta, T *__restrict__ dq,
                                                   int Tn, int D, float scale, int causal, int drop,
                                                   DropoutParams dp) {
    extern __shared__ float smem[];
    float *ks = smem;
    float *vs = smem + kRows * D;
    const int ntiles = (Tn + kRows - 1) / kRows;
    int tile;
    long long bh;
    tile_and_head(ntiles, tile, bh);
    const size_t base = (size_t)bh * Tn * D;
    const int i = tile * kRows + threadIdx.x;
    const bool row_ok = i < Tn;

    float qr[DMAX], gr[DMAX], acc[DMAX];
#pragma unroll
    for (int d = 0; d < DMAX; ++d) {
        qr[d] = (row_ok && d < D) ? to_f(q[base + (size_t)i * D + d]) : 0.f;
        gr[d] = (row_ok && d < D) ? to_f(dO[base + (size_t)i * D + d]) : 0.f;
        acc[d] = 0.f;
    }
    const float lse_i = row_ok ? lse[(size_t)bh * Tn + i] : 0.f;
    const float delta_i = row_ok ? delta[(size_t)bh * Tn + i] : 0.f;
    const int last_key = causal ? min(tile * kRows + kRows, Tn) - 1 : Tn - 1;
    const int my_last = causal ? i : Tn - 1;
    for (int j0 = 0; j0 <= last_key; j0 += kRows) {
        __syncthreads();
        stage_rows(ks, k + base, j0, Tn, D);
        stage_rows(vs, v + base, j0, Tn, D);
        __syncthreads();
        if (row_ok) {
            const int jend = min(j0 + kRows - 1, my_last);
            uint32_t kb = 0xFFu;
            for (int j = j0; j <= jend; ++j) {
                const float *kj = ks + (j - j0) * D;
                const float *vj = vs + (j - j0) * D;
                if (drop && (j & 7) == 0)
                    kb = philox::keep_byte(dp, (uint32_t)i, (uint32_t)j >> 3, (uint32_t)bh);
                float s = 0.f, dpv = 0.f;
#pragma unroll
                for (int d = 0; d < DMAX; ++d)
                    if (d < D) {
                        s = fmaf(qr[d], kj[d], s);
                        dpv = fmaf(gr[d], vj[d], dpv);
                    }
                const float p = expf(s * scale - lse_i);
                const float dz = drop ? (((kb >> (j & 7)) & 1u) ? dp.keep_scale * dpv : 0.f) : dpv;
                const float ds = p * (dz - delta_i);
#pragma unroll
                for (int d = 0; d < DMAX; ++d)
                    if (d < D) acc[d] = fmaf(ds, kj[d], acc[d]);
            }
        }
    }
    if (row_ok) {
#pragma unroll
        for (int d = 0; d < DMAX; ++d)
            if (d < D) from_f(&dq[base + (size_t)i * D + d], acc[d] * scale);
    }
}

// dV_j = sum_{i>=j} P_ij dO_i and dK_j = scale * sum_{i>=j} dS_ij q_i (all i
// when not causal), thread per key row.
template <typename T, int DMAX>
__global__ void __launch_bounds__(kRows) dkdv_kernel(const T *__restrict__ q, const T *__restrict__ k,
                                                     const T *__restrict__ v,
                                                     const float *__restrict__ lse,
                                                     const T *__restrict__ dO,
                                                     const float *__restrict__ delta,
                                                     T *__restrict__ dk, T *__restrict__ dv, int Tn,
                                                     int D, float scale, int causal, int drop,
                                                     DropoutParams dp) {
    extern __shared__ float smem[];
    float *qs = smem;
    float *gs = smem + kRows * D;
    float *ls = smem + 2 * kRows * D;
    float *ds_ = ls + kRows;
    const int ntiles = (Tn + kRows - 1) / kRows;
    int tile;
    long long bh;
    {
        // key tiles near the start see the most query rows: launch them first
        const long long b = blockIdx.x;
        bh = b / ntiles;
        tile = (int)(b - bh * ntiles);
    }
    const size_t base = (size_t)bh * Tn * D;
    const int j = tile * kRows + threadIdx.x;
    const bool row_ok = j < Tn;

    float kr[DMAX], vr[DMAX], dka[DMAX], dva[DMAX];
#pragma unroll
    for (int d = 0; d < DMAX; ++d) {
        kr[d] = (row_ok && d < D) ? to_f(k[base + (size_t)j * D + d]) : 0.f;
        vr[d] = (row_ok && d < D) ? to_f(v[base + (size_t)j * D + d]) : 0.f;
        dka[d] = 0.f;
        dva[d] = 0.f;
    }
    for (int i0 = causal ? tile * kRows : 0; i0 < Tn; i0 += kRows) {
        __syncthreads();
        stage_rows(qs, q + base, i0, Tn, D);
        stage_rows(gs, dO + base, i0, Tn, D);
        for (int r = threadIdx.x; r < kRows; r += blockDim.x) {
            const int row = i0 + r;
            ls[r] = row < Tn ? lse[(size_t)bh * Tn + row] : 0.f;
            ds_[r] = row < Tn ? delta[(size_t)bh * Tn + row] : 0.f;
        }
        __syncthreads();
        if (row_ok) {
            const int iend = min(i0 + kRows, Tn);
            for (int i = causal ? max(i0, j) : i0; i < iend; ++i) {
                const float *qi = qs + (i - i0) * D;
                const float *gi = gs + (i - i0) * D;
                float s = 0.f, dpv = 0.f;
#pragma unroll
                for (int d = 0; d < DMAX; ++d)
                    if (d < D) {
                        s = fmaf(qi[d], kr[d], s);
                        dpv = fmaf(gi[d], vr[d], dpv);
                    }
                const float p = expf(s * scale - ls[i - i0]);
                bool keep = true;
                if (drop)
                    keep = (philox::keep_byte(dp, (uint32_t)i, (uint32_t)j >> 3, (uint32_t)bh) >>
                            (j & 7)) & 1u;
                const float dz = drop ? (keep ? dp.keep_scale * dpv : 0.f) : dpv;
                const float dsv = p * (dz - ds_[i - i0]);
                const float pz = keep ? p : 0.f;
#pragma unroll
                for (int d = 0; d < DMAX; ++d)
                    if (d < D) {
                        dva[d] = fmaf(pz, gi[d], dva[d]);
                        dka[d] = fmaf(dsv, qi[d], dka[d]);
                    }
            }
        }
    }
    if (row_ok) {
#pragma unroll
        for (int d = 0; d < DMAX; ++d)
            if (d < D) {
                from_f(&dk[base + (size_t)j * D + d], dka[d] * scale);
                from_f(&dv[base + (size_t)j * D + d], dva[d] * (drop ? dp.keep_scale : 1.f));
            }
    }
}

}  // namespace

#define ATTN_SIMT_DISPATCH(D, KERN, T)                      \
    ((D) <= 16   ? (void *)&KERN<T, 16>                      \
     : (D) <= 32 ? (void *)&KERN<T, 32>                      \
     : (D) <= 64 ? (void *)&KERN<T, 64>                      \
                 : (void *)&KERN<T, 128>)

template <typename T>
cudaError_t simt_fwd(const T *q, const T *k, const T *v, T *o, float *lse, Shape s,
                     cudaStream_t st, LaunchInfo &li) {
    const int ntiles = (s.T + kRows - 1) / kRows;
    const long long blocks = (long long)s.B * s.H * ntiles;
    const size_t smem = 2ull * kRows * s.D * sizeof(float);
    const void *fn = ATTN_SIMT_DISPATCH(s.D, fwd_kernel, T);
    int drop = s.dropout ? 1 : 0;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    void *args[] = {(void *)&q, (void *)&k, (void *)&v, (void *)&o, (void *)&lse,
                    (void *)&s.T, (void *)&s.D, (void *)&s.scale, (void *)&s.causal,
                    (void *)&drop, (void *)&s.drop};
    if ((e = mark_main_start(li, st)) != cudaSuccess) return e;
    e = cudaLaunchKernel(fn, dim3((unsigned)blocks), dim3(kRows), args, smem, st);
    if (e != cudaSuccess) return e;
    li.kernels += 1;
    return mark_main_end(li, st);
}

template <typename T>
cudaError_t simt_bwd(const T *q, const T *k, const T *v, const T *o, const float *lse,
                     const T *dO, T *dq, T *dk, T *dv, float *delta, Shape s,
                     cudaStream_t st, LaunchInfo &li) {
    const long long rows = (long long)s.B * s.H * s.T;
    const int ntiles = (s.T + kRows - 1) / kRows;
    const long long blocks = (long long)s.B * s.H * ntiles;
    int drop = s.dropout ? 1 : 0;
    delta_kernel<T><<<(unsigned)((rows + 255) / 256), 256, 0, st>>>(o, dO, delta, rows, s.D);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    li.kernels += 1;

    const size_t smem_dq = 2ull * kRows * s.D * sizeof(float);
    const void *fdq = ATTN_SIMT_DISPATCH(s.D, dq_kernel, T);
    e = cudaFuncSetAttribute(fdq, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_dq);
    if (e != cudaSuccess) return e;
    const float *delta_c = delta;
    void *a1[] = {(void *)&q, (void *)&k, (void *)&v, (void *)&lse, (void *)&dO,
                  (void *)&delta_c, (void *)&dq, (void *)&s.T, (void *)&s.D, (void *)&s.scale,
                  (void *)&s.causal, (void *)&drop, (void *)&s.drop};
    e = cudaLaunchKernel(fdq, dim3((unsigned)blocks), dim3(kRows), a1, smem_dq, st);
    if (e != cudaSuccess) return e;
    li.kernels += 1;

    const size_t smem_kv = (2ull * kRows * s.D + 2 * kRows) * sizeof(float);
    const void *fkv = ATTN_SIMT_DISPATCH(s.D, dkdv_kernel, T);
    e = cudaFuncSetAttribute(fkv, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_kv);
    if (e != cudaSuccess) return e;
    void *a2[] = {(void *)&q, (void *)&k, (void *)&v, (void *)&lse, (void *)&dO,
                  (void *)&delta_c, (void *)&dk, (void *)&dv, (void *)&s.T, (void *)&s.D,
                  (void *)&s.scale, (void *)&s.causal, (void *)&drop, (void *)&s.drop};
    if ((e = mark_main_start(li, st)) != cudaSuccess) return e;
    e = cudaLaunchKernel(fkv, dim3((unsigned)blocks), dim3(kRows), a2, smem_kv, st);
    if (e != cudaSuccess) return e;
    li.kernels += 1;
    return mark_main_end(li, st);
}

template cudaError_t simt_fwd<float>(const float *, const float *, const float *, float *, float *,
                                     Shape, cudaStream_t, LaunchInfo &);
template cudaError_t simt_fwd<__nv_bfloat16>(const __nv_bfloat16 *, const __nv_bfloat16 *,
                                             const __nv_bfloat16 *, __nv_bfloat16 *, float *, Shape,
                                             cudaStream_t, LaunchInfo &);
template cudaError_t simt_bwd<float>(const float *, const float *, const float *, const float *,
                                     const float *, const float *, float *, float *, float *,
                                     float *, Shape, cudaStream_t, LaunchInfo &);
template cudaError_t simt_bwd<__nv_bfloat16>(const __nv_bfloat16 *, const __nv_bfloat16 *,
                                             const __nv_bfloat16 *, const __nv_bfloat16 *,
                                             const float *, const __nv_bfloat16 *, __nv_bfloat16 *,
                                             __nv_bfloat16 *, __nv_bfloat16 *, float *, Shape,
                                             cudaStream_t, LaunchInfo &);

}  // namespace attn
