// Step 3 for fp32 inputs (D 64 or 128) and bf16 with D = 64: forward
// attention over the listed 128 x 128 tiles in fp32 FFMA (SparSTAR,
// pith.science review, "What carries the argument": only the chosen blocks
// are attended, and only forward).
//
// fp32 inputs must meet a 1e-4 max-abs tolerance, which rules out TF32
// tensor cores; this kernel keeps every product and sum in fp32.  It is the
// correctness path for the small fp32 workloads, not a performance path.
//
// One CTA per (b, h, query block), one thread per query row.  Q is staged
// transposed in shared memory ([d][row], conflict-free per-thread reads);
// each listed K/V tile is staged as fp32 and read as warp-wide broadcasts.
// Keys are processed 32 at a time with an online softmax (running max m,
// running sum l, accumulator rescaled when m grows).
#include <cuda_bf16.h>

#include "sparstar.h"
#include "sparstar_internal.h"

namespace sparstar {
namespace {

constexpr int kChunk = 32;

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}
template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

template <typename T, int D>
__global__ void __launch_bounds__(kBlock)
attn_simt_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                 int64_t Lq, int64_t Lk, int64_t nQB, int64_t nKB, float tau,
                 const int32_t *__restrict__ kv_idx, const int32_t *__restrict__ kv_cnt,
                 int64_t max_sel, T *__restrict__ out, float *__restrict__ lse,
                 int32_t *__restrict__ status) {
    extern __shared__ __align__(16) float sm[];
    float *Qs = sm;                  // [D][128]
    float *Ks = Qs + D * kBlock;     // [128][D]
    float *Vs = Ks + kBlock * D;     // [128][D]

    const int64_t bh = blockIdx.x / nQB;
    const int64_t i = blockIdx.x % nQB;
    const int r = threadIdx.x;
    const int64_t qrow = i * kBlock + r;

    for (int idx = threadIdx.x; idx < kBlock * D; idx += kBlock) {
        const int row = idx / D, d = idx % D;
        const int64_t g = i * kBlock + row;
        Qs[d * kBlock + row] = g < Lq ? to_f32(q[(bh * Lq + g) * D + d]) : 0.0f;
    }

    const int64_t list = bh * nQB + i;
    int cnt = kv_cnt[list];
    if (cnt < 0) cnt = 0;
    if (cnt > max_sel) cnt = (int)max_sel;

    float acc[D];
#pragma unroll
    for (int d = 0; d < D; ++d) acc[d] = 0.0f;
    float m = -INFINITY, l = 0.0f;
    bool any = false;

    for (int c = 0; c < cnt; ++c) {
        const int j = kv_idx[list * max_sel + c];
        if (j < 0 || j >= nKB) {
            if (threadIdx.x == 0 && status) atomicOr(status, SPARSTAR_STATUS_BAD_INDEX);
            continue;  // uniform across the CTA
        }
        __syncthreads();  // previous tile fully consumed (and Q staged)
        const int64_t t0 = (int64_t)j * kBlock;
        for (int idx = threadIdx.x; idx < kBlock * D; idx += kBlock) {
            const int row = idx / D, d = idx % D;
            const int64_t t = t0 + row;
            const bool ok = t < Lk;
            Ks[idx] = ok ? to_f32(k[(bh * Lk + t) * D + d]) : 0.0f;
            Vs[idx] = ok ? to_f32(v[(bh * Lk + t) * D + d]) : 0.0f;
        }
        __syncthreads();
        const int nvalid = (int)((Lk - t0) < kBlock ? (Lk - t0) : kBlock);
        any = true;
        for (int u0 = 0; u0 < nvalid; u0 += kChunk) {
            float s[kChunk];
#pragma unroll
            for (int u = 0; u < kChunk; ++u) s[u] = 0.0f;
            for (int d = 0; d < D; ++d) {
                const float qd = Qs[d * kBlock + r];
#pragma unroll
                for (int u = 0; u < kChunk; ++u) s[u] = fmaf(qd, Ks[(u0 + u) * D + d], s[u]);
            }
            float cmax = -INFINITY;
#pragma unroll
            for (int u = 0; u < kChunk; ++u) {
                s[u] = (u0 + u < nvalid) ? s[u] * tau : -INFINITY;
                cmax = fmaxf(cmax, s[u]);
            }
            const float m_new = fmaxf(m, cmax);
            const float corr = expf(m - m_new);  // 0 on the first chunk
            l *= corr;
#pragma unroll
            for (int d = 0; d < D; ++d) acc[d] *= corr;
            m = m_new;
#pragma unroll
            for (int u = 0; u < kChunk; ++u) {
                s[u] = expf(s[u] - m);
                l += s[u];
            }
            for (int u = 0; u < kChunk; ++u) {
                if (u0 + u >= nvalid) break;
                const float p = s[u];
                const float *vr = Vs + (u0 + u) * D;
#pragma unroll
                for (int d = 0; d < D; ++d) acc[d] = fmaf(p, vr[d], acc[d]);
            }
        }
    }

    if (qrow < Lq) {
        T *o = out + (bh * Lq + qrow) * D;
        const float inv = any ? 1.0f / l : 0.0f;
#pragma unroll
        for (int d = 0; d < D; ++d) o[d] = from_f32<T>(acc[d] * inv);
        if (lse) lse[bh * Lq + qrow] = any ? m + logf(l) : -INFINITY;
    }
}

template <typename T, int D>
cudaError_t launch(const void *q, const void *k, const void *v, int64_t BH, int64_t Lq,
                   int64_t Lk, float tau, const int32_t *kv_idx, const int32_t *kv_cnt,
                   int64_t max_sel, void *out, float *lse, int32_t *status, cudaStream_t s) {
    const int64_t nQB = ceil_div(Lq, kBlock), nKB = ceil_div(Lk, kBlock);
    const size_t smem = sizeof(float) * 3 * kBlock * D;
    cudaError_t e = cudaFuncSetAttribute(attn_simt_kernel<T, D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attn_simt_kernel<T, D><<<(unsigned)(BH * nQB), kBlock, smem, s>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), Lq, Lk,
        nQB, nKB, tau, kv_idx, kv_cnt, max_sel, static_cast<T *>(out), lse, status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_simt(const void *q, const void *k, const void *v, int dtype,
                             int64_t BH, int64_t Lq, int64_t Lk, int D, float tau,
                             const int32_t *kv_idx, const int32_t *kv_cnt, int64_t max_sel,
                             void *out, float *lse, int32_t *status, cudaStream_t stream) {
    if (dtype == 0)
        return D == 128 ? launch<__nv_bfloat16, 128>(q, k, v, BH, Lq, Lk, tau, kv_idx, kv_cnt,
                                                     max_sel, out, lse, status, stream)
                        : launch<__nv_bfloat16, 64>(q, k, v, BH, Lq, Lk, tau, kv_idx, kv_cnt,
                                                    max_sel, out, lse, status, stream);
    return D == 128 ? launch<float, 128>(q, k, v, BH, Lq, Lk, tau, kv_idx, kv_cnt, max_sel, out,
                                         lse, status, stream)
                    : launch<float, 64>(q, k, v, BH, Lq, Lk, tau, kv_idx, kv_cnt, max_sel, out,
                                        lse, status, stream);
}

}  // namespace sparstar
