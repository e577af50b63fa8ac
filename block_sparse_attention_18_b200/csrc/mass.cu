// Diagnostic — retained attention mass of a block list, and the token-wise
// Top-K bound at the same budget (SparSTAR, pith.science review, "Extended
// reading notes / Core claim": block-wise Top-K recomputed at every scale
// stays close to the token-wise upper bound in retained attention mass;
// "What would settle it": the exact token-wise Top-K at the same densities
// is the comparison).
//
// For one query row with dense weights p_t = softmax_t(tau q.k_t) over every
// key t < Lk:
//   lse_dense   = log sum_t exp(tau q.k_t);
//   mass_block  = sum of p_t over the tokens of the row's listed blocks;
//   mass_forced = sum of p_t over the tokens of blocks 0 .. nF-1;
//   M           = real tokens in the listed blocks j >= nF;
//   mass_tok    = mass_forced + the sum of the M largest candidate p_t
//                 (tokens t >= 128 nF).
//
// One CTA per sampled row, 256 threads, three passes over the row:
//   1. every key's score tau * (q . k_t), fp32 FMAs over d, into the
//      caller's scratch row, and the row max;
//   2. fp64 sums of exp(s - max): the normaliser, the listed-block and the
//      forced sums, and the candidate budget M (listed blocks in a shared
//      bitmap);
//   3. the exact M-th largest candidate score T by a 32-step bitwise search
//      on order-preserving keys (each step a CTA-wide count), then the fp64
//      sum of the candidates above T plus (M - count above T) copies of T's
//      weight.
// Memory: each row reads all of K for its head once (Lk * D * esize) and its
// scratch row (Lk * 4 bytes) 34 times; this is a sampled-row diagnostic, not
// part of the timed step.
#include <cuda_bf16.h>

#include "sparstar_internal.h"

namespace sparstar {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7fffffffu) == 0u) u = 0u;  // -0 -> +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// CTA-wide reductions through shared scratch (every thread gets the result).
__device__ double cta_sum(double v, double *red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();  // red is free
    if (lane == 0) red[warp] = v;
    __syncthreads();
    double t = 0.0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) t += red[w];
    return t;
}
__device__ uint32_t cta_sum_u(uint32_t v, uint32_t *red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = __reduce_add_sync(0xffffffffu, v);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    uint32_t t = 0u;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) t += red[w];
    return t;
}
__device__ float cta_max(float v, float *red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float t = red[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) t = fmaxf(t, red[w]);
    return t;
}

// One key row dotted with the query row in shared memory (fp32, d ascending).
__device__ __forceinline__ float dot_row(const float *qv, const __nv_bfloat16 *kr, int D) {
    float acc = 0.0f;
    const uint4 *p = reinterpret_cast<const uint4 *>(kr);
    for (int c = 0; c < D / 8; ++c) {
        const uint4 u = p[c];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            acc = fmaf(qv[8 * c + 2 * i], __uint_as_float(w[i] << 16), acc);
            acc = fmaf(qv[8 * c + 2 * i + 1], __uint_as_float(w[i] & 0xffff0000u), acc);
        }
    }
    return acc;
}
__device__ __forceinline__ float dot_row(const float *qv, const float *kr, int D) {
    float acc = 0.0f;
    const float4 *p = reinterpret_cast<const float4 *>(kr);
    for (int c = 0; c < D / 4; ++c) {
        const float4 u = p[c];
        acc = fmaf(qv[4 * c + 0], u.x, acc);
        acc = fmaf(qv[4 * c + 1], u.y, acc);
        acc = fmaf(qv[4 * c + 2], u.z, acc);
        acc = fmaf(qv[4 * c + 3], u.w, acc);
    }
    return acc;
}
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f32(float x) { return x; }

template <typename T>
__global__ void __launch_bounds__(kThreads)
mass_kernel(const T *__restrict__ q, const T *__restrict__ k, int64_t n_flat, int64_t Lq,
            int64_t Lk, int D, int nKB, float tau, int nF, const int32_t *__restrict__ kv_idx,
            const int32_t *__restrict__ kv_cnt, int64_t max_sel, const int64_t *__restrict__ rows,
            float *__restrict__ scratch, double *__restrict__ lse_out,
            double *__restrict__ mb_out, double *__restrict__ mt_out,
            double *__restrict__ mf_out) {
    extern __shared__ __align__(16) float smem[];
    float *qv = smem;                                         // [D]
    uint32_t *listed = reinterpret_cast<uint32_t *>(qv + D);  // [ceil(nKB / 32)]
    __shared__ double red_d[kWarps];
    __shared__ float red_f[kWarps];
    __shared__ uint32_t red_u[kWarps];

    const int tid = threadIdx.x;
    const int64_t n = blockIdx.x;
    const int64_t flat = rows[n];
    if (flat < 0 || flat >= n_flat) {  // not a row: NaN results, nothing read
        if (tid == 0) mb_out[n] = mt_out[n] = mf_out[n] = lse_out[n] = __longlong_as_double(0x7ff8000000000000ll);
        return;
    }
    const int64_t bh = flat / Lq, r = flat - bh * Lq;
    const int64_t nQB = (Lq + kBlock - 1) / kBlock;
    const int64_t list = bh * nQB + r / kBlock;
    const int words = (nKB + 31) / 32;
    for (int d = tid; d < D; d += kThreads) qv[d] = to_f32(q[flat * D + d]);
    for (int w = tid; w < words; w += kThreads) listed[w] = 0u;
    __syncthreads();
    int64_t cnt = kv_cnt[list];
    if (cnt > max_sel) cnt = max_sel;
    for (int64_t c = tid; c < cnt; c += kThreads) {
        const int j = kv_idx[list * max_sel + c];
        if (j >= 0 && j < nKB) atomicOr(&listed[j >> 5], 1u << (j & 31));
    }
    __syncthreads();

    // 1. scores and the row max
    float *s = scratch + n * Lk;
    const T *kb = k + bh * Lk * D;
    float mx = -INFINITY;
    for (int64_t t = tid; t < Lk; t += kThreads) {
        const float sv = dot_row(qv, kb + t * D, D) * tau;
        s[t] = sv;
        mx = fmaxf(mx, sv);
    }
    const float m = cta_max(mx, red_f);

    // 2. the normaliser, the listed and forced sums, the candidate budget
    const int64_t f_end = (int64_t)nF * kBlock < Lk ? (int64_t)nF * kBlock : Lk;
    double z = 0.0, mb = 0.0, mf = 0.0;
    uint32_t budget = 0u;
    for (int64_t t = tid; t < Lk; t += kThreads) {
        const double e = exp((double)s[t] - (double)m);
        z += e;
        const int64_t j = t / kBlock;
        if ((listed[j >> 5] >> (j & 31)) & 1u) {
            mb += e;
            if (t >= f_end) ++budget;
        }
        if (t < f_end) mf += e;
    }
    z = cta_sum(z, red_d);
    mb = cta_sum(mb, red_d);
    mf = cta_sum(mf, red_d);
    const uint32_t M = cta_sum_u(budget, red_u);

    // 3. the M largest candidate weights
    const uint32_t nc = (uint32_t)(Lk - f_end);
    double top = 0.0;
    if (M > 0u) {
        uint32_t T = 0u, need = 0u;  // M >= nc: every candidate (all keys > 0)
        if (M < nc) {
            uint32_t prefix = 0u;
            for (int bit = 31; bit >= 0; --bit) {
                const uint32_t cand = prefix | (1u << bit);
                uint32_t c = 0u;
                for (int64_t t = f_end + tid; t < Lk; t += kThreads)
                    c += order_key(s[t]) >= cand ? 1u : 0u;
                if (cta_sum_u(c, red_u) >= M) prefix = cand;
            }
            T = prefix;
            uint32_t c = 0u;
            for (int64_t t = f_end + tid; t < Lk; t += kThreads) c += order_key(s[t]) > T ? 1u : 0u;
            need = M - cta_sum_u(c, red_u);
        }
        double part = 0.0;
        for (int64_t t = f_end + tid; t < Lk; t += kThreads)
            if (order_key(s[t]) > T) part += exp((double)s[t] - (double)m);
        top = cta_sum(part, red_d);
        if (need > 0u) top += (double)need * exp((double)key_value(T) - (double)m);
    }
    if (tid == 0) {
        lse_out[n] = (double)m + log(z);
        mb_out[n] = mb / z;
        mf_out[n] = mf / z;
        mt_out[n] = (mf + top) / z;
    }
}

}  // namespace

int64_t mass_max_nkb() { return (int64_t)1 << 20; }

cudaError_t launch_retained_mass(const void *q, const void *k, int dtype, int64_t BH, int64_t Lq,
                                 int64_t Lk, int D, float tau, int64_t nF, const int32_t *kv_idx,
                                 const int32_t *kv_cnt, int64_t max_sel, const int64_t *rows,
                                 int64_t n_rows, float *scratch, double *lse_dense,
                                 double *mass_block, double *mass_tok, double *mass_forced,
                                 cudaStream_t stream) {
    const int64_t nKB = ceil_div(Lk, kBlock);
    const size_t smem = sizeof(float) * (size_t)D + sizeof(uint32_t) * (size_t)ceil_div(nKB, 32);
    if (dtype == 0) {
        cudaError_t e = cudaFuncSetAttribute(mass_kernel<__nv_bfloat16>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        mass_kernel<__nv_bfloat16><<<(unsigned)n_rows, kThreads, smem, stream>>>(
            static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k),
            BH * Lq, Lq, Lk, D, (int)nKB, tau, (int)nF, kv_idx, kv_cnt, max_sel, rows, scratch,
            lse_dense, mass_block, mass_tok, mass_forced);
    } else {
        cudaError_t e = cudaFuncSetAttribute(mass_kernel<float>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        mass_kernel<float><<<(unsigned)n_rows, kThreads, smem, stream>>>(
            static_cast<const float *>(q), static_cast<const float *>(k), BH * Lq, Lq, Lk, D,
            (int)nKB, tau, (int)nF, kv_idx, kv_cnt, max_sel, rows, scratch, lse_dense, mass_block,
            mass_tok, mass_forced);
    }
    return cudaGetLastError();
}

}  // namespace sparstar
