// Step 1 — 128-token block mean pooling of Q or K (SparSTAR, pith.science
// review, "What carries the argument": the score uses the mean query and the
// mean key of each run of 128 consecutive tokens).
//
// One CTA per (b, h, block).  The block's rows are 128 x D elements; each
// row is split into 16-byte chunks.  Thread (stripe r, chunk c) sums, in
// ascending token order, the tokens t = r, r+8, ..., r+120 of chunk c: this
// is exactly stripe r of the fixed order.  The 8 stripe sums of every
// coordinate then meet in shared memory and are combined as
// ((s0+s1)+(s2+s3))+((s4+s5)+(s6+s7)) and divided once by the real token
// count with IEEE round-to-nearest.  Every add and the division are
// explicit _rn intrinsics, so no contraction or reassociation can change
// the bits.
//
// pool2_kernel does the same for two tensors (Q and K) in one launch.
//
// Memory: a warp covers 2 stripes x 16 chunks (bf16, D = 128), i.e. two
// full 256-byte rows per load instruction; every thread keeps its 16 loads
// in flight before the first add.  HBM-bound: bytes = L*D*esize read +
// nblk*D*4 written.
#include <cuda_bf16.h>

#include "sparstar_internal.h"

namespace sparstar {
namespace {

constexpr int kStripes = 8;
constexpr int kRowsPerStripe = kBlock / kStripes;  // 16

template <typename T>
struct Vec;  // one 16-byte chunk
template <>
struct Vec<float> {
    static constexpr int kElems = 4;
    __device__ static void widen(const uint4 &u, float *f) {
        f[0] = __uint_as_float(u.x);
        f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z);
        f[3] = __uint_as_float(u.w);
    }
};
template <>
struct Vec<__nv_bfloat16> {
    static constexpr int kElems = 8;
    // bf16 -> fp32 is exact: the bf16 bits are the top half of the fp32 bits.
    __device__ static void widen(const uint4 &u, float *f) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};

// Mean of block `blk` of head `bh` of x [.., L, D] into xbar[row].
template <typename T, int D>
__device__ __forceinline__ void pool_block(const T *__restrict__ x, int64_t L, int64_t bh,
                                           int64_t blk, int64_t row, float *__restrict__ xbar,
                                           float (*stripe_sum)[D]) {
    constexpr int kElems = Vec<T>::kElems;
    constexpr int kChunks = D / kElems;  // 16-byte chunks per row
    const int64_t t0 = blk * kBlock;
    const int n = (int)((L - t0) < kBlock ? (L - t0) : kBlock);

    const int c = threadIdx.x % kChunks;  // chunk within a row
    const int r = threadIdx.x / kChunks;  // stripe
    const uint4 *base =
        reinterpret_cast<const uint4 *>(x + (bh * L + t0) * D) + c;  // row 0, chunk c

    uint4 raw[kRowsPerStripe];
#pragma unroll
    for (int u = 0; u < kRowsPerStripe; ++u) {
        const int t = r + kStripes * u;
        if (t < n)
            raw[u] = __ldcs(base + (int64_t)t * kChunks);
        else
            raw[u] = make_uint4(0, 0, 0, 0);
    }
    float acc[kElems];
#pragma unroll
    for (int e = 0; e < kElems; ++e) acc[e] = 0.0f;
#pragma unroll
    for (int u = 0; u < kRowsPerStripe; ++u) {
        const int t = r + kStripes * u;
        if (t < n) {  // absent tokens are not added (a +0 add could flip -0)
            float f[kElems];
            Vec<T>::widen(raw[u], f);
#pragma unroll
            for (int e = 0; e < kElems; ++e) acc[e] = __fadd_rn(acc[e], f[e]);
        }
    }
#pragma unroll
    for (int e = 0; e < kElems; ++e) stripe_sum[r][c * kElems + e] = acc[e];
    __syncthreads();

    const float fn = (float)n;
    for (int d = threadIdx.x; d < D; d += blockDim.x) {
        const float left = __fadd_rn(__fadd_rn(stripe_sum[0][d], stripe_sum[1][d]),
                                     __fadd_rn(stripe_sum[2][d], stripe_sum[3][d]));
        const float right = __fadd_rn(__fadd_rn(stripe_sum[4][d], stripe_sum[5][d]),
                                      __fadd_rn(stripe_sum[6][d], stripe_sum[7][d]));
        xbar[row * D + d] = __fdiv_rn(__fadd_rn(left, right), fn);
    }
}

template <typename T, int D>
__global__ void __launch_bounds__(kStripes * (D * sizeof(T) / 16))
pool_kernel(const T *__restrict__ x, int64_t L, int64_t nblk, float *__restrict__ xbar) {
    __shared__ float stripe_sum[kStripes][D];
    const int64_t row = blockIdx.x;  // (bh, blk) flattened
    const int64_t bh = row / nblk;
    pool_block<T, D>(x, L, bh, row - bh * nblk, row, xbar, stripe_sum);
}

// Q and K in one launch: CTAs [0, rows0) pool tensor 0, the rest tensor 1.
template <typename T, int D>
__global__ void __launch_bounds__(kStripes * (D * sizeof(T) / 16))
pool2_kernel(const T *__restrict__ x0, int64_t L0, int64_t nblk0, float *__restrict__ out0,
             const T *__restrict__ x1, int64_t L1, int64_t nblk1, float *__restrict__ out1,
             int64_t rows0) {
    __shared__ float stripe_sum[kStripes][D];
    const bool second = blockIdx.x >= rows0;
    const int64_t nblk = second ? nblk1 : nblk0;
    const int64_t row = second ? blockIdx.x - rows0 : blockIdx.x;
    const int64_t bh = row / nblk;
    pool_block<T, D>(second ? x1 : x0, second ? L1 : L0, bh, row - bh * nblk, row,
                     second ? out1 : out0, stripe_sum);
}

template <typename T, int D>
cudaError_t launch2(const void *x0, int64_t L0, float *out0, const void *x1, int64_t L1,
                    float *out1, int64_t BH, cudaStream_t s) {
    const int64_t n0 = ceil_div(L0, kBlock), n1 = ceil_div(L1, kBlock);
    const int threads = kStripes * (D * (int)sizeof(T) / 16);
    pool2_kernel<T, D><<<(unsigned)(BH * (n0 + n1)), threads, 0, s>>>(
        static_cast<const T *>(x0), L0, n0, out0, static_cast<const T *>(x1), L1, n1, out1,
        BH * n0);
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch(const void *x, int64_t BH, int64_t L, float *xbar, cudaStream_t s) {
    const int64_t nblk = ceil_div(L, kBlock);
    const int threads = kStripes * (D * (int)sizeof(T) / 16);
    pool_kernel<T, D><<<(unsigned)(BH * nblk), threads, 0, s>>>(static_cast<const T *>(x), L,
                                                                nblk, xbar);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pool2(const void *x0, int64_t L0, float *out0, const void *x1, int64_t L1,
                         float *out1, int dtype, int64_t BH, int D, cudaStream_t stream) {
    if (dtype == 0)
        return D == 128 ? launch2<__nv_bfloat16, 128>(x0, L0, out0, x1, L1, out1, BH, stream)
                        : launch2<__nv_bfloat16, 64>(x0, L0, out0, x1, L1, out1, BH, stream);
    return D == 128 ? launch2<float, 128>(x0, L0, out0, x1, L1, out1, BH, stream)
                    : launch2<float, 64>(x0, L0, out0, x1, L1, out1, BH, stream);
}

cudaError_t launch_pool(const void *x, int dtype, int64_t BH, int64_t L, int D, float *xbar,
                        cudaStream_t stream) {
    if (dtype == 0)
        return D == 128 ? launch<__nv_bfloat16, 128>(x, BH, L, xbar, stream)
                        : launch<__nv_bfloat16, 64>(x, BH, L, xbar, stream);
    return D == 128 ? launch<float, 128>(x, BH, L, xbar, stream)
                    : launch<float, 64>(x, BH, L, xbar, stream);
}

}  // namespace sparstar
