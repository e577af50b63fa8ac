// Step 2a — the aggregated block score S_ij = tau * qbar_i^T kbar_j
// (SparSTAR, the paper's Eq. 2, as restated in the pith.science review,
// "What carries the argument"; tau = D^-1/2).
//
// Fixed order: acc = +0; acc = fma(qbar[d], kbar[d], acc) for d ascending;
// S = acc * tau (one IEEE multiply).  That order is a register-tiled SIMT
// product: each thread owns an 8 x 8 block of (i, j) outputs and walks d
// once, so the order per output is the sequential one whatever the tiling.
// Tensor cores are not used: their internal accumulation order is not
// specified, and the result must be reproducible bit for bit.
//
// CTA tile 64 (query blocks) x 128 (key blocks), 128 threads; all of D is
// staged once in shared memory, transposed ([d][i] and [d][j]), so the FMA
// loop runs without barriers and two CTAs share an SM (one staging while
// the other computes).  Thread (ti, tj) owns rows {4ti..4ti+3} u
// {32+4ti..32+4ti+3} and columns {4tj..4tj+3} u {64+4tj..64+4tj+3}:
// consecutive threads read consecutive 16-byte words (conflict-free), and
// every 4 shared loads feed 64 fused multiply-adds.
#include "sparstar_internal.h"

namespace sparstar {
namespace {

constexpr int kTI = 64, kTJ = 128, kThreads = 128;

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
score_kernel(const float *__restrict__ qbar, const float *__restrict__ kbar, int64_t nQB,
             int64_t nKB, float tau, float *__restrict__ S) {
    extern __shared__ __align__(16) float smem[];
    float *qs = smem;              // [D][kTI]
    float *ks = smem + D * kTI;    // [D][kTJ]

    const int64_t bh = blockIdx.z;
    const int64_t i0 = (int64_t)blockIdx.y * kTI;
    const int64_t j0 = (int64_t)blockIdx.x * kTJ;
    const float *qb = qbar + bh * nQB * D;
    const float *kb = kbar + bh * nKB * D;
    const int tj = threadIdx.x % 16, ti = threadIdx.x / 16;

    // Stage all of D, transposed.  Consecutive threads take consecutive
    // rows (conflict-free stores); out-of-range rows are zero (never stored).
    // Loops unrolled 16-wide keep 16 loads in flight per thread.
    constexpr int kVec = D / 4;
#pragma unroll 16
    for (int idx = threadIdx.x; idx < kTI * kVec; idx += kThreads) {
        const int row = idx % kTI, v = idx / kTI;
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i0 + row < nQB) a = *reinterpret_cast<const float4 *>(qb + (i0 + row) * D + 4 * v);
        qs[(4 * v + 0) * kTI + row] = a.x;
        qs[(4 * v + 1) * kTI + row] = a.y;
        qs[(4 * v + 2) * kTI + row] = a.z;
        qs[(4 * v + 3) * kTI + row] = a.w;
    }
#pragma unroll 16
    for (int idx = threadIdx.x; idx < kTJ * kVec; idx += kThreads) {
        const int row = idx % kTJ, v = idx / kTJ;
        float4 b = make_float4(0.f, 0.f, 0.f, 0.f);
        if (j0 + row < nKB) b = *reinterpret_cast<const float4 *>(kb + (j0 + row) * D + 4 * v);
        ks[(4 * v + 0) * kTJ + row] = b.x;
        ks[(4 * v + 1) * kTJ + row] = b.y;
        ks[(4 * v + 2) * kTJ + row] = b.z;
        ks[(4 * v + 3) * kTJ + row] = b.w;
    }
    __syncthreads();

    float acc[8][8];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = 0.0f;
#pragma unroll 4
    for (int d = 0; d < D; ++d) {
        const float4 q0 = *reinterpret_cast<const float4 *>(qs + d * kTI + 4 * ti);
        const float4 q1 = *reinterpret_cast<const float4 *>(qs + d * kTI + 32 + 4 * ti);
        const float4 k0 = *reinterpret_cast<const float4 *>(ks + d * kTJ + 4 * tj);
        const float4 k1 = *reinterpret_cast<const float4 *>(ks + d * kTJ + 64 + 4 * tj);
        const float qv[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
        const float kv[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
            for (int b = 0; b < 8; ++b) acc[a][b] = __fmaf_rn(qv[a], kv[b], acc[a][b]);
    }

#pragma unroll
    for (int a = 0; a < 8; ++a) {
        const int64_t i = i0 + (a < 4 ? 4 * ti + a : 32 + 4 * ti + (a - 4));
        if (i >= nQB) continue;
        float *dst = S + (bh * nQB + i) * nKB;
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            const int64_t j = j0 + (b < 4 ? 4 * tj + b : 64 + 4 * tj + (b - 4));
            if (j < nKB) dst[j] = __fmul_rn(acc[a][b], tau);
        }
    }
}

template <int D>
cudaError_t launch(const float *qbar, const float *kbar, int64_t BH, int64_t nQB, int64_t nKB,
                   float tau, float *S, cudaStream_t s) {
    const size_t smem = sizeof(float) * D * (kTI + kTJ);
    cudaError_t e = cudaFuncSetAttribute(score_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)ceil_div(nKB, kTJ), (unsigned)ceil_div(nQB, kTI), (unsigned)BH);
    score_kernel<D><<<grid, kThreads, smem, s>>>(qbar, kbar, nQB, nKB, tau, S);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_score(const float *qbar, const float *kbar, int64_t BH, int64_t nQB,
                         int64_t nKB, int D, float tau, float *S, cudaStream_t stream) {
    return D == 128 ? launch<128>(qbar, kbar, BH, nQB, nKB, tau, S, stream)
                    : launch<64>(qbar, kbar, BH, nQB, nKB, tau, S, stream);
}

}  // namespace sparstar
