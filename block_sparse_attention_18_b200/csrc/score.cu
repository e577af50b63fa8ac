// Step 2a — the aggregated block score S_ij = tau * qbar_i^T kbar_j
// (SparSTAR, the paper's Eq. 2, as restated in the pith.science review,
// "What carries the argument"; tau = D^-1/2).
//
// Fixed order: acc = +0; acc = fma(qbar[d], kbar[d], acc) for d ascending;
// S = acc * tau (one IEEE multiply).  That order is a register-tiled SIMT
// product: each thread owns a 4 x 4 block of (i, j) outputs and walks d
// once, so the order per output is the sequential one whatever the tiling.
// Tensor cores are not used: their internal accumulation order is not
// specified, and the result must be reproducible bit for bit.
//
// CTA tile 64 (query blocks) x 64 (key blocks), 256 threads.  Both operand
// tiles are staged in shared memory transposed ([d][i] and [d][j]) so a
// thread fetches its 4 i-values and 4 j-values with one 16-byte load each.
#include "sparstar_internal.h"

namespace sparstar {
namespace {

constexpr int kTI = 64, kTJ = 64, kThreads = 256;

template <int D>
__global__ void __launch_bounds__(kThreads)
score_kernel(const float *__restrict__ qbar, const float *__restrict__ kbar, int64_t nQB,
             int64_t nKB, float tau, float *__restrict__ S) {
    extern __shared__ __align__(16) float smem[];
    float *qs = smem;             // [D][kTI]
    float *ks = smem + D * kTI;   // [D][kTJ]

    const int64_t bh = blockIdx.z;
    const int64_t i0 = (int64_t)blockIdx.y * kTI;
    const int64_t j0 = (int64_t)blockIdx.x * kTJ;
    const float *qb = qbar + bh * nQB * D;
    const float *kb = kbar + bh * nKB * D;

    // Stage: element (row, d) of the tile -> qs[d * 64 + row].  Consecutive
    // threads take consecutive rows, so the transposed shared-memory stores
    // are conflict-free; out-of-range rows are zero (never stored).
    constexpr int kVecPerRow = D / 4;
    for (int idx = threadIdx.x; idx < kTI * kVecPerRow; idx += kThreads) {
        const int row = idx % kTI, v = idx / kTI;
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
        if (i0 + row < nQB) a = reinterpret_cast<const float4 *>(qb + (i0 + row) * D)[v];
        if (j0 + row < nKB) b = reinterpret_cast<const float4 *>(kb + (j0 + row) * D)[v];
        qs[(4 * v + 0) * kTI + row] = a.x;
        qs[(4 * v + 1) * kTI + row] = a.y;
        qs[(4 * v + 2) * kTI + row] = a.z;
        qs[(4 * v + 3) * kTI + row] = a.w;
        ks[(4 * v + 0) * kTJ + row] = b.x;
        ks[(4 * v + 1) * kTJ + row] = b.y;
        ks[(4 * v + 2) * kTJ + row] = b.z;
        ks[(4 * v + 3) * kTJ + row] = b.w;
    }
    __syncthreads();

    const int tj = threadIdx.x % 16;  // j = 4*tj .. 4*tj+3
    const int ti = threadIdx.x / 16;  // i = 4*ti .. 4*ti+3
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.0f;

#pragma unroll 8
    for (int d = 0; d < D; ++d) {
        const float4 qa = *reinterpret_cast<const float4 *>(qs + d * kTI + 4 * ti);
        const float4 kv = *reinterpret_cast<const float4 *>(ks + d * kTJ + 4 * tj);
        const float qv[4] = {qa.x, qa.y, qa.z, qa.w};
        const float kk[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) acc[a][b] = __fmaf_rn(qv[a], kk[b], acc[a][b]);
    }

#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int64_t i = i0 + 4 * ti + a;
        if (i >= nQB) continue;
        float *dst = S + (bh * nQB + i) * nKB;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int64_t j = j0 + 4 * tj + b;
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
