// Diagnostic — block lists reused across scales: the lists selected at a
// source scale, carried by token position to a target scale (SparSTAR,
// pith.science review, "Extended reading notes / Core claim": a selection
// carried from one scale to another keeps less of the attention mass than a
// fresh one, which is why the method selects anew at every scale; Figure 1 of the
// review: blocks that matter at the new scale can lie outside a mask carried
// over from the earlier one).
//
// The pages give no map between two scales' token positions.  Reading: the
// block mask is resampled by nearest neighbour along each key segment g of
// [text | image_ref | ref | cur]: target offset p has as image the source
// offset floor(p * len_s[g] / len_t[g]) (none when len_s[g] = 0).  Target
// query block i takes the list of the source query block that holds the
// image of i's centre query token; target key block j is kept when j < nF_t
// or when the image of j's centre token lies in a listed source block (the
// centre of a block of n real tokens starting at a is a + (n - 1) / 2).
//
// The map from a target key block to the source block holding the image of
// its centre token is the same for every row, so each CTA builds it once in
// shared memory (-2: forced at the target, -1: no image) and then runs one
// warp per target row, eight rows in flight, striding over the rows:
//   1. the source row's list becomes a bitmap in shared memory (one bit per
//      source key block, entries outside [0, nKB_s) dropped);
//   2. the 32 lanes test 32 consecutive target blocks at a time: a map
//      lookup and a bitmap lookup each;
//   3. a ballot and a prefix popcount write the kept blocks in ascending
//      order; the rest of the row is filled with -1.
// Memory: the source lists are read once and the target lists written once
// (B*H*nQB_t*max_sel_t int32); the lookups stay in shared memory.
#include <algorithm>
#include <functional>
#include <vector>

#include "sparstar_internal.h"

namespace sparstar {
namespace {

constexpr int kWarpsPerCta = 8;

// Source block of the image of target block j's centre token; -1 if that
// token's segment is empty at the source.
__host__ __device__ inline int32_t centre_image_block(const TransferLayout &ly, int64_t j) {
    const int64_t a = j * kBlock;
    const int64_t n_real = ly.Lk_t - a < kBlock ? ly.Lk_t - a : kBlock;
    const int64_t t = a + (n_real - 1) / 2;  // the block's centre token
    int g = 0;
    while (g < 3 && t >= ly.off_t[g] + ly.len_t[g]) ++g;
    if (ly.len_s[g] == 0) return -1;
    return (int32_t)((ly.off_s[g] + (t - ly.off_t[g]) * ly.len_s[g] / ly.len_t[g]) / kBlock);
}

__global__ void __launch_bounds__(kWarpsPerCta * 32)
    transfer_kernel(const int32_t *__restrict__ src_idx, const int32_t *__restrict__ src_cnt,
                    int64_t src_max_sel, TransferLayout ly, int64_t rows,
                    int32_t *__restrict__ dst_idx, int32_t *__restrict__ dst_cnt,
                    int64_t dst_max_sel, int words) {
    extern __shared__ uint32_t smem[];
    int32_t *map = reinterpret_cast<int32_t *>(smem);  // [nKB_t]
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    uint32_t *bm = smem + ly.nKB_t + warp * words;
    for (int j = threadIdx.x; j < ly.nKB_t; j += blockDim.x)
        map[j] = j < ly.nF_t ? -2 : centre_image_block(ly, j);
    __syncthreads();
    for (int64_t row = (int64_t)blockIdx.x * kWarpsPerCta + warp; row < rows;
         row += (int64_t)gridDim.x * kWarpsPerCta) {
        const int64_t bh = row / ly.nQB_t;
        const int64_t i = row % ly.nQB_t;
        // the source row: the block of the image of i's centre query token
        const int64_t qa = i * kBlock;
        const int64_t qn = ly.len_t[3] - qa < kBlock ? ly.len_t[3] - qa : kBlock;
        const int64_t q_img = (qa + (qn - 1) / 2) * ly.len_s[3] / ly.len_t[3];
        const int64_t src_row = bh * ly.nQB_s + q_img / kBlock;

        for (int w = lane; w < words; w += 32) bm[w] = 0u;
        __syncwarp();
        int64_t n_src = src_cnt[src_row];
        n_src = n_src < 0 ? 0 : (n_src > src_max_sel ? src_max_sel : n_src);
        const int32_t *list = src_idx + src_row * src_max_sel;
        for (int64_t c = lane; c < n_src; c += 32) {
            const int32_t j = __ldg(list + c);
            if (j >= 0 && j < ly.nKB_s) atomicOr(bm + (j >> 5), 1u << (j & 31));
        }
        __syncwarp();

        int32_t *out = dst_idx + row * dst_max_sel;
        int n = 0;
        for (int base = 0; base < ly.nKB_t; base += 32) {
            const int j = base + lane;
            bool keep = false;
            if (j < ly.nKB_t) {
                const int32_t sb = map[j];
                keep = sb == -2 || (sb >= 0 && ((bm[sb >> 5] >> (sb & 31)) & 1u));
            }
            const uint32_t ballot = __ballot_sync(0xffffffffu, keep);
            const int pos = n + __popc(ballot & ((1u << lane) - 1u));
            // the host sized the stride for the worst case; the guard only
            // keeps a wrong stride from writing into the next row
            if (keep && pos < dst_max_sel) out[pos] = j;
            n += __popc(ballot);
        }
        for (int64_t c = n + lane; c < dst_max_sel; c += 32) out[c] = -1;
        if (lane == 0) dst_cnt[row] = n;
        __syncwarp();  // the bitmap is cleared for the next row only after every lookup
    }
}

}  // namespace

TransferLayout make_transfer_layout(const int64_t *len_s, const int64_t *len_t) {
    TransferLayout ly{};
    int64_t Ls = 0, Lt = 0;
    for (int g = 0; g < 4; ++g) {
        ly.len_s[g] = len_s[g];
        ly.len_t[g] = len_t[g];
        ly.off_s[g] = Ls;
        ly.off_t[g] = Lt;
        Ls += len_s[g];
        Lt += len_t[g];
    }
    ly.Lk_t = Lt;
    ly.nKB_s = (int32_t)ceil_div(Ls, kBlock);
    ly.nKB_t = (int32_t)ceil_div(Lt, kBlock);
    ly.nQB_s = (int32_t)ceil_div(len_s[3], kBlock);
    ly.nQB_t = (int32_t)ceil_div(len_t[3], kBlock);
    ly.nF_t = (int32_t)ceil_div(len_t[0] + len_t[1], kBlock);
    return ly;
}

// Source and target key blocks: 4 KB of bitmap per warp and a 128 KB block
// map, 160 KB of shared memory at most.
int64_t transfer_max_nkb() { return 32768; }

// Exact worst case of a transferred row's length: every non-forced target
// block is kept through exactly one source block (the one holding the image
// of its centre token), so a row that lists m distinct source blocks keeps
// at most nF_t + the m largest per-source-block counts.
int64_t transfer_max_sel(const TransferLayout &ly, int64_t src_max_sel) {
    std::vector<int64_t> hist((size_t)ly.nKB_s, 0);
    for (int64_t j = ly.nF_t; j < ly.nKB_t; ++j) {
        const int32_t sb = centre_image_block(ly, j);
        if (sb >= 0) ++hist[(size_t)sb];
    }
    const size_t m = (size_t)std::min<int64_t>(src_max_sel, ly.nKB_s);
    std::partial_sort(hist.begin(), hist.begin() + m, hist.end(), std::greater<int64_t>());
    int64_t worst = ly.nF_t < ly.nKB_t ? ly.nF_t : ly.nKB_t;
    for (size_t c = 0; c < m; ++c) worst += hist[c];
    return worst;
}

cudaError_t launch_transfer_lists(const int32_t *src_idx, const int32_t *src_cnt,
                                  int64_t src_max_sel, int64_t BH, const TransferLayout &ly,
                                  int32_t *dst_idx, int32_t *dst_cnt, int64_t dst_max_sel,
                                  cudaStream_t stream) {
    const int64_t rows = BH * ly.nQB_t;
    if (rows == 0) return cudaSuccess;
    const int words = (int)((ly.nKB_s + 31) / 32);
    const size_t smem = ((size_t)ly.nKB_t + (size_t)kWarpsPerCta * words) * sizeof(uint32_t);
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(
            transfer_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    // Each CTA builds the block map, then its warps stride over the rows.
    // A row is a chain of dependent loads (count, list, bitmap), so up to
    // eight CTAs per SM keep enough rows in flight; the map (a few integer
    // divisions per thread) is cheap to rebuild per CTA.
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    int64_t ctas = ceil_div(rows, kWarpsPerCta);
    if (ctas > (int64_t)sms * 8) ctas = (int64_t)sms * 8;
    transfer_kernel<<<(unsigned)ctas, kWarpsPerCta * 32, smem, stream>>>(
        src_idx, src_cnt, src_max_sel, ly, rows, dst_idx, dst_cnt, dst_max_sel, words);
    return cudaGetLastError();
}

}  // namespace sparstar
