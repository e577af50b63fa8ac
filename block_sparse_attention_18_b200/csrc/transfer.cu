// Diagnostic — block lists reused across scales: the lists selected at a
// source scale, carried by token position to a target scale (SparSTAR,
// pith.science review, "Extended reading notes / Core claim": reusing a
// block-selection pattern across scales loses retained attention mass, which
// is why the method recomputes the selection at every scale; Figure 1 of the
// review: a reused support misses blocks that become active).
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
// One warp per target row, eight rows in flight per CTA:
//   1. the source row's list becomes a bitmap in shared memory (one bit per
//      source key block, entries outside [0, nKB_s) dropped);
//   2. the 32 lanes test 32 consecutive target blocks at a time: each lane
//      maps its block's centre token to the source and looks up the bit;
//   3. a ballot and a prefix popcount write the kept blocks in ascending
//      order; the rest of the row is filled with -1.
// Memory: the source lists are read once and the target lists written once
// (B*H*nQB_t*max_sel_t int32); the bitmap lookups stay in shared memory.
#include "sparstar_internal.h"

namespace sparstar {
namespace {

constexpr int kWarpsPerCta = 8;

__global__ void __launch_bounds__(kWarpsPerCta * 32)
    transfer_kernel(const int32_t *__restrict__ src_idx, const int32_t *__restrict__ src_cnt,
                    int64_t src_max_sel, TransferLayout ly, int64_t rows,
                    int32_t *__restrict__ dst_idx, int32_t *__restrict__ dst_cnt,
                    int64_t dst_max_sel, int words) {
    extern __shared__ uint32_t bitmaps[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    uint32_t *bm = bitmaps + warp * words;
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
                keep = j < ly.nF_t;
                if (!keep) {
                    const int64_t a = (int64_t)j * kBlock;
                    const int64_t n_real = ly.Lk_t - a < kBlock ? ly.Lk_t - a : kBlock;
                    const int64_t t = a + (n_real - 1) / 2;  // the block's centre token
                    int g = 0;
                    while (g < 3 && t >= ly.off_t[g] + ly.len_t[g]) ++g;
                    if (ly.len_s[g] > 0) {
                        const int64_t img =
                            ly.off_s[g] + (t - ly.off_t[g]) * ly.len_s[g] / ly.len_t[g];
                        const int64_t sb = img / kBlock;
                        keep = (bm[sb >> 5] >> (sb & 31)) & 1u;
                    }
                }
            }
            const uint32_t ballot = __ballot_sync(0xffffffffu, keep);
            if (keep) out[n + __popc(ballot & ((1u << lane) - 1u))] = j;
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

int64_t transfer_max_nkb() { return 32768; }  // 4 KB of bitmap per warp

cudaError_t launch_transfer_lists(const int32_t *src_idx, const int32_t *src_cnt,
                                  int64_t src_max_sel, int64_t BH, const TransferLayout &ly,
                                  int32_t *dst_idx, int32_t *dst_cnt, int64_t dst_max_sel,
                                  cudaStream_t stream) {
    const int64_t rows = BH * ly.nQB_t;
    if (rows == 0) return cudaSuccess;
    const int words = (int)((ly.nKB_s + 31) / 32);
    const size_t smem = (size_t)kWarpsPerCta * words * sizeof(uint32_t);
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(
            transfer_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    // Rows are independent and short: enough CTAs for every SM several
    // times over, each warp striding over the rows.
    int64_t ctas = ceil_div(rows, kWarpsPerCta);
    if (ctas > 148 * 16) ctas = 148 * 16;
    transfer_kernel<<<(unsigned)ctas, kWarpsPerCta * 32, smem, stream>>>(
        src_idx, src_cnt, src_max_sel, ly, rows, dst_idx, dst_cnt, dst_max_sel, words);
    return cudaGetLastError();
}

}  // namespace sparstar
