// Step 2b — clip-aware block Top-K written straight into a forward-only
// block list (SparSTAR, pith.science review, "What carries the argument":
// text / Clip-1 reference blocks retained, reference and current blocks
// ranked jointly under the density, only the forward part of the mask kept;
// "Referee Report", minor comment 5: block-wise Top-K).
//
// One warp per (b, h, query block) row.  Candidates are the blocks
// j in [nF, nKB); their fp32 scores map to order-preserving 32-bit keys
// (-0 canonicalised to +0 first, so IEEE-equal scores get equal keys).
// The k-th largest key T is found by a 32-step bitwise search: the largest
// T with count(key >= T) >= k, each count a warp-wide sum.  Candidates are
// then swept in ascending j, 32 at a time: a candidate is kept if its key
// is > T, or == T and it is among the first (k - count(key > T)) ties in j
// order (ties to the lower index).  Ballots give each kept block its slot,
// so the list comes out ascending without a sort: forced prefix 0..nF-1,
// then the kept candidates, then -1 in unused slots.
//
// Keys live in registers (kPerLane slots per lane, candidate c in lane
// c % 32, slot c / 32) for C <= 2048; larger rows use shared memory.
#include "sparstar_internal.h"

namespace sparstar {
namespace {

constexpr int kWarpsPerCta = 4;

__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7fffffffu) == 0u) u = 0u;  // -0 -> +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Key access abstraction: registers (fixed slots) or shared memory.
template <int kPerLane>
struct RegKeys {
    uint32_t key[kPerLane];
    __device__ void load(const float *srow, int C, int lane, uint32_t *) {
#pragma unroll
        for (int s = 0; s < kPerLane; ++s) {
            const int c = s * 32 + lane;
            key[s] = c < C ? order_key(srow[c]) : 0u;  // 0 < every real key
        }
    }
    __device__ int count_ge(uint32_t t, int C, int lane) const {
        int n = 0;
#pragma unroll
        for (int s = 0; s < kPerLane; ++s) n += (s * 32 + lane < C && key[s] >= t) ? 1 : 0;
        return n;
    }
    __device__ int count_gt(uint32_t t, int C, int lane) const {
        int n = 0;
#pragma unroll
        for (int s = 0; s < kPerLane; ++s) n += (s * 32 + lane < C && key[s] > t) ? 1 : 0;
        return n;
    }
    // Ascending sweep: keep key > T, and the first `need` keys == T in j order.
    __device__ int sweep(uint32_t T, uint32_t need, int C, int nF, int lane, int32_t *out,
                         int written) const {
        const unsigned lt_mask = (1u << lane) - 1u;
        uint32_t ties_seen = 0u;
#pragma unroll
        for (int s = 0; s < kPerLane; ++s) {
            if (s * 32 >= C) break;  // warp-uniform
            const int c = s * 32 + lane;
            const bool valid = c < C;
            const bool gt = valid && key[s] > T;
            const bool eq = valid && key[s] == T;
            const unsigned eq_ballot = __ballot_sync(0xffffffffu, eq);
            const uint32_t eq_rank = ties_seen + __popc(eq_ballot & lt_mask);
            const bool take = gt || (eq && eq_rank < need);
            const unsigned take_ballot = __ballot_sync(0xffffffffu, take);
            if (take) out[written + __popc(take_ballot & lt_mask)] = nF + c;
            written += __popc(take_ballot);
            ties_seen += __popc(eq_ballot);
        }
        return written;
    }
};

struct SmemKeys {
    uint32_t *key;
    __device__ void load(const float *srow, int C, int lane, uint32_t *buf) {
        key = buf;
        for (int c = lane; c < C; c += 32) key[c] = order_key(srow[c]);
        __syncwarp();
    }
    __device__ int count_ge(uint32_t t, int C, int lane) const {
        int n = 0;
        for (int c = lane; c < C; c += 32) n += key[c] >= t ? 1 : 0;
        return n;
    }
    __device__ int count_gt(uint32_t t, int C, int lane) const {
        int n = 0;
        for (int c = lane; c < C; c += 32) n += key[c] > t ? 1 : 0;
        return n;
    }
    __device__ int sweep(uint32_t T, uint32_t need, int C, int nF, int lane, int32_t *out,
                         int written) const {
        const unsigned lt_mask = (1u << lane) - 1u;
        uint32_t ties_seen = 0u;
        for (int base = 0; base < C; base += 32) {
            const int c = base + lane;
            const bool valid = c < C;
            const uint32_t kc = valid ? key[c] : 0u;
            const bool gt = valid && kc > T;
            const bool eq = valid && kc == T;
            const unsigned eq_ballot = __ballot_sync(0xffffffffu, eq);
            const uint32_t eq_rank = ties_seen + __popc(eq_ballot & lt_mask);
            const bool take = gt || (eq && eq_rank < need);
            const unsigned take_ballot = __ballot_sync(0xffffffffu, take);
            if (take) out[written + __popc(take_ballot & lt_mask)] = nF + c;
            written += __popc(take_ballot);
            ties_seen += __popc(eq_ballot);
        }
        return written;
    }
};

template <class Keys>
__device__ void select_row(const float *__restrict__ S, int64_t row, int64_t nKB, int nF, int k,
                           int32_t *__restrict__ kv_idx, int32_t *__restrict__ kv_cnt,
                           int64_t max_sel, uint32_t *smem_keys) {
    const int lane = threadIdx.x & 31;
    const int C = (int)nKB - nF;
    const float *srow = S + row * nKB + nF;
    int32_t *out = kv_idx + row * max_sel;

    for (int f = lane; f < nF; f += 32) out[f] = f;

    Keys keys;
    int written = nF;
    if (k > 0) {
        keys.load(srow, C, lane, smem_keys);
        uint32_t T = 0u, need = 0u;
        if (k >= C) {
            T = 0u;  // every candidate has key > 0
            need = 0u;
        } else {
            uint32_t prefix = 0u;
            for (int bit = 31; bit >= 0; --bit) {
                const uint32_t cand = prefix | (1u << bit);
                if (warp_sum(keys.count_ge(cand, C, lane)) >= k) prefix = cand;
            }
            T = prefix;
            need = (uint32_t)(k - warp_sum(keys.count_gt(T, C, lane)));
        }
        written = keys.sweep(T, need, C, nF, lane, out, written);
    }
    for (int64_t s = written + lane; s < max_sel; s += 32) out[s] = -1;
    if (lane == 0) kv_cnt[row] = nF + k;
}

template <int kPerLane>
__global__ void __launch_bounds__(32 * kWarpsPerCta)
select_kernel_regs(const float *__restrict__ S, int64_t rows, int64_t nKB, int nF, int k,
                   int32_t *__restrict__ kv_idx, int32_t *__restrict__ kv_cnt, int64_t max_sel) {
    const int64_t row = (int64_t)blockIdx.x * kWarpsPerCta + threadIdx.x / 32;
    if (row >= rows) return;
    select_row<RegKeys<kPerLane>>(S, row, nKB, nF, k, kv_idx, kv_cnt, max_sel, nullptr);
}

__global__ void __launch_bounds__(32)
select_kernel_smem(const float *__restrict__ S, int64_t rows, int64_t nKB, int nF, int k,
                   int32_t *__restrict__ kv_idx, int32_t *__restrict__ kv_cnt, int64_t max_sel) {
    extern __shared__ uint32_t keys_smem[];
    const int64_t row = blockIdx.x;
    if (row >= rows) return;
    select_row<SmemKeys>(S, row, nKB, nF, k, kv_idx, kv_cnt, max_sel, keys_smem);
}

template <int kPerLane>
cudaError_t launch_regs(const float *S, int64_t rows, int64_t nKB, int nF, int k, int32_t *idx,
                        int32_t *cnt, int64_t max_sel, cudaStream_t s) {
    const unsigned grid = (unsigned)ceil_div(rows, kWarpsPerCta);
    select_kernel_regs<kPerLane><<<grid, 32 * kWarpsPerCta, 0, s>>>(S, rows, nKB, nF, k, idx,
                                                                    cnt, max_sel);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select(const float *S, int64_t rows, int64_t nKB, int64_t nF, int64_t k,
                          int32_t *kv_idx, int32_t *kv_cnt, int64_t max_sel,
                          cudaStream_t stream) {
    const int64_t C = nKB - nF;
    const int inF = (int)nF, ik = (int)k;
    if (C <= 32) return launch_regs<1>(S, rows, nKB, inF, ik, kv_idx, kv_cnt, max_sel, stream);
    if (C <= 64) return launch_regs<2>(S, rows, nKB, inF, ik, kv_idx, kv_cnt, max_sel, stream);
    if (C <= 128) return launch_regs<4>(S, rows, nKB, inF, ik, kv_idx, kv_cnt, max_sel, stream);
    if (C <= 256) return launch_regs<8>(S, rows, nKB, inF, ik, kv_idx, kv_cnt, max_sel, stream);
    if (C <= 512) return launch_regs<16>(S, rows, nKB, inF, ik, kv_idx, kv_cnt, max_sel, stream);
    if (C <= 1024) return launch_regs<32>(S, rows, nKB, inF, ik, kv_idx, kv_cnt, max_sel, stream);
    if (C <= 1280) return launch_regs<40>(S, rows, nKB, inF, ik, kv_idx, kv_cnt, max_sel, stream);
    if (C <= 2048) return launch_regs<64>(S, rows, nKB, inF, ik, kv_idx, kv_cnt, max_sel, stream);
    const size_t smem = sizeof(uint32_t) * (size_t)C;
    cudaError_t e = cudaFuncSetAttribute(select_kernel_smem,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    select_kernel_smem<<<(unsigned)rows, 32, smem, stream>>>(S, rows, nKB, inF, ik, kv_idx,
                                                             kv_cnt, max_sel);
    return cudaGetLastError();
}

}  // namespace sparstar
