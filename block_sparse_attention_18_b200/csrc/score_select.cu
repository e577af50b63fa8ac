// Steps 2a + 2b fused — block scores S_ij = tau * qbar_i^T kbar_j (SparSTAR,
// the paper's Eq. 2, restated in the pith.science review, "What carries the
// argument") and the clip-aware block Top-K (same review: text / Clip-1
// reference blocks retained, reference and current blocks ranked jointly
// under the density), without S ever leaving the SM.
//
// One CTA per (b, h, 16 query blocks).  The CTA scores its 16 rows against
// every key block into rows of shared memory, then each of its 8 warps
// selects two of those rows.  Results are bit for bit those of the separate
// score and select kernels:
//   - score: acc = +0; acc = fma(qbar[d], kbar[d], acc) for d ascending;
//     S = acc * tau, each step an explicit round-to-nearest intrinsic.  The
//     score rows hold the order-preserving 32-bit key of S (-0 canonicalised
//     to +0), written as the scores are produced;
//   - select: the k-th largest key T, then an ascending sweep that keeps
//     every key > T and the first k - count(key > T) keys == T (ties to the
//     lower block index).  T is found through a 256-bucket histogram of the
//     scores and an exact search inside the one bucket that holds it (see
//     "selection" below) instead of the separate kernel's 32-step bitwise
//     search over the whole row; both give the same T.
//
// Two score tilings share that selection:
//   - tiled (nKB <= 1664): key tiles of 256 key blocks arrive by TMA, one
//     32-wide d-chunk (256 rows x 128 B, 128-byte swizzle) per slot of a
//     three-slot ring, so the next chunks load while the current one is
//     multiplied.  Each thread owns 4 rows x 4 columns of the 16 x 256 tile:
//     per 4 values of d it issues 8 16-byte shared loads for 64 FMAs.  A
//     tail tile with at most 128 live columns computes only half of them.
//   - wide (nKB up to 2432 for D = 128, 2944 for D = 64): 128-key-block
//     tiles transposed through registers, 2 rows x 4 columns per thread.
//     Slower, but its score rows need less shared memory per key block.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "sparstar.h"
#include "sparstar_internal.h"

namespace sparstar {
namespace {

constexpr int kRows = 16;       // query blocks per CTA
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 256;
constexpr int64_t kMaxSmem = 232448;  // opt-in shared memory per CTA on sm_100
constexpr uint64_t kTimeoutNs = 2000000000ull;

__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7fffffffu) == 0u) u = 0u;  // -0 -> +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ------------------------------------------------------------- selection
//
// Selection of one row: k of the C candidate keys.
//   1. A 256-bin histogram of the candidates over a fixed monotone bucket of
//      the score, b(S) = clamp(floor(32 S), -128, 127) + 128 (buckets 1/32
//      wide on [-4, 4), the two outer buckets open).  The tiled kernel
//      builds it while scoring; the wide kernel builds it from the keys.
//   2. A top-down scan of the histogram gives the bucket b* holding the
//      k-th largest candidate and the count of candidates above it.
//   3. The keys of bucket b* are compacted into a per-warp list and the
//      remaining need' = k - above is resolved exactly there: T = the
//      need'-th largest list key by a bitwise search that starts below the
//      list's common leading bits.
//   4. An ascending sweep keeps every key > T and the first
//      k - count(key > T) keys == T.
// The bucket only decides how much work step 3 does: any data gives the
// same T.  Bucket edges are exact floats ((b-128)/32) whose keys bound each
// bucket, so membership is tested on keys.  A list larger than the warp's
// scratch falls back to a radix select over the whole row.

__device__ __forceinline__ int bucket_of(float s) {
    float f = floorf(s * 32.0f);  // scaling by a power of two is exact
    f = fminf(fmaxf(f, -128.0f), 127.0f);
    return (int)f + 128;
}
// Smallest key of bucket b (b >= 1); bucket 0 starts at key 0.
__device__ __forceinline__ uint32_t bucket_lo_key(int b) {
    return b == 0 ? 0u : order_key((float)(b - 128) * 0.03125f);
}
__device__ __forceinline__ float key_value(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// Top-down scan of a 256-bin histogram: the bin holding the need-th
// largest element and the count of elements in higher bins.
__device__ __forceinline__ void find_bin(const uint32_t *hist, uint32_t need, uint32_t &bin,
                                         uint32_t &above) {
    const int lane = threadIdx.x & 31;
    // Lane l owns bins 255-8l down to 248-8l.
    uint32_t cnt[8], local = 0u;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        cnt[e] = hist[kBins - 1 - 8 * lane - e];
        local += cnt[e];
    }
    uint32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    const uint32_t excl = incl - local;
    const unsigned hit = __ballot_sync(0xffffffffu, excl < need && need <= incl);
    const int src = __ffs(hit) - 1;
    uint32_t b = 0u, a = 0u;
    if (lane == src) {
        uint32_t run = excl;
        bool found = false;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            if (!found && run + cnt[e] >= need) {
                found = true;
                b = (uint32_t)(kBins - 1 - 8 * lane - e);
                a = run;
            }
            if (!found) run += cnt[e];
        }
    }
    bin = __shfl_sync(0xffffffffu, b, src);
    above = __shfl_sync(0xffffffffu, a, src);
}

// Fallback: T = the k-th largest of keys[0..C) (1 <= k < C) and
// need = k - count(key > T) by four 8-bit radix digits, most significant
// first, over the whole row.  Invariant before each digit: `need` of the
// keys whose higher digits equal `prefix` are still to be taken.
__device__ void radix_threshold(const uint32_t *keys, int C, uint32_t k, uint32_t *hist,
                                uint32_t &T, uint32_t &need) {
    const int lane = threadIdx.x & 31;
    uint32_t prefix = 0u, pmask = 0u;
    need = k;
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int b = lane; b < kBins; b += 32) hist[b] = 0u;
        __syncwarp();
        for (int c = lane; c < C; c += 32) {
            const uint32_t kc = keys[c];
            if ((kc & pmask) == prefix) atomicAdd(&hist[(kc >> shift) & 0xffu], 1u);
        }
        __syncwarp();
        uint32_t digit, above;
        find_bin(hist, need, digit, above);
        need -= above;
        prefix |= digit << shift;
        pmask |= 0xffu << shift;
        __syncwarp();  // every lane has read hist before the next digit clears it
    }
    T = prefix;
}

// T = the need1-th largest of list[0..m) (1 <= need1 <= m) and
// need = need1 - count(list > T).  Keys are > 0.
//   m <= 64: every list element gets its rank in a strict order (key
//   descending, list position ascending) from all-pairs comparisons via
//   shuffles (independent, so they pipeline); the element of rank need1-1
//   holds T.
//   m > 64: a bitwise search for the largest t with count(list >= t) >=
//   need1, starting below the list's common leading bits.
__device__ void list_threshold(const uint32_t *list, int m, uint32_t need1, uint32_t &T,
                               uint32_t &need) {
    const int lane = threadIdx.x & 31;
    if (m <= 64) {
        const uint32_t a0 = lane < m ? list[lane] : 0u;
        const uint32_t a1 = lane + 32 < m ? list[lane + 32] : 0u;
        uint32_t r0 = 0u, r1 = 0u;  // ranks of elements lane and lane + 32
#pragma unroll 8
        for (int f = 0; f < 32; ++f) {
            const uint32_t b0 = __shfl_sync(0xffffffffu, a0, f);  // element f
            const uint32_t b1 = __shfl_sync(0xffffffffu, a1, f);  // element f + 32
            r0 += (b0 > a0 || (b0 == a0 && f < lane)) ? 1u : 0u;
            r0 += b1 > a0 ? 1u : 0u;  // position f + 32 is after lane
            r1 += b0 >= a1 ? 1u : 0u;  // position f is before lane + 32
            r1 += (b1 > a1 || (b1 == a1 && f < lane)) ? 1u : 0u;
        }
        // Padding elements are 0, below every key: they never outrank one.
        const bool h0 = lane < m && r0 == need1 - 1u;
        const bool h1 = lane + 32 < m && r1 == need1 - 1u;
        const unsigned hb = __ballot_sync(0xffffffffu, h0 || h1);
        const int src = __ffs(hb) - 1;
        T = __shfl_sync(0xffffffffu, h0 ? a0 : a1, src);
        need = need1 - (uint32_t)(__popc(__ballot_sync(0xffffffffu, a0 > T)) +
                                  __popc(__ballot_sync(0xffffffffu, a1 > T)));
        return;
    }
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    for (int c = lane; c < m; c += 32) {
        const uint32_t v = list[c];
        kmin = min(kmin, v);
        kmax = max(kmax, v);
    }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    const int p = __clz(kmin ^ kmax);  // common leading bits; 32 when all equal
    uint32_t prefix = p == 32 ? kmin : (p == 0 ? 0u : kmin & ~(0xffffffffu >> p));
    for (int bit = 31 - p; bit >= 0; --bit) {
        const uint32_t cand = prefix | (1u << bit);
        uint32_t n = 0u;
        for (int c = lane; c < m; c += 32) n += list[c] >= cand ? 1u : 0u;
        if (__reduce_add_sync(0xffffffffu, n) >= need1) prefix = cand;
    }
    T = prefix;
    uint32_t gt = 0u;
    for (int c = lane; c < m; c += 32) gt += list[c] > T ? 1u : 0u;
    need = need1 - __reduce_add_sync(0xffffffffu, gt);
}

// Warp w selects rows w and w + 8 of the CTA's score rows (keys, row stride
// `stride`), writing the forward block list of each row that exists.
//   hist_rows  [kRows][256] candidate histograms built while scoring, or
//              NULL to build them here;
//   scratch    per-warp scratch of `words` 32-bit words (histogram when
//              hist_rows is NULL, then the bucket list).
// `failed` rows (a timed-out CTA) get an empty list.
__device__ void select_rows(const uint32_t *srows, int stride, const uint32_t *hist_rows,
                           uint32_t *scratch, int words, int64_t bh, int64_t i0, int64_t nQB,
                           int nKB, int nF, int k, bool failed, int32_t *__restrict__ kv_idx,
                           int32_t *__restrict__ kv_cnt, int64_t max_sel) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned lt_mask = (1u << lane) - 1u;
    uint32_t *ws = scratch + warp * words;
    const int C = nKB - nF;
    for (int r = warp; r < kRows; r += kWarps) {
        const int64_t i = i0 + r;
        if (i >= nQB) break;  // warp-uniform; later rows are further out
        const int64_t grow = bh * nQB + i;
        int32_t *out = kv_idx + grow * max_sel;
        int written = 0;
        if (!failed) {
            for (int f = lane; f < nF; f += 32) out[f] = f;
            written = nF;
        }
        if (!failed && k > 0) {
            const uint32_t *keys = srows + r * stride + nF;
            uint32_t T = 0u, need = 0u;  // k == C: every key is > 0, all taken
            if (k < C) {
                const uint32_t *hist = hist_rows ? hist_rows + r * kBins : ws;
                if (!hist_rows) {
                    for (int b = lane; b < kBins; b += 32) ws[b] = 0u;
                    __syncwarp();
                    for (int c = lane; c < C; c += 32)
                        atomicAdd(&ws[bucket_of(key_value(keys[c]))], 1u);
                    __syncwarp();
                }
                uint32_t bin, above;
                find_bin(hist, (uint32_t)k, bin, above);
                const uint32_t lo = bucket_lo_key((int)bin);
                const bool open = bin == kBins - 1;
                const uint32_t hi = open ? 0u : bucket_lo_key((int)bin + 1);
                uint32_t *list = hist_rows ? ws : ws + kBins;
                const int cap = hist_rows ? words : words - kBins;
                __syncwarp();  // the histogram has been read before the list overwrites it
                int m = 0;
#pragma unroll 8
                for (int base = 0; base < C; base += 32) {
                    const int c = base + lane;
                    const uint32_t kc = c < C ? keys[c] : 0u;
                    const bool in = c < C && kc >= lo && (open || kc < hi);
                    const unsigned bal = __ballot_sync(0xffffffffu, in);
                    const int pos = m + __popc(bal & lt_mask);
                    if (in && pos < cap) list[pos] = kc;
                    m += __popc(bal);
                }
                __syncwarp();
                if (m <= cap)
                    list_threshold(list, m, (uint32_t)k - above, T, need);
                else
                    radix_threshold(keys, C, (uint32_t)k, ws, T, need);
                __syncwarp();  // list reads done before the next row reuses it
            }
            uint32_t ties_seen = 0u;
#pragma unroll 8
            for (int base = 0; base < C; base += 32) {
                const int c = base + lane;
                const bool valid = c < C;
                const uint32_t kc = valid ? keys[c] : 0u;
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
        }
        for (int64_t s = written + lane; s < max_sel; s += 32) out[s] = -1;
        if (lane == 0) kv_cnt[grow] = failed ? 0 : nF + k;
    }
}

// ---------------------------------------------------------- tiled scores

constexpr int kTileW = 256;                        // key blocks per tile (TMA box rows)
constexpr int kChunkD = 32;                        // d values per chunk: 128-byte rows
constexpr int kSlots = 3;                          // ring depth, in chunks
constexpr int kChunkBytes = kTileW * kChunkD * 4;  // 32 KB
constexpr int kQChunkBytes = kRows * kChunkD * 4;  // 2 KB
constexpr int64_t kTiledMaxNkb = 1664;
constexpr int kHistBytes = kRows * kBins * 4;      // 16 KB: per-row candidate histograms

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded poll (about two seconds of %globaltimer); false on expiry.
__device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = globaltimer();
    while (!mbar_test(bar, parity))
        if (globaltimer() - t0 > kTimeoutNs) return false;
    return true;
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    return mbar_test(bar, parity) || mbar_wait_slow(bar, parity);
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

// 16-byte column j of row `row` of a 128-byte-row, 128-byte-swizzled buffer.
__device__ __forceinline__ float4 ld_sw128(const unsigned char *buf, int row, int j) {
    return *reinterpret_cast<const float4 *>(buf + row * 128 + ((j ^ (row & 7)) << 4));
}

// One 32-wide d-chunk of the 16 x 256 tile: rows rg + 4a (a < 4), columns
// cg + 64e (e < NE).  Each accumulator takes its 32 FMAs in ascending d;
// the 4 x NE accumulators are interleaved so that consecutive FMAs are
// independent, and the shared loads of the next 4 values of d are issued
// before the current ones are multiplied.
template <int NE>
__device__ __forceinline__ void chunk_fma(const unsigned char *qc, const unsigned char *kc, int rg,
                                          int cg, float (&acc)[4][4]) {
    float4 qv[2][4], kv[2][NE];
#pragma unroll
    for (int a = 0; a < 4; ++a) qv[0][a] = ld_sw128(qc, rg + 4 * a, 0);
#pragma unroll
    for (int e = 0; e < NE; ++e) kv[0][e] = ld_sw128(kc, cg + 64 * e, 0);
#pragma unroll
    for (int j = 0; j < kChunkD / 4; ++j) {  // d = 4j .. 4j+3 of the chunk
        const int cur = j & 1, nxt = cur ^ 1;
        if (j + 1 < kChunkD / 4) {
#pragma unroll
            for (int a = 0; a < 4; ++a) qv[nxt][a] = ld_sw128(qc, rg + 4 * a, j + 1);
#pragma unroll
            for (int e = 0; e < NE; ++e) kv[nxt][e] = ld_sw128(kc, cg + 64 * e, j + 1);
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int e = 0; e < NE; ++e) acc[a][e] = __fmaf_rn(qv[cur][a].x, kv[cur][e].x, acc[a][e]);
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int e = 0; e < NE; ++e) acc[a][e] = __fmaf_rn(qv[cur][a].y, kv[cur][e].y, acc[a][e]);
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int e = 0; e < NE; ++e) acc[a][e] = __fmaf_rn(qv[cur][a].z, kv[cur][e].z, acc[a][e]);
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int e = 0; e < NE; ++e) acc[a][e] = __fmaf_rn(qv[cur][a].w, kv[cur][e].w, acc[a][e]);
    }
}

template <int D>
constexpr int64_t tiled_fixed_smem() {
    return 1024 + (int64_t)kSlots * kChunkBytes + (int64_t)(D / kChunkD) * kQChunkBytes +
           kHistBytes + 8 * kSlots;
}
inline int64_t tiled_stride(int64_t nKB) { return ceil_div(nKB, 128) * 128 + 8; }

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
score_select_tiled_kernel(const __grid_constant__ CUtensorMap tmK, const float *__restrict__ qbar,
                          int64_t nQB, int nKB, int stride, int64_t n_qtiles, float tau, int nF,
                          int k, int32_t *__restrict__ kv_idx, int32_t *__restrict__ kv_cnt,
                          int64_t max_sel, int32_t *status) {
    constexpr int kChunks = D / kChunkD;  // chunks per tile
    extern __shared__ __align__(16) unsigned char smem_raw[];
    // The 128-byte swizzle repeats every 1024 bytes: align the ring to that.
    unsigned char *ks = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    unsigned char *qs = ks + kSlots * kChunkBytes;
    uint32_t *hist = reinterpret_cast<uint32_t *>(qs + kChunks * kQChunkBytes);  // [kRows][256]
    uint64_t *bars = reinterpret_cast<uint64_t *>(hist + kRows * kBins);
    uint32_t *srows = reinterpret_cast<uint32_t *>(bars + kSlots);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t bh = blockIdx.x / n_qtiles;
    const int64_t i0 = (blockIdx.x - bh * n_qtiles) * kRows;
    const int ntiles = (nKB + kTileW - 1) / kTileW;
    const int nsteps = ntiles * kChunks;
    auto bar = [&](int s) { return smem_addr(bars + s); };
    auto issue = [&](int step) {  // thread 0 only
        const int slot = step % kSlots;
        mbar_expect_tx(bar(slot), kChunkBytes);
        tma_load_3d(smem_addr(ks + slot * kChunkBytes), &tmK, bar(slot),
                    (step % kChunks) * kChunkD, (step / kChunks) * kTileW, (int)bh);
    };

    int issued = 0;  // meaningful in thread 0
    if (tid == 0) {
        for (int s = 0; s < kSlots; ++s) mbar_init(bar(s), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        for (; issued < kSlots && issued < nsteps; ++issued) issue(issued);
    }
    // Query means, swizzled like the key chunks; rows past nQB are zero.
    for (int idx = tid; idx < kRows * (D / 4); idx += kThreads) {
        const int row = idx / (D / 4), v = idx % (D / 4);
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i0 + row < nQB) a = *reinterpret_cast<const float4 *>(qbar + ((bh * nQB) + i0 + row) * D + 4 * v);
        *reinterpret_cast<float4 *>(qs + (v / 8) * kQChunkBytes + row * 128 +
                                    (((v % 8) ^ (row & 7)) << 4)) = a;
    }
    for (int idx = tid; idx < kRows * kBins; idx += kThreads) hist[idx] = 0u;
    __syncthreads();

    const int rg = lane & 3;               // rows rg + 4a
    const int cg = warp * 8 + (lane >> 2);  // columns cg + 64e of the tile
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[a][e] = 0.0f;
    bool failed = false;
    int step = 0;
#pragma unroll 1
    for (; step < nsteps; ++step) {
        const int slot = step % kSlots, t = step / kChunks, c = step % kChunks;
        const bool ok = mbar_wait(bar(slot), (uint32_t)(step / kSlots) & 1u);
        const unsigned char *kc = ks + slot * kChunkBytes;
        const unsigned char *qc = qs + c * kQChunkBytes;
        // A tile with at most 128 live columns computes only e = 0, 1.
        const bool half = nKB - t * kTileW <= 128;
        if (half)
            chunk_fma<2>(qc, kc, rg, cg, acc);
        else
            chunk_fma<4>(qc, kc, rg, cg, acc);
        if (c == kChunks - 1) {  // tile done: keys into the score rows, candidates counted
            const int j0 = t * kTileW;
            const int ne = half ? 2 : 4;
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if (e < ne) {
                        const float sv = __fmul_rn(acc[a][e], tau);
                        const int j = j0 + cg + 64 * e;
                        srows[(rg + 4 * a) * stride + j] = order_key(sv);
                        if (j >= nF && j < nKB)
                            atomicAdd(&hist[(rg + 4 * a) * kBins + bucket_of(sv)], 1u);
                    }
                    acc[a][e] = 0.0f;
                }
        }
        // Every thread is done with this slot (and learns of any timeout).
        if (__syncthreads_or(!ok)) {
            failed = true;
            break;
        }
        if (tid == 0 && issued < nsteps) issue(issued++);
    }
    if (failed) {
        // Let the copies in flight land (bounded) before the CTA exits.
        if (tid == 0) {
            for (int s = step; s < issued; ++s) mbar_wait(bar(s % kSlots), (uint32_t)(s / kSlots) & 1u);
            if (status) atomicOr(status, SPARSTAR_STATUS_TIMEOUT);
        }
        __syncthreads();
    }
    // The ring is idle: it becomes the per-warp bucket lists (12 KB each,
    // more than any row's candidates).
    select_rows(srows, stride, hist, reinterpret_cast<uint32_t *>(ks),
                kSlots * kChunkBytes / 4 / kWarps, bh, i0, nQB, nKB, nF, k, failed, kv_idx,
                kv_cnt, max_sel);
}

// ------------------------------------------------------- column scores
//
// The column kernel (nKB <= 256 * kMaxNc), 512 threads: thread t owns key
// columns t % 256 + 256 c (c < NC) and the 8 query rows 8 (t / 256) .. +7 of
// the CTA's 16, so it accumulates 8 x NC outputs as 4 x NC float2 row pairs
// advanced by the packed fp32x2 FMA (two independent round-to-nearest fmas
// per instruction).  Key means arrive by TMA as 16-wide d-chunks of every
// key column (NC boxes of 16 floats x 256 rows, 64-byte rows, 64-byte
// swizzle) through a two-slot ring; the query means sit in shared memory,
// row pairs interleaved, and every read of them is a warp-wide broadcast.
// Per 4 values of d a thread issues NC key loads (one wavefront per 8 lanes)
// and 8 query loads for 16 NC packed FMAs; a warp whose columns in the last
// block all lie past nKB skips that block.  Each output takes its FMAs in
// ascending d from acc = +0, so the scores are bit for bit those of the
// other kernels.
// When the last chunk is multiplied the ring is idle and holds the score
// rows.
//
// Its selection (select_rows_bits) keeps one row per warp in registers:
// lane l holds the row's columns l * kpl .. l * kpl + kpl - 1 (kpl a
// multiple of 4 whose quarter is odd, so the lanes' 16-byte loads spread
// over all banks; the selection is compiled for both values kpl takes at a
// given NC), non-candidates as key 0 (every score's key is above 0).
// The threshold T, the k-th largest key, comes from a bitwise search below
// the row's common leading bits, each step one count over the registers
// and a warp sum, that narrows a window [prefix, prefix + 2^(b+1)) holding
// T (on long rows whose keys span several binades, T's binade is found
// first by galloping from kmax or kmin and bisecting); once the window
// holds at most 64 keys they are compacted into a per-warp list, two keys
// per lane, and the bitwise search goes on over those registers down to
// bit 0.  Then every lane counts its keys > T and == T, and a warp prefix
// sum places them: all keys > T and the first k - count(> T) keys == T in
// ascending column order (ties to the lower block index; the prefix sum
// over the ties only runs when there are more keys == T than places).  The
// same lists as select_rows.

constexpr int kMaxNc = 6;          // up to 1536 key blocks
constexpr int kColRing = 2;        // ring depth, in chunks
constexpr int kColChunkD = 16;     // d values per chunk (64-byte rows)
constexpr int kColThreads = 512;   // two row groups of 256 column threads
constexpr int kColWarps = kColThreads / 32;
constexpr int kGroupRows = kRows / 2;

// Lane segment length: the smallest multiple of 4 with an odd quarter that
// covers nKB with 32 lanes.
constexpr int seg_len(int nKB) {
    int q = (nKB + 127) / 128;  // quarter of ceil(nKB / 32), rounded up
    return 4 * (q | 1);
}
constexpr int kpl_max(int NC) { return seg_len(256 * NC); }
constexpr int64_t col_stride(int NC) { return 32LL * kpl_max(NC); }
constexpr int64_t col_slot_bytes(int NC) { return (int64_t)NC * 256 * kColChunkD * 4; }
constexpr int64_t col_rows_bytes(int NC) { return 4LL * kRows * col_stride(NC); }
constexpr int64_t col_region_bytes(int NC) {
    return kColRing * col_slot_bytes(NC) > col_rows_bytes(NC) ? kColRing * col_slot_bytes(NC)
                                                              : col_rows_bytes(NC);
}
static_assert(kColRing * col_slot_bytes(1) >= col_rows_bytes(1) + kColWarps * 64 * 4 &&
                  kColRing * col_slot_bytes(6) >= col_rows_bytes(6) + kColWarps * 64 * 4,
              "the ring region holds the score rows and the per-warp window lists");
template <int D, int NC>
constexpr int64_t col_smem() {
    return 1024 + col_region_bytes(NC) + (int64_t)kRows * D * 4 + 8 * kColRing;
}

// Warp-wide exclusive prefix sum of v; *total receives the sum.
__device__ __forceinline__ uint32_t warp_excl_scan(uint32_t v, uint32_t &total) {
    const int lane = threadIdx.x & 31;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    total = __shfl_sync(0xffffffffu, incl, 31);
    return incl - v;
}

// Selection of the CTA's rows from register-held segments (see above).
// Same contract as select_rows, with NW warps: warp w takes rows w, w + NW,
// ...; `failed` rows get an empty list.
constexpr uint32_t kWindowList = 64;  // window size at which the search moves to a list

template <int KPL, int NW>
__device__ void select_rows_bits(const uint32_t *srows, int stride, int kpl, uint32_t *scratch,
                                 int64_t bh, int64_t i0, int64_t nQB, int nKB, int nF, int k,
                                 bool failed, int32_t *__restrict__ kv_idx,
                                 int32_t *__restrict__ kv_cnt, int64_t max_sel) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t *list = scratch + warp * kWindowList;
    const int C = nKB - nF;
    const int c0 = lane * kpl;  // first column of this lane's segment
    for (int r = warp; r < kRows; r += NW) {
        const int64_t i = i0 + r;
        if (i >= nQB) break;  // warp-uniform; later rows are further out
        const int64_t grow = bh * nQB + i;
        int32_t *out = kv_idx + grow * max_sel;
        int written = 0;
        if (!failed) {
            for (int f = lane; f < nF; f += 32) out[f] = f;
            written = nF;
        }
        if (!failed && k > 0) {
            // Candidate keys of this lane's segment; the score rows hold 0
            // for the forced blocks and past nKB, below every candidate key.
            uint32_t v[KPL];
            const uint32_t *seg = srows + r * stride + c0;
#pragma unroll
            for (int g = 0; g < KPL / 4; ++g) {
                uint4 w4 = make_uint4(0u, 0u, 0u, 0u);
                if (4 * g < kpl) w4 = *reinterpret_cast<const uint4 *>(seg + 4 * g);
                v[4 * g] = w4.x;
                v[4 * g + 1] = w4.y;
                v[4 * g + 2] = w4.z;
                v[4 * g + 3] = w4.w;
            }
            uint32_t T = 0u;  // k == C: every candidate key is > 0, all taken
            if (k < C) {
                // Four partial minima and maxima (shorter dependency chains).
                uint32_t mn[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
                uint32_t mx[4] = {0u, 0u, 0u, 0u};
#pragma unroll
                for (int e = 0; e < KPL; ++e) {
                    if (v[e]) mn[e & 3] = min(mn[e & 3], v[e]);
                    mx[e & 3] = max(mx[e & 3], v[e]);
                }
                uint32_t kmin = min(min(mn[0], mn[1]), min(mn[2], mn[3]));
                uint32_t kmax = max(max(mx[0], mx[1]), max(mx[2], mx[3]));
                kmin = __reduce_min_sync(0xffffffffu, kmin);
                kmax = __reduce_max_sync(0xffffffffu, kmax);
                // The k-th largest key: the largest t with count(key >= t) >= k,
                // built bit by bit below the common leading bits of kmin, kmax.
                // The window [prefix, prefix + 2^(bit+1)) holds it, with
                // count(>= prefix) = lo >= k and count(>= window end) = hi < k.
                auto count_ge = [&](uint32_t cand) {  // warp-wide count of keys >= cand
                    uint32_t nc[4] = {0u, 0u, 0u, 0u};  // KPL is a multiple of 4
#pragma unroll
                    for (int e = 0; e < KPL; ++e) nc[e & 3] += v[e] >= cand ? 1u : 0u;
                    return __reduce_add_sync(0xffffffffu, (nc[0] + nc[1]) + (nc[2] + nc[3]));
                };
                const int p = __clz(kmin ^ kmax);
                uint32_t prefix = p == 32 ? kmin : (p == 0 ? 0u : kmin & ~(0xffffffffu >> p));
                uint32_t lo = (uint32_t)C, hi = 0u;
                int bit = 31 - p;
                if (p < 9 && C > 4 * (int)kWindowList) {
                    // kmin and kmax lie in different binades (the top 9 key bits:
                    // sign and exponent) and the row is long: find T's binade
                    // first, galloping from the end nearer to T (from kmax when
                    // k <= C / 2, else from kmin), then bisecting; counts are of
                    // keys >= j << 23.  (Short rows reach the 64-key window in a
                    // few bitwise steps anyway.)
                    // Invariant: count(>= j << 23) = lo >= k > hi = count(>= jh << 23).
                    const uint32_t jmin = kmin >> 23, jmax = kmax >> 23;
                    uint32_t j, jh;
                    if (2 * (uint32_t)k <= (uint32_t)C) {
                        j = jmax;
                        jh = jmax + 1;  // nothing lies above kmax's binade: hi = 0
                        lo = count_ge(j << 23 > 1u ? j << 23 : 1u);
                        for (uint32_t d = 1; lo < (uint32_t)k; d <<= 1) {
                            jh = j;
                            hi = lo;
                            j = j > jmin + d ? j - d : jmin;  // all C keys lie >= jmin << 23
                            lo = count_ge(j << 23 > 1u ? j << 23 : 1u);
                        }
                    } else {
                        j = jmin;  // lo = C
                        jh = jmin + 1;
                        hi = count_ge(jh << 23);
                        for (uint32_t d = 2; hi >= (uint32_t)k; d <<= 1) {
                            j = jh;
                            lo = hi;
                            jh = jh + d < jmax + 1 ? jh + d : jmax + 1;
                            hi = jh == jmax + 1 ? 0u : count_ge(jh << 23);
                        }
                    }
                    while (jh - j > 1) {
                        const uint32_t jm = (j + jh) >> 1;
                        const uint32_t cm = count_ge(jm << 23);
                        if (cm >= (uint32_t)k) {
                            j = jm;
                            lo = cm;
                        } else {
                            jh = jm;
                            hi = cm;
                        }
                    }
                    prefix = j << 23;
                    bit = 22;  // the window is binade j: [j << 23, (j + 1) << 23)
                }
                for (; bit >= 0 && lo - hi > kWindowList; --bit) {
                    const uint32_t cand = prefix | (1u << bit);
                    const uint32_t c = count_ge(cand);
                    if (c >= (uint32_t)k) {
                        prefix = cand;
                        lo = c;
                    } else {
                        hi = c;
                    }
                }
                if (bit < 0) {
                    T = prefix;  // the window is one key value
                } else {
                    // The window's lo - hi keys into the list, then the
                    // (k - hi)-th largest of them.  Non-candidates are key 0,
                    // below every candidate: the window starts at 1 at least.
                    const uint32_t start = prefix > 1u ? prefix : 1u;
                    const uint64_t end = (uint64_t)prefix + (2ull << bit);
                    uint32_t n_in = 0u;
#pragma unroll
                    for (int e = 0; e < KPL; ++e)
                        n_in += (v[e] >= start && (uint64_t)v[e] < end) ? 1u : 0u;
                    uint32_t m;
                    uint32_t pos = warp_excl_scan(n_in, m);
#pragma unroll
                    for (int e = 0; e < KPL; ++e)
                        if (v[e] >= start && (uint64_t)v[e] < end) list[pos++] = v[e];
                    __syncwarp();
                    // The bitwise search goes on over the list, two keys per
                    // lane: T = the largest t with count(list >= t) >= k - hi.
                    const uint32_t a0 = lane < (int)m ? list[lane] : 0u;
                    const uint32_t a1 = lane + 32 < (int)m ? list[lane + 32] : 0u;
                    __syncwarp();  // list reads done before the next row reuses it
                    const uint32_t need1 = (uint32_t)k - hi;
                    for (; bit >= 0; --bit) {
                        const uint32_t cand = prefix | (1u << bit);
                        const uint32_t c = __reduce_add_sync(
                            0xffffffffu, (a0 >= cand ? 1u : 0u) + (a1 >= cand ? 1u : 0u));
                        if (c >= need1) prefix = cand;
                    }
                    T = prefix;
                }
            }
            uint32_t n_gt = 0u, n_eq = 0u;
#pragma unroll
            for (int e = 0; e < KPL; ++e) {
                n_gt += v[e] > T ? 1u : 0u;
                n_eq += v[e] == T ? 1u : 0u;
            }
            const uint32_t gt_total = __reduce_add_sync(0xffffffffu, n_gt);
            const uint32_t eq_total = __reduce_add_sync(0xffffffffu, n_eq);
            const uint32_t need = (uint32_t)k - gt_total;  // keys == T still to take
            // Ties go to the lower block index: the first `need` keys == T in
            // ascending column order, i.e. lane order then register order.
            // Without surplus ties (eq_total == need) every key == T is taken.
            uint32_t eq_take = n_eq;
            if (eq_total > need) {  // warp-uniform
                uint32_t tmp;
                const uint32_t eq_before = warp_excl_scan(n_eq, tmp);
                eq_take = need > eq_before ? min(need - eq_before, n_eq) : 0u;
            }
            uint32_t taken;
            uint32_t dst = (uint32_t)nF + warp_excl_scan(n_gt + eq_take, taken);
            uint32_t eq_seen = 0u;
#pragma unroll
            for (int e = 0; e < KPL; ++e) {
                const bool eq = v[e] == T;
                if (v[e] > T || (eq && eq_seen < eq_take)) out[dst++] = c0 + e;
                eq_seen += eq ? 1u : 0u;
            }
            written = nF + (int)taken;
        }
        for (int64_t s2 = written + lane; s2 < max_sel; s2 += 32) out[s2] = -1;
        if (lane == 0) kv_cnt[grow] = failed ? 0 : nF + k;
    }
}

// One 16-wide d-chunk of the column kernel's product for the first NCC of
// the thread's NC column blocks: per d, one packed fp32x2 FMA per (column,
// row pair), the key mean in both halves; each half is the same
// round-to-nearest fma as the scalar form, in ascending d.
template <int D, int NCC, int NC>
__device__ __forceinline__ void col_chunk_fma(const unsigned char *kc, const float *qg, int step,
                                              int swz, float2 (&acc)[NC][kGroupRows / 2]) {
#pragma unroll
    for (int h = 0; h < kColChunkD / 4; ++h) {  // d = 16 step + 4h .. + 3
        float4 kv[NCC > 0 ? NCC : 1], qv[kGroupRows / 2][2];
#pragma unroll
        for (int c = 0; c < NCC; ++c)
            kv[c] = *reinterpret_cast<const float4 *>(kc + c * 256 * kColChunkD * 4 +
                                                      ((h ^ swz) << 4));
#pragma unroll
        for (int pr = 0; pr < kGroupRows / 2; ++pr)
#pragma unroll
            for (int e = 0; e < 2; ++e)
                qv[pr][e] = *reinterpret_cast<const float4 *>(
                    qg + (pr * D + kColChunkD * step + 4 * h + 2 * e) * 2);
#pragma unroll
        for (int pr = 0; pr < kGroupRows / 2; ++pr)
#pragma unroll
            for (int c = 0; c < NCC; ++c)
                acc[c][pr] = __ffma2_rn(make_float2(qv[pr][0].x, qv[pr][0].y), make_float2(kv[c].x, kv[c].x),
                                        acc[c][pr]);
#pragma unroll
        for (int pr = 0; pr < kGroupRows / 2; ++pr)
#pragma unroll
            for (int c = 0; c < NCC; ++c)
                acc[c][pr] = __ffma2_rn(make_float2(qv[pr][0].z, qv[pr][0].w), make_float2(kv[c].y, kv[c].y),
                                        acc[c][pr]);
#pragma unroll
        for (int pr = 0; pr < kGroupRows / 2; ++pr)
#pragma unroll
            for (int c = 0; c < NCC; ++c)
                acc[c][pr] = __ffma2_rn(make_float2(qv[pr][1].x, qv[pr][1].y), make_float2(kv[c].z, kv[c].z),
                                        acc[c][pr]);
#pragma unroll
        for (int pr = 0; pr < kGroupRows / 2; ++pr)
#pragma unroll
            for (int c = 0; c < NCC; ++c)
                acc[c][pr] = __ffma2_rn(make_float2(qv[pr][1].z, qv[pr][1].w), make_float2(kv[c].w, kv[c].w),
                                        acc[c][pr]);
    }
}

template <int D, int NC>
__global__ void __launch_bounds__(kColThreads, 1)
score_select_cols_kernel(const __grid_constant__ CUtensorMap tmK, const float *__restrict__ qbar,
                         int64_t nQB, int nKB, int kpl, int64_t n_qtiles, float tau, int nF,
                         int k, int32_t *__restrict__ kv_idx, int32_t *__restrict__ kv_cnt,
                         int64_t max_sel, int32_t *status) {
    constexpr int kChunks = D / kColChunkD;
    constexpr int kSlotBytes = (int)col_slot_bytes(NC);
    constexpr int kStride = (int)col_stride(NC);
    extern __shared__ __align__(16) unsigned char smem_raw[];
    unsigned char *ks = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    float *qs = reinterpret_cast<float *>(ks + col_region_bytes(NC));     // [kRows][D]
    uint64_t *bars = reinterpret_cast<uint64_t *>(qs + kRows * D);
    uint32_t *srows = reinterpret_cast<uint32_t *>(ks);  // after scoring: [kRows][kStride]

    const int tid = threadIdx.x;
    const int grp = tid / 256, tc = tid % 256;  // row group (rows 8 grp ..), column thread
    const int64_t bh = blockIdx.x / n_qtiles;
    const int64_t i0 = (blockIdx.x - bh * n_qtiles) * kRows;
    auto bar = [&](int sl) { return smem_addr(bars + sl); };
    auto issue = [&](int step) {  // thread 0 only: chunk `step` of every column
        const int slot = step % kColRing;
        mbar_expect_tx(bar(slot), kSlotBytes);
#pragma unroll
        for (int b = 0; b < NC; ++b)
            tma_load_3d(smem_addr(ks + slot * kSlotBytes + b * 256 * kColChunkD * 4), &tmK,
                        bar(slot), step * kColChunkD, b * 256, (int)bh);
    };

    int issued = 0;  // meaningful in thread 0
    if (tid == 0) {
        for (int sl = 0; sl < kColRing; ++sl) mbar_init(bar(sl), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        for (; issued < kColRing && issued < kChunks; ++issued) issue(issued);
    }
    for (int idx = tid; idx < kRows * (D / 4); idx += kColThreads) {
        const int row = idx / (D / 4), v = idx % (D / 4);
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i0 + row < nQB)
            a = *reinterpret_cast<const float4 *>(qbar + ((bh * nQB) + i0 + row) * D + 4 * v);
        // Row pairs interleaved: float2 (row 2P, row 2P + 1) of group g at d
        // is qs[((4 g + P) D + d) 2 ..].
        float *dst = qs + (((row / kGroupRows) * (kGroupRows / 2) + (row % kGroupRows) / 2) * D +
                           4 * v) * 2 + (row % 2);
        dst[0] = a.x;
        dst[2] = a.y;
        dst[4] = a.z;
        dst[6] = a.w;
    }
    __syncthreads();

    // This thread: rows 8 grp .. 8 grp + 7, columns tc + 256 c.  Its column's
    // 64-byte row in a box holds d chunks of 16 bytes, chunk h stored at
    // h ^ ((tc >> 1) & 3) (the 64-byte swizzle), which spreads a warp's
    // loads of one chunk over all banks.
    const float *qg = qs + grp * kGroupRows * D;
    const int swz = (tc >> 1) & 3;
    // A warp whose lowest column in the last column block is past nKB skips
    // that block (its outputs are never written).
    const bool last_live = (tc & ~31) + 256 * (NC - 1) < nKB;
    float2 acc[NC][kGroupRows / 2];  // (row 2P, row 2P + 1) of column c
#pragma unroll
    for (int c = 0; c < NC; ++c)
#pragma unroll
        for (int r = 0; r < kGroupRows / 2; ++r) acc[c][r] = make_float2(0.0f, 0.0f);
    bool failed = false;
    int step = 0;
#pragma unroll 1
    for (; step < kChunks; ++step) {
        const int slot = step % kColRing;
        const bool ok = mbar_wait(bar(slot), (uint32_t)(step / kColRing) & 1u);
        const unsigned char *kc = ks + slot * kSlotBytes + tc * kColChunkD * 4;
        if (last_live)
            col_chunk_fma<D, NC, NC>(kc, qg, step, swz, acc);
        else
            col_chunk_fma<D, NC - 1, NC>(kc, qg, step, swz, acc);
        // Every thread is done with this slot (and learns of any timeout).
        if (__syncthreads_or(!ok)) {
            failed = true;
            break;
        }
        if (tid == 0 && issued < kChunks) issue(issued++);
    }
    if (failed) {
        if (tid == 0) {
            for (int st = step; st < issued; ++st)
                mbar_wait(bar(st % kColRing), (uint32_t)(st / kColRing) & 1u);
            if (status) atomicOr(status, SPARSTAR_STATUS_TIMEOUT);
        }
        __syncthreads();
    } else {
        // Keys into the score rows, over the ring: every thread is past the
        // last chunk, and no copy is in flight.  Forced blocks and columns
        // past nKB hold key 0 (below every score's key), so the selection
        // reads its segments without masking.
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            const int j = tc + 256 * c;
            const bool cand = j >= nF && j < nKB;
#pragma unroll
            for (int pr = 0; pr < kGroupRows / 2; ++pr) {
                srows[(grp * kGroupRows + 2 * pr) * kStride + j] =
                    cand ? order_key(__fmul_rn(acc[c][pr].x, tau)) : 0u;
                srows[(grp * kGroupRows + 2 * pr + 1) * kStride + j] =
                    cand ? order_key(__fmul_rn(acc[c][pr].y, tau)) : 0u;
            }
        }
        // Segments may reach past the 256 NC columns (32 kpl > 256 NC).
        for (int idx = tid; idx < kRows * (32 * kpl - 256 * NC); idx += kColThreads) {
            const int w = 32 * kpl - 256 * NC;
            srows[(idx / w) * kStride + 256 * NC + idx % w] = 0u;
        }
        __syncthreads();
    }
    // kpl is kpl_max(NC) or kpl_max(NC) - 8 (seg_len of nKB in (256 (NC - 1), 256 NC]);
    // the selection loops run over exactly kpl registers.
    if (kpl == kpl_max(NC))
        select_rows_bits<kpl_max(NC), kColWarps>(srows, kStride, kpl, srows + kRows * kStride,
                                                 bh, i0, nQB, nKB, nF, k, failed, kv_idx, kv_cnt,
                                                 max_sel);
    else
        select_rows_bits<kpl_max(NC) - 8, kColWarps>(srows, kStride, kpl,
                                                     srows + kRows * kStride, bh, i0, nQB, nKB,
                                                     nF, k, failed, kv_idx, kv_cnt, max_sel);
}

// ----------------------------------------------------------- wide scores

constexpr int kWTile = 128;      // key blocks per staged tile
constexpr int kKS = kWTile + 4;  // padded row stride of the transposed key tile

template <int D>
constexpr int64_t wide_fixed_smem() {
    return 4 * ((int64_t)D * kKS + (int64_t)D * kRows);
}
inline int64_t wide_stride(int64_t nKB) { return ceil_div(nKB, kWTile) * kWTile; }

// Key tile t into registers.  Chunk u of a warp covers 16 key blocks x 2
// adjacent float4 (32 contiguous bytes each): with w = warp + 8u,
// row = 16 * (w & 7) + lane / 2 and v = 2 * (w >> 3) + (lane & 1).
template <int D>
__device__ __forceinline__ void wide_load(const float *__restrict__ kb, int nKB, int t,
                                          float4 (&pre)[D / 8]) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int u = 0; u < D / 8; ++u) {
        const int w = warp + kWarps * u;
        const int row = 16 * (w & 7) + (lane >> 1);
        const int v = 2 * (w >> 3) + (lane & 1);
        const int j = t * kWTile + row;
        pre[u] = j < nKB ? *reinterpret_cast<const float4 *>(kb + (int64_t)j * D + 4 * v)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

// The registers of wide_load, transposed: ks[d][row], stride kKS.  For a
// fixed element the 32 lanes hit banks 16 * (lane & 1) + row % 16 + const.
template <int D>
__device__ __forceinline__ void wide_store(float *__restrict__ ks, const float4 (&pre)[D / 8]) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int u = 0; u < D / 8; ++u) {
        const int w = warp + kWarps * u;
        const int row = 16 * (w & 7) + (lane >> 1);
        const int v = 2 * (w >> 3) + (lane & 1);
        ks[(4 * v + 0) * kKS + row] = pre[u].x;
        ks[(4 * v + 1) * kKS + row] = pre[u].y;
        ks[(4 * v + 2) * kKS + row] = pre[u].z;
        ks[(4 * v + 3) * kKS + row] = pre[u].w;
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
score_select_wide_kernel(const float *__restrict__ qbar, const float *__restrict__ kbar,
                         int64_t nQB, int nKB, int stride, int64_t n_qtiles, float tau, int nF,
                         int k, int32_t *__restrict__ kv_idx, int32_t *__restrict__ kv_cnt,
                         int64_t max_sel) {
    extern __shared__ __align__(16) float smem[];
    float *ks = smem;                                               // [D][kKS]
    float *qs = ks + D * kKS;                                       // [D][kRows]
    uint32_t *srows = reinterpret_cast<uint32_t *>(qs + D * kRows);  // [kRows][stride]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t bh = blockIdx.x / n_qtiles;
    const int64_t i0 = (blockIdx.x - bh * n_qtiles) * kRows;
    const float *qb = qbar + bh * nQB * D;
    const float *kb = kbar + bh * (int64_t)nKB * D;

    for (int idx = tid; idx < kRows * (D / 4); idx += kThreads) {
        const int row = idx % kRows, v = idx / kRows;
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i0 + row < nQB) a = *reinterpret_cast<const float4 *>(qb + (i0 + row) * D + 4 * v);
        qs[(4 * v + 0) * kRows + row] = a.x;
        qs[(4 * v + 1) * kRows + row] = a.y;
        qs[(4 * v + 2) * kRows + row] = a.z;
        qs[(4 * v + 3) * kRows + row] = a.w;
    }

    const int rg = lane & 7;                // rows 2rg, 2rg+1
    const int cg = warp * 4 + (lane >> 3);  // columns 4cg .. 4cg+3
    const int ntiles = (nKB + kWTile - 1) / kWTile;
    float4 pre[D / 8];
    wide_load<D>(kb, nKB, 0, pre);
#pragma unroll 1
    for (int t = 0; t < ntiles; ++t) {
        __syncthreads();  // the previous tile's products are done (and qs is staged)
        wide_store<D>(ks, pre);
        __syncthreads();
        if (t + 1 < ntiles) wide_load<D>(kb, nKB, t + 1, pre);

        float acc[2][4];
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) acc[a][b] = 0.0f;
#pragma unroll 8
        for (int d = 0; d < D; ++d) {
            const float2 qv = *reinterpret_cast<const float2 *>(qs + d * kRows + 2 * rg);
            const float4 kv = *reinterpret_cast<const float4 *>(ks + d * kKS + 4 * cg);
            acc[0][0] = __fmaf_rn(qv.x, kv.x, acc[0][0]);
            acc[0][1] = __fmaf_rn(qv.x, kv.y, acc[0][1]);
            acc[0][2] = __fmaf_rn(qv.x, kv.z, acc[0][2]);
            acc[0][3] = __fmaf_rn(qv.x, kv.w, acc[0][3]);
            acc[1][0] = __fmaf_rn(qv.y, kv.x, acc[1][0]);
            acc[1][1] = __fmaf_rn(qv.y, kv.y, acc[1][1]);
            acc[1][2] = __fmaf_rn(qv.y, kv.z, acc[1][2]);
            acc[1][3] = __fmaf_rn(qv.y, kv.w, acc[1][3]);
        }
        // stride is a multiple of 128, so the whole tile lands inside the row.
#pragma unroll
        for (int a = 0; a < 2; ++a) {
            uint4 o;
            o.x = order_key(__fmul_rn(acc[a][0], tau));
            o.y = order_key(__fmul_rn(acc[a][1], tau));
            o.z = order_key(__fmul_rn(acc[a][2], tau));
            o.w = order_key(__fmul_rn(acc[a][3], tau));
            *reinterpret_cast<uint4 *>(srows + (2 * rg + a) * stride + t * kWTile + 4 * cg) = o;
        }
    }
    __syncthreads();  // all rows scored; the key-tile buffer is free
    // The key-tile buffer is idle: per-warp histogram + bucket list.
    select_rows(srows, stride, nullptr, reinterpret_cast<uint32_t *>(ks), D * kKS / kWarps, bh,
                i0, nQB, nKB, nF, k, false, kv_idx, kv_cnt, max_sel);
}

// ------------------------------------------------------------------ host

PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// kbar [BH, nKB, D] fp32 as a 3-D tensor; box = 32 floats x 256 rows x 1,
// 128-byte swizzle.  Rows past nKB read as zero.
bool encode_kbar(CUtensorMap *map, const float *kbar, int64_t BH, int64_t nKB, int D) {
    auto fn = get_encoder();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)nKB, (cuuint64_t)BH};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)nKB * D * 4};
    const cuuint32_t box[3] = {(cuuint32_t)kChunkD, (cuuint32_t)kTileW, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(kbar), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// kbar [BH, nKB, D] fp32 as a 3-D tensor; box = 16 floats x 256 rows x 1
// (64-byte rows), 64-byte swizzle.  Rows past nKB read as zero.
bool encode_kbar_cols(CUtensorMap *map, const float *kbar, int64_t BH, int64_t nKB, int D) {
    auto fn = get_encoder();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)nKB, (cuuint64_t)BH};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)nKB * D * 4};
    const cuuint32_t box[3] = {(cuuint32_t)kColChunkD, 256, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(kbar), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int NC>
cudaError_t launch_cols_nc(const float *qbar, const float *kbar, int64_t BH, int64_t nQB,
                           int64_t nKB, float tau, int64_t nF, int64_t k, int32_t *kv_idx,
                           int32_t *kv_cnt, int64_t max_sel, int32_t *status, cudaStream_t s) {
    CUtensorMap tm;
    if (!encode_kbar_cols(&tm, kbar, BH, nKB, D)) return cudaErrorInvalidValue;
    constexpr int64_t smem = col_smem<D, NC>();
    static_assert(smem <= kMaxSmem, "column kernel shared memory");
    cudaError_t e = cudaFuncSetAttribute(score_select_cols_kernel<D, NC>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t n_qtiles = ceil_div(nQB, kRows);
    score_select_cols_kernel<D, NC><<<(unsigned)(BH * n_qtiles), kColThreads, (size_t)smem, s>>>(
        tm, qbar, nQB, (int)nKB, seg_len((int)nKB), n_qtiles, tau, (int)nF, (int)k, kv_idx,
        kv_cnt, max_sel, status);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_cols(const float *qbar, const float *kbar, int64_t BH, int64_t nQB,
                        int64_t nKB, float tau, int64_t nF, int64_t k, int32_t *kv_idx,
                        int32_t *kv_cnt, int64_t max_sel, int32_t *status, cudaStream_t s) {
    switch (ceil_div(nKB, 256)) {
    case 1: return launch_cols_nc<D, 1>(qbar, kbar, BH, nQB, nKB, tau, nF, k, kv_idx, kv_cnt, max_sel, status, s);
    case 2: return launch_cols_nc<D, 2>(qbar, kbar, BH, nQB, nKB, tau, nF, k, kv_idx, kv_cnt, max_sel, status, s);
    case 3: return launch_cols_nc<D, 3>(qbar, kbar, BH, nQB, nKB, tau, nF, k, kv_idx, kv_cnt, max_sel, status, s);
    case 4: return launch_cols_nc<D, 4>(qbar, kbar, BH, nQB, nKB, tau, nF, k, kv_idx, kv_cnt, max_sel, status, s);
    case 5: return launch_cols_nc<D, 5>(qbar, kbar, BH, nQB, nKB, tau, nF, k, kv_idx, kv_cnt, max_sel, status, s);
    case 6: return launch_cols_nc<D, 6>(qbar, kbar, BH, nQB, nKB, tau, nF, k, kv_idx, kv_cnt, max_sel, status, s);
    default: return cudaErrorInvalidValue;
    }
}

template <int D>
cudaError_t launch_tiled(const float *qbar, const float *kbar, int64_t BH, int64_t nQB,
                         int64_t nKB, float tau, int64_t nF, int64_t k, int32_t *kv_idx,
                         int32_t *kv_cnt, int64_t max_sel, int32_t *status, cudaStream_t s) {
    CUtensorMap tm;
    if (!encode_kbar(&tm, kbar, BH, nKB, D)) return cudaErrorInvalidValue;
    const int64_t stride = tiled_stride(nKB);
    const int64_t smem = tiled_fixed_smem<D>() + 4 * kRows * stride;
    if (smem > kMaxSmem) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(score_select_tiled_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t n_qtiles = ceil_div(nQB, kRows);
    score_select_tiled_kernel<D><<<(unsigned)(BH * n_qtiles), kThreads, (size_t)smem, s>>>(
        tm, qbar, nQB, (int)nKB, (int)stride, n_qtiles, tau, (int)nF, (int)k, kv_idx, kv_cnt,
        max_sel, status);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_wide(const float *qbar, const float *kbar, int64_t BH, int64_t nQB,
                        int64_t nKB, float tau, int64_t nF, int64_t k, int32_t *kv_idx,
                        int32_t *kv_cnt, int64_t max_sel, cudaStream_t s) {
    const int64_t stride = wide_stride(nKB);
    const int64_t smem = wide_fixed_smem<D>() + 4 * kRows * stride;
    if (smem > kMaxSmem) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(score_select_wide_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t n_qtiles = ceil_div(nQB, kRows);
    score_select_wide_kernel<D><<<(unsigned)(BH * n_qtiles), kThreads, (size_t)smem, s>>>(
        qbar, kbar, nQB, (int)nKB, (int)stride, n_qtiles, tau, (int)nF, (int)k, kv_idx, kv_cnt,
        max_sel);
    return cudaGetLastError();
}

}  // namespace

int64_t score_select_max_nkb(int D) {
    const int64_t fixed = D == 128 ? wide_fixed_smem<128>() : wide_fixed_smem<64>();
    return (kMaxSmem - fixed) / (4 * kRows) / kWTile * kWTile;
}

int64_t score_select_tiled_max_nkb() { return kTiledMaxNkb; }

int64_t score_select_ctas(int64_t BH, int64_t nQB) { return BH * ceil_div(nQB, kRows); }

cudaError_t launch_score_select(const float *qbar, const float *kbar, int64_t BH, int64_t nQB,
                                int64_t nKB, int D, float tau, int64_t nF, int64_t k,
                                int32_t *kv_idx, int32_t *kv_cnt, int64_t max_sel,
                                int32_t *status, cudaStream_t stream) {
    if (nKB <= 256 * kMaxNc)
        return D == 128 ? launch_cols<128>(qbar, kbar, BH, nQB, nKB, tau, nF, k, kv_idx, kv_cnt,
                                           max_sel, status, stream)
                        : launch_cols<64>(qbar, kbar, BH, nQB, nKB, tau, nF, k, kv_idx, kv_cnt,
                                          max_sel, status, stream);
    if (nKB <= kTiledMaxNkb)
        return D == 128 ? launch_tiled<128>(qbar, kbar, BH, nQB, nKB, tau, nF, k, kv_idx, kv_cnt,
                                            max_sel, status, stream)
                        : launch_tiled<64>(qbar, kbar, BH, nQB, nKB, tau, nF, k, kv_idx, kv_cnt,
                                           max_sel, status, stream);
    return D == 128 ? launch_wide<128>(qbar, kbar, BH, nQB, nKB, tau, nF, k, kv_idx, kv_cnt,
                                       max_sel, stream)
                    : launch_wide<64>(qbar, kbar, BH, nQB, nKB, tau, nF, k, kv_idx, kv_cnt,
                                      max_sel, stream);
}

}  // namespace sparstar
