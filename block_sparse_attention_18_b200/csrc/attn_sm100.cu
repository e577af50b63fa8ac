// Step 3, bf16 with head dim 128 — forward attention over the listed
// 128 x 128 tiles on the 5th-generation tensor cores (SparSTAR, pith.science
// review, "What carries the argument": the selected blocks run through a
// forward-only attention; the block list holds only forward fields).
//
// One CTA per (b, h, query block) in head-major order, so the CTAs that run
// together share one head's K/V in L2.  Eleven warps, specialised:
//   warps 0-7  softmax + epilogue.  Warp w serves TMEM lanes 32*(w%4)..+31
//              (query rows) and half h = w/4 of each key tile (keys
//              64h..64h+63), so every query row is owned by two threads and
//              each SM sub-partition runs two softmax warps;
//   warp 8     TMA producer: Q once, then K/V tiles in consumption order
//              K0, K1, V0, K2, V1, ..., V(n-1) through a 6-stage ring;
//   warp 9     TMEM allocation and the S = Q K^T MMAs;
//   warp 10    the O += P V MMAs.
// Two MMA warps, so each pays one wait/issue round per tile and the two
// streams run side by side; the only cross-warp hazard (S_{j+2} written
// over the buffer P_j is read from) is closed by the QK warp waiting for
// the PV MMAs of tile j to complete.
// TMEM (512 columns): S double buffer at columns 0 and 128 (fp32 128 x 128);
// two O accumulators, O_0 at 256 and O_1 at 384, one per key half.  P of
// half h (bf16, packed two per column) is written over columns 64h..64h+31
// of the S buffer it came from (inside the columns the same thread read)
// and feeds the second product straight from TMEM (tcgen05.mma with A in
// tensor memory), so P never touches shared memory.
//
// Per tile j: S_j = Q K_j^T (8 MMAs of K = 16, A = Q and B = K both
// K-major, 128-byte swizzle), the softmax turns S_j into P_j, then
// O_h += P_j,h V_j[64h..64h+63] for h = 0, 1 (4 MMAs each, A = P from
// TMEM, B = V MN-major).  The MMA thread issues S_{j+1} before waiting for
// P_j, so the tensor core computes the next scores while the softmax runs.
//
// Each key half runs its own online softmax (running max m_h, sum l_h,
// accumulator O_h), so the two threads of a row never synchronise inside
// the loop; the halves are merged once in the epilogue:
//   M = max(m_0, m_1), O = sum_h 2^(m_h - M) O_h / sum_h 2^(m_h - M) l_h.
// Scores are kept in log2 units (scaled by tau * log2(e)); a half only
// rescales O_h and l_h when its tile max exceeds m_h by more than 8 (a
// factor 256), which keeps P below 256 and makes the O rescale (a TMEM
// round trip) rare.
//
// Every wait is bounded (about two seconds of %globaltimer): on expiry the
// CTA raises SPARSTAR_STATUS_TIMEOUT in *status, every role leaves its
// loop, the producer waits (bounded) for its copies in flight, the MMA
// thread drains its MMAs, and TMEM is freed before exit.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "sparstar.h"
#include "sparstar_internal.h"

namespace sparstar {
namespace {

constexpr int kHD = 128;                  // head dim
constexpr int kStages = 6;                // K/V ring depth
constexpr int kTileBytes = kBlock * kHD * 2;  // 32 KB: one Q, K or V tile
constexpr int kPanelBytes = kTileBytes / 2;   // 16 KB: 128 rows x 64 columns
constexpr int kSoftmaxThreads = 256;  // warps 0-7
constexpr int kThreads = kSoftmaxThreads + 96;
constexpr int kProducerWarp = 8, kMmaWarp = 9, kPvWarp = 10;
constexpr uint32_t kTmemCols = 512;
__host__ __device__ constexpr uint32_t col_s(int b) { return (b & 1) ? 128u : 0u; }  // S buffers
__host__ __device__ constexpr uint32_t col_o(int h) { return h ? 384u : 256u; }  // O_0, O_1
constexpr uint64_t kTimeoutNs = 2000000000ull;

// Shared-memory map (offsets from a 1024-byte aligned base).
constexpr int kOffQ = 0;
constexpr int kOffStage = kTileBytes;
constexpr int kOffBar = kOffStage + kStages * kTileBytes;
struct Bars {
    uint64_t q_full;
    uint64_t st_full[kStages];
    uint64_t st_empty[kStages];
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t pv_done[2];
    uint64_t drain;
    uint32_t tmem_base;
    int32_t abort_flag;
    int32_t n_valid;
};
constexpr int kSmemBytes = kOffBar + (int)sizeof(Bars) + 1024;  // + alignment slack

// Instruction descriptor, kind::f16: D fp32, A and B bf16, M = N = 128.
constexpr uint32_t make_idesc(bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
           ((uint32_t)(128 >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}
constexpr uint32_t kIdescQK = make_idesc(false);
constexpr uint32_t kIdescPV = make_idesc(true);

// ------------------------------------------------------------ PTX helpers

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
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
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

// Single-thread bounded wait.  False on timeout (flag raised) or when
// another role already raised the abort flag.  The polling loop is out of
// line; the common case (phase already complete) costs one try_wait.
__device__ __noinline__ bool wait1_slow(uint32_t bar, uint32_t parity,
                                        volatile int32_t *abort_flag, int32_t *status) {
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
        if (mbar_test(bar, parity)) return true;
        if ((it & 63u) == 0u) {
            if (*abort_flag) return false;
            if (globaltimer() - t0 > kTimeoutNs) {
                *abort_flag = 1;
                if (status) atomicOr(status, SPARSTAR_STATUS_TIMEOUT);
                return false;
            }
        }
    }
}

__device__ __forceinline__ bool wait1(uint32_t bar, uint32_t parity, volatile int32_t *abort_flag,
                                      int32_t *status) {
    return mbar_test(bar, parity) || wait1_slow(bar, parity, abort_flag, status);
}

// Bounded wait that ignores the abort flag: used on the way out, for work
// already issued (copies in flight, MMAs to drain).
__device__ __noinline__ void drain_wait(uint32_t bar, uint32_t parity) {
    if (mbar_test(bar, parity)) return;
    const uint64_t t0 = globaltimer();
    while (!mbar_test(bar, parity) && globaltimer() - t0 < kTimeoutNs) {
    }
}

// Warp-uniform bounded wait for warp-collective roles: the warp leaves
// together, so the .sync.aligned tcgen05 instructions after it stay
// converged.  Fast path inline (one try_wait per lane); polling out of line.
__device__ __noinline__ bool wait_warp_slow(uint32_t bar, uint32_t parity,
                                            volatile int32_t *abort_flag, int32_t *status) {
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 0;; ++it) {
        const bool ok = mbar_test(bar, parity);
        if (__all_sync(0xffffffffu, ok)) return true;
        if ((it & 63u) == 63u) {
            int give_up = 0;
            if ((threadIdx.x & 31) == 0) {
                if (*abort_flag) {
                    give_up = 1;
                } else if (globaltimer() - t0 > kTimeoutNs) {
                    *abort_flag = 1;
                    if (status) atomicOr(status, SPARSTAR_STATUS_TIMEOUT);
                    give_up = 1;
                }
            }
            if (__shfl_sync(0xffffffffu, give_up, 0)) return false;
        }
    }
}
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity,
                                          volatile int32_t *abort_flag, int32_t *status) {
    if (__all_sync(0xffffffffu, mbar_test(bar, parity))) return true;
    return wait_warp_slow(bar, parity, abort_flag, status);
}

// L2 eviction policies for TMA loads: Q tiles are read once per CTA
// (evict first); K/V tiles, re-read by the other query blocks of the head,
// keep the normal policy.
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t policy_evict_normal() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int c0, int c1, int c2, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptors, 128-byte swizzle, sm_100 format
// (version 1 at bit 46, layout type 2 = SWIZZLE_128B at bits 61-63).
// K-major: rows of 128 bytes, 8-row groups 1024 bytes apart (SBO).
__device__ __forceinline__ uint64_t desc_k_major(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) |
           ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// MN-major (V as the B operand, N = head dim contiguous): 64-element
// panels 16 KB apart (LBO), 8-row groups along K 1024 bytes apart (SBO).
__device__ __forceinline__ uint64_t desc_mn_major(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(kPanelBytes >> 4) << 16) |
           ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

#define SPX_R8(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), "=r"(r[i + 4]), \
                  "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])
#define SPX_W8(i) "r"(r[i]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), "r"(r[i + 4]), \
                  "r"(r[i + 5]), "r"(r[i + 6]), "r"(r[i + 7])

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31}, [%32];"
        : SPX_R8(0), SPX_R8(8), SPX_R8(16), SPX_R8(24)
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, "
        "%10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, "
        "%27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        SPX_W8(0), SPX_W8(8), SPX_W8(16), SPX_W8(24)
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// Register fence: the registers a tcgen05.ld wrote are only valid after
// tcgen05.wait::ld; routing them through an empty asm placed after the wait
// keeps the compiler from moving their uses above it.
#define SPX_RW8(i) "+r"(r[i]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3]), "+r"(r[i + 4]), \
                   "+r"(r[i + 5]), "+r"(r[i + 6]), "+r"(r[i + 7])
__device__ __forceinline__ void reg_fence(uint32_t (&r)[32]) {
    asm volatile("" : SPX_RW8(0), SPX_RW8(8), SPX_RW8(16), SPX_RW8(24));
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// True in exactly one lane of the (fully active) warp.
__device__ __forceinline__ bool elect_one() {
    uint32_t pred;
    asm volatile(
        "{\n\t.reg .b32 r;\n\t.reg .pred p;\n\t"
        "elect.sync r|p, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(pred));
    return pred != 0;
}

// Three-input maximum (one instruction on sm_100).
__device__ __forceinline__ float max3f(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // .x (low half) = lo
    return *reinterpret_cast<uint32_t *>(&h);
}

// Cursor over a query block's list that skips entries outside [0, nKB);
// every role walks the same list and sees the same valid sequence.
__device__ __forceinline__ int next_valid(const int32_t *list, int cnt, int &cur, int nKB) {
    while (cur < cnt) {
        const int j = __ldg(list + cur++);
        if (j >= 0 && j < nKB) return j;
    }
    return 0;  // unreachable when the caller counts valid entries first
}

// ------------------------------------------------------------------ kernel

__global__ void __launch_bounds__(kThreads, 1)
attn_sm100_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, int Lq, int Lk, int nQB, int nKB,
                  float tau, const int32_t *__restrict__ kv_idx,
                  const int32_t *__restrict__ kv_cnt, int max_sel,
                  __nv_bfloat16 *__restrict__ out, float *__restrict__ lse,
                  int32_t *__restrict__ status) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base - raw_addr);
    Bars *bars = reinterpret_cast<Bars *>(smem + kOffBar);
    volatile int32_t *abort_flag = &bars->abort_flag;

    const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
    const int bh = blockIdx.x / nQB;
    const int qb = blockIdx.x % nQB;
    const int32_t *list = kv_idx + (int64_t)blockIdx.x * max_sel;

    const uint32_t bar_q = smem_addr(&bars->q_full);
    auto bar_full = [&](int s) { return smem_addr(&bars->st_full[s]); };
    auto bar_empty = [&](int s) { return smem_addr(&bars->st_empty[s]); };
    auto bar_s = [&](int b) { return smem_addr(&bars->s_full[b]); };
    auto bar_p = [&](int b) { return smem_addr(&bars->p_full[b]); };
    auto bar_pv = [&](int b) { return smem_addr(&bars->pv_done[b]); };
    const uint32_t bar_drain = smem_addr(&bars->drain);

    // ---- set-up: barriers, valid-entry count, TMEM
    int cnt = __ldg(kv_cnt + blockIdx.x);
    cnt = cnt < 0 ? 0 : (cnt > max_sel ? max_sel : cnt);
    if (warp == kProducerWarp) {
        if (lane == 0) {
            mbar_init(bar_q, 1);
            for (int s = 0; s < kStages; ++s) {
                mbar_init(bar_full(s), 1);
                mbar_init(bar_empty(s), 1);
            }
            for (int b = 0; b < 2; ++b) {
                mbar_init(bar_s(b), 1);
                mbar_init(bar_p(b), kSoftmaxThreads);
                mbar_init(bar_pv(b), 1);
            }
            mbar_init(bar_drain, 2);  // one commit from each MMA warp
            bars->abort_flag = 0;
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmQ)));
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmK)));
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmV)));
        }
        int nv = 0;
        for (int c = lane; c < cnt; c += 32) {
            const int j = __ldg(list + c);
            if (j >= 0 && j < nKB)
                ++nv;
            else if (status)
                atomicOr(status, SPARSTAR_STATUS_BAD_INDEX);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) nv += __shfl_xor_sync(0xffffffffu, nv, o);
        if (lane == 0) bars->n_valid = nv;
    } else if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(&bars->tmem_base)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const int n = bars->n_valid;

    if (warp == kProducerWarp) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0 && n > 0) {
            const uint32_t sQ = base + kOffQ;
            const uint64_t pol_q = policy_evict_first(), pol_kv = policy_evict_normal();
            mbar_expect_tx(bar_q, kTileBytes);
            tma_load_3d(sQ, &tmQ, bar_q, 0, qb * kBlock, bh, pol_q);
            tma_load_3d(sQ + kPanelBytes, &tmQ, bar_q, 64, qb * kBlock, bh, pol_q);
            int curK = 0, curV = 0;
            int issued = 0;
            bool ok = true;
            for (int e = 0; e < 2 * n && ok; ++e) {
                const int stage = e % kStages;
                const uint32_t ph = (uint32_t)(e / kStages) & 1u;
                if (!wait1(bar_empty(stage), ph ^ 1u, abort_flag, status)) {
                    ok = false;
                    break;
                }
                const bool is_v = (e == 2 * n - 1) || (e > 0 && (e & 1) == 0);
                const int kb = is_v ? next_valid(list, cnt, curV, nKB)
                                    : next_valid(list, cnt, curK, nKB);
                const uint32_t dst = base + kOffStage + stage * kTileBytes;
                const CUtensorMap *map = is_v ? &tmV : &tmK;
                mbar_expect_tx(bar_full(stage), kTileBytes);
                tma_load_3d(dst, map, bar_full(stage), 0, kb * kBlock, bh, pol_kv);
                tma_load_3d(dst + kPanelBytes, map, bar_full(stage), 64, kb * kBlock, bh, pol_kv);
                ++issued;
            }
            // Copies in flight must land before the CTA may exit: wait for
            // Q and for the latest arming of every stage (no-ops normally).
            drain_wait(bar_q, 0);
            const int first = issued > kStages ? issued - kStages : 0;
            for (int e = first; e < issued; ++e)
                drain_wait(bar_full(e % kStages), (uint32_t)(e / kStages) & 1u);
        }
    } else if (warp == kMmaWarp) {
        // -------------------------------------------- S = Q K^T MMA issuer
        // The whole warp runs the control flow, so descriptors and TMEM
        // addresses stay warp-uniform; one elected lane issues.  Descriptors
        // are built once per operand and advanced by compile-time offsets.
        const uint64_t dQ = desc_k_major(base + kOffQ);
        bool ok = n > 0 && wait_warp(bar_q, 0, abort_flag, status);
        for (int j = 0; j < n && ok; ++j) {
            const int e = j == 0 ? 0 : 2 * j - 1;  // ring slot of K_j
            const int stage = e % kStages;
            if (!wait_warp(bar_full(stage), (uint32_t)(e / kStages) & 1u, abort_flag, status)) {
                ok = false;
                break;
            }
            if (j >= 2) {
                // S buffer j&1 still holds P_{j-2} until its PV MMAs complete.
                if (!wait_warp(bar_pv(j & 1), (uint32_t)((j - 2) >> 1) & 1u, abort_flag, status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
            }
            const uint64_t dK = desc_k_major(base + kOffStage + stage * kTileBytes);
            const uint32_t dS = tmem + col_s(j & 1);
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < kHD / 16; ++kk) {
                    const uint64_t off = (uint64_t)(((kk >> 2) * kPanelBytes + (kk & 3) * 32) >> 4);
                    mma_ss(dS, dQ + off, dK + off, kIdescQK, kk > 0 ? 1u : 0u);
                }
                mma_commit(bar_empty(stage));
                mma_commit(bar_s(j & 1));
            }
            __syncwarp();
        }
        // Drain: every MMA this warp issued completes before TMEM is freed.
        if (n > 0) {
            if (elect_one()) mma_commit(bar_drain);
            __syncwarp();
        }
    } else if (warp == kPvWarp) {
        // ---------------------------------------------- O += P V MMA issuer
        bool ok = n > 0;
        for (int jj = 0; jj < n && ok; ++jj) {
            if (!wait_warp(bar_p(jj & 1), (uint32_t)(jj >> 1) & 1u, abort_flag, status)) {
                ok = false;
                break;
            }
            tc_fence_after();  // orders the softmax's tcgen05.st of P before the MMA
            const int e = jj == n - 1 ? 2 * n - 1 : 2 * jj + 2;  // ring slot of V_jj
            const int stage = e % kStages;
            if (!wait_warp(bar_full(stage), (uint32_t)(e / kStages) & 1u, abort_flag, status)) {
                ok = false;
                break;
            }
            const uint64_t dV = desc_mn_major(base + kOffStage + stage * kTileBytes);
            const uint32_t aP = tmem + col_s(jj & 1);
            const uint32_t first = jj > 0 ? 1u : 0u;
            if (elect_one()) {
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ts(tmem + col_o(h), aP + 64u * h + 8u * kk,
                               dV + (uint64_t)(((4 * h + kk) * 16 * 128) >> 4), kIdescPV,
                               kk > 0 ? 1u : first);
                mma_commit(bar_empty(stage));
                mma_commit(bar_pv(jj & 1));
            }
            __syncwarp();
        }
        if (n > 0) {
            if (elect_one()) mma_commit(bar_drain);
            __syncwarp();
            // Both MMA warps have committed to the drain barrier; its phase
            // completes once every MMA of the CTA has.
            if (lane == 0) drain_wait(bar_drain, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------ softmax + epilogue (256 thr)
        const int quarter = warp & 3;      // TMEM lane quarter
        const int half = warp >> 2;        // key half of every tile
        const int row = quarter * 32 + lane;  // TMEM lane == tile row
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const uint32_t colO = col_o(half);
        const float sc = tau * 1.4426950408889634f;  // scores in log2 units
        float m_ref = -INFINITY, l = 0.0f;
        bool ok = true;
        int cur = 0;
        for (int j = 0; j < n; ++j) {
            const int kb = next_valid(list, cnt, cur, nKB);
            if (!wait_warp(bar_s(j & 1), (uint32_t)(j >> 1) & 1u, abort_flag, status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t colS = col_s(j & 1) + 64u * half;
            float s[64];
            {
                uint32_t r[2][32];
                tmem_ld32(tmem + lane_base + colS, r[0]);
                tmem_ld32(tmem + lane_base + colS + 32, r[1]);
                tmem_wait_ld();
                reg_fence(r[0]);
                reg_fence(r[1]);
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int u = 0; u < 32; ++u) s[32 * c + u] = __uint_as_float(r[c][u]);
            }
            const int valid = Lk - kb * kBlock - 64 * half;  // keys of this half that exist
            if (valid < 64) {
#pragma unroll
                for (int c = 0; c < 64; ++c)
                    if (c >= valid) s[c] = -INFINITY;
            }
            float mx[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
            for (int c = 4; c < 64; c += 8) {
#pragma unroll
                for (int t = 0; t < 4; ++t) mx[t] = max3f(mx[t], s[c + t], s[c + 4 + t]);
            }
            const float m_tile = max3f(mx[0], mx[1], fmaxf(mx[2], mx[3])) * sc;
            const float m_new = fmaxf(m_ref, m_tile);
            if (__any_sync(0xffffffffu, m_new > m_ref + 8.0f)) {
                if (j > 0) {
                    if (!wait_warp(bar_pv((j - 1) & 1), (uint32_t)((j - 1) >> 1) & 1u, abort_flag,
                                   status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const float f = m_new > -INFINITY ? ex2(m_ref - m_new) : 1.0f;  // 0 if no key seen yet
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t r[32];
                        tmem_ld32(tmem + lane_base + colO + 32 * c, r);
                        tmem_wait_ld();
                        reg_fence(r);
#pragma unroll
                        for (int u = 0; u < 32; ++u)
                            r[u] = __float_as_uint(__uint_as_float(r[u]) * f);
                        tmem_st32(tmem + lane_base + colO + 32 * c, r);
                    }
                    tmem_wait_st();
                }
                if (m_new > -INFINITY) {  // a half with no key yet keeps l = 0
                    l *= ex2(m_ref - m_new);
                    m_ref = m_new;
                }
            }
            // m_ref = -inf only while every key of this half so far was masked:
            // then every p is 0 (a finite offset keeps -inf * sc + offset = -inf).
            const float neg_m = m_ref > -INFINITY ? -m_ref : 0.0f;
            float ls[4] = {0.f, 0.f, 0.f, 0.f};
            uint32_t pk[32];
#pragma unroll
            for (int u = 0; u < 32; u += 2) {
                const int c = 2 * u;
                const float p0 = ex2(fmaf(s[c], sc, neg_m));
                const float p1 = ex2(fmaf(s[c + 1], sc, neg_m));
                const float p2 = ex2(fmaf(s[c + 2], sc, neg_m));
                const float p3 = ex2(fmaf(s[c + 3], sc, neg_m));
                ls[0] += p0;
                ls[1] += p1;
                ls[2] += p2;
                ls[3] += p3;
                pk[u] = pack_bf16(p0, p1);
                pk[u + 1] = pack_bf16(p2, p3);
            }
            tmem_st32(tmem + lane_base + colS, pk);
            l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar_p(j & 1));
        }

        // ---- epilogue: merge the two halves, O / l -> bf16, LSE
        const bool have = n > 0 && ok &&
                          wait_warp(bar_pv((n - 1) & 1), (uint32_t)((n - 1) >> 1) & 1u, abort_flag,
                                    status);
        // Exchange (m, l) with the partner thread of the other half.  Every
        // MMA has completed once the last O update has (or the CTA is
        // aborting), so the Q tile's shared memory is free for this.
        float *xm = reinterpret_cast<float *>(smem + kOffQ);  // [2][128]
        float *xl = xm + 2 * kBlock;                           // [2][128]
        xm[half * kBlock + row] = m_ref;
        xl[half * kBlock + row] = l;
        asm volatile("bar.sync 1, %0;" ::"n"(kSoftmaxThreads) : "memory");
        const float m_o = xm[(half ^ 1) * kBlock + row];
        const float l_o = xl[(half ^ 1) * kBlock + row];
        const float M = fmaxf(m_ref, m_o);
        const float a_self = m_ref > -INFINITY ? ex2(m_ref - M) : 0.0f;
        const float a_oth = m_o > -INFINITY ? ex2(m_o - M) : 0.0f;
        const float L = l * a_self + l_o * a_oth;
        const float a0 = half == 0 ? a_self : a_oth;  // weight of O_0
        const float a1 = half == 0 ? a_oth : a_self;  // weight of O_1

        const int64_t grow = (int64_t)qb * kBlock + row;
        const bool store = grow < Lq;
        __nv_bfloat16 *orow = out + ((int64_t)bh * Lq + grow) * kHD + 64 * half;
        if (n == 0) {
            if (store) {
                uint4 *o4 = reinterpret_cast<uint4 *>(orow);
#pragma unroll
                for (int c = 0; c < 8; ++c) o4[c] = make_uint4(0, 0, 0, 0);
                if (lse && half == 0) lse[(int64_t)bh * Lq + grow] = -INFINITY;
            }
        } else if (have) {
            tc_fence_after();
            const float inv = 1.0f / L;
            const float w0 = a0 * inv, w1 = a1 * inv;
#pragma unroll
            for (int c = 0; c < 2; ++c) {  // output columns 64*half + 32c .. +31
                uint32_t r0[32], r1[32];
                tmem_ld32(tmem + lane_base + col_o(0) + 64 * half + 32 * c, r0);
                tmem_ld32(tmem + lane_base + col_o(1) + 64 * half + 32 * c, r1);
                tmem_wait_ld();
                reg_fence(r0);
                reg_fence(r1);
                if (store) {
                    uint4 *o4 = reinterpret_cast<uint4 *>(orow + 32 * c);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        float f[8];
#pragma unroll
                        for (int t = 0; t < 8; ++t)
                            f[t] = __uint_as_float(r0[8 * u + t]) * w0 +
                                   __uint_as_float(r1[8 * u + t]) * w1;
                        uint4 wv;
                        wv.x = pack_bf16(f[0], f[1]);
                        wv.y = pack_bf16(f[2], f[3]);
                        wv.z = pack_bf16(f[4], f[5]);
                        wv.w = pack_bf16(f[6], f[7]);
                        __stcs(o4 + u, wv);  // O is not re-read: stream past L2
                    }
                }
            }
            if (store && lse && half == 0)
                lse[(int64_t)bh * Lq + grow] = (M + log2f(L)) * 0.6931471805599453f;
        }
    }

    // ---- teardown: TMEM is freed by the warp that allocated it
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTmemCols)
                     : "memory");
    }
}

// ------------------------------------------------------------------- host

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

// [BH, L, 128] bf16 viewed as a 3-D tensor; box = 64 columns x 128 rows x 1.
bool encode(CUtensorMap *map, const void *ptr, int64_t BH, int64_t L) {
    auto fn = get_encoder();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)kHD, (cuuint64_t)L, (cuuint64_t)BH};
    const cuuint64_t strides[2] = {(cuuint64_t)kHD * 2, (cuuint64_t)L * kHD * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)kBlock, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

int launch_attn_sm100(const void *q, const void *k, const void *v, int64_t BH, int64_t Lq,
                      int64_t Lk, float tau, const int32_t *kv_idx, const int32_t *kv_cnt,
                      int64_t max_sel, void *out, float *lse, int32_t *status,
                      cudaStream_t stream) {
    CUtensorMap mq, mk, mv;
    if (!encode(&mq, q, BH, Lq) || !encode(&mk, k, BH, Lk) || !encode(&mv, v, BH, Lk))
        return SPARSTAR_ECUDA;
    if (cudaFuncSetAttribute(attn_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemBytes) != cudaSuccess)
        return SPARSTAR_ECUDA;
    const int64_t nQB = ceil_div(Lq, kBlock), nKB = ceil_div(Lk, kBlock);
    attn_sm100_kernel<<<(unsigned)(BH * nQB), kThreads, kSmemBytes, stream>>>(
        mq, mk, mv, (int)Lq, (int)Lk, (int)nQB, (int)nKB, tau, kv_idx, kv_cnt, (int)max_sel,
        static_cast<__nv_bfloat16 *>(out), lse, status);
    return cudaGetLastError() == cudaSuccess ? SPARSTAR_OK : SPARSTAR_ECUDA;
}

}  // namespace sparstar
