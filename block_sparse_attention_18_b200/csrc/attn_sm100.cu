// Step 3, bf16 with head dim 128 — forward attention over the listed
// 128 x 128 tiles on the 5th-generation tensor cores (SparSTAR, pith.science
// review, "What carries the argument": the selected blocks run through a
// forward-only attention; the block list holds only forward fields).
//
// One CTA per (b, h, pair of query blocks 2p, 2p+1), head-major, so the CTAs
// that run together share one head's K/V in L2.  The two query blocks, A
// and B, have their own block lists and run as two interleaved pipelines:
// while the softmax of one works, the tensor core multiplies for the other.
// Eleven warps:
//   warps 0-3  softmax + epilogue of block A, warps 4-7 of block B: warp w
//              serves TMEM lanes 32*(w%4)..+31, one query row per thread,
//              all 128 columns of each key tile;
//   warp 8     TMA producer: Q_A and Q_B once, then the key and value tiles
//              through a 5-stage ring in the order the MMAs consume them:
//              K_A(0), K_B(0), then per step j: K_A(j+1), V_A(j), K_B(j+1),
//              V_B(j);
//   warp 9     TMEM allocation and the S = Q K^T MMAs, in the order A(0),
//              B(0), A(1), B(1), ...;
//   warp 10    the O += P V MMAs, in the same order.
// TMEM (512 columns): one S buffer at 0 (fp32 128 x 128) that the two blocks
// take in turn, P_A at 128 and P_B at 192 (bf16, two per column), O_A at
// 256 and O_B at 384.  The softmax of a block frees S as soon as it has read
// its scores into registers, so the other block's S = Q K^T runs on the
// tensor core while this one computes its exponentials.  P goes to tensor
// memory with tcgen05.st and is the A operand of O += P V (tcgen05.mma with
// A in tensor memory, B = V from shared memory), handed over in two 64-key
// halves so that the first half's MMAs start while the second half's
// exponentials run.  P never touches shared memory, which holds only Q_A,
// Q_B and the ring.
//
// Each row runs an online softmax in log2 units (running max m, sum l,
// accumulator O_X in TMEM); O_X and l are rescaled only when the tile max
// exceeds m by more than 8 (a factor 256), which keeps P below 256 and
// makes the O rescale (a TMEM round trip) rare.
//
// Every wait is bounded (about two seconds of %globaltimer): on expiry the
// CTA raises SPARSTAR_STATUS_TIMEOUT in *status, every role leaves its
// loop, the producer waits (bounded) for its copies in flight, the MMA
// warps drain their MMAs, and TMEM is freed before exit.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "sparstar.h"
#include "sparstar_internal.h"

namespace sparstar {
namespace {

constexpr int kHD = 128;                      // head dim
constexpr int kStages = 5;                    // K/V ring depth
constexpr int kTileBytes = kBlock * kHD * 2;  // 32 KB: one Q, K or V tile
constexpr int kPanelBytes = kTileBytes / 2;   // 16 KB: 128 rows x 64 columns
constexpr int kSoftmaxThreads = 256;          // warps 0-7 (128 per query block)
constexpr int kThreads = kSoftmaxThreads + 96;
constexpr int kProducerWarp = 8, kMmaWarp = 9, kPvWarp = 10;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;                                                    // S (A and B in turn)
__host__ __device__ constexpr uint32_t col_p(int x) { return x ? 192u : 128u; }  // P_A, P_B
__host__ __device__ constexpr uint32_t col_o(int x) { return x ? 384u : 256u; }  // O_A, O_B
constexpr uint64_t kTimeoutNs = 2000000000ull;

// Shared-memory map (offsets from a 1024-byte aligned base).
constexpr int kOffQ = 0;                          // Q_A, then Q_B
constexpr int kOffStage = 2 * kTileBytes;
constexpr int kOffBar = kOffStage + kStages * kTileBytes;
struct Bars {
    uint64_t q_full;
    uint64_t st_full[kStages][2];  // [stage][use & 1]
    uint64_t st_empty[kStages];
    uint64_t s_full[2];      // per query block: S holds this block's scores
    uint64_t s_free;         // the reader of the latest S has it in registers
    uint64_t p_full[2][2];   // [block][half of P]: keys 64h .. 64h+63 stored
    uint64_t pv_done[2];     // per block: O += P V complete (P buffer free)
    uint64_t drain;
    uint32_t tmem_base;
    int32_t abort_flag;
    int32_t n_valid[2];
};
constexpr int kSmemBytes = kOffBar + (int)sizeof(Bars) + 1024;  // + alignment slack
static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");

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
// A in tensor memory (P), B from shared memory (V).
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
// 32 consecutive 32-bit columns of this thread's TMEM lane from registers.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t *r) {
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

// 8 consecutive fp32 columns of this thread's TMEM lane (the rare O rescale
// uses these narrow chunks so that a full row of scores stays in registers).
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
                 ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
                   "r"(r[6]), "r"(r[7])
                 : "memory");
}

// Producer order (the order the MMA warps consume the tiles): K(A,0),
// K(B,0), then for j = 0, 1, ...: K(A,j+1), V(A,j), K(B,j+1), V(B,j), each
// present while its tile index is below that block's tile count.  The ring
// index of a tile is the number of tiles loaded before it; loads_before(j)
// counts the tiles ahead of step j's group.
__device__ __forceinline__ int imin(int a, int b) { return a < b ? a : b; }
__device__ __forceinline__ int loads_before(int j, int nA, int nB) {
    int c = (nA > 0) + (nB > 0);
    c += imin(j, nA - 1) > 0 ? imin(j, nA - 1) : 0;
    c += imin(j, nA);
    c += imin(j, nB - 1) > 0 ? imin(j, nB - 1) : 0;
    c += imin(j, nB);
    return c;
}
__device__ __forceinline__ int slot_k(int x, int j, int nA, int nB) {
    if (j == 0) return x == 0 ? 0 : (nA > 0 ? 1 : 0);
    const int g = j - 1, b = loads_before(g, nA, nB);
    return x == 0 ? b : b + (g + 1 < nA) + (g < nA);
}
__device__ __forceinline__ int slot_v(int x, int j, int nA, int nB) {
    const int b = loads_before(j, nA, nB);
    return x == 0 ? b + (j + 1 < nA) : b + (j + 1 < nA) + (j < nA) + (j + 1 < nB);
}
// The QK warp consumes the key tiles and the PV warp the value tiles, so a
// stage's previous occupant (slot e - kStages) can be the other warp's tile
// and still be in flight when this warp tests slot e; with one full barrier
// per stage a parity test cannot tell that state from "slot e landed".
// Each stage therefore has two full barriers, for its even and its odd
// uses: slot e waits on barrier (e / kStages) & 1 for that barrier's phase
// e / (2 kStages), whose previous phase is slot e - 2 kStages.  That slot
// has always landed before the test (the waits between the roles guarantee
// it for every pair of list lengths; tests/test_ring_protocol.py checks
// the happens-before chains), so the wait is exact.
__device__ __forceinline__ uint32_t ring_parity(int e) {
    return (uint32_t)(e / (2 * kStages)) & 1u;
}
// ------------------------------------------------------------------ kernel

__global__ void __maxnreg__(168)
attn_sm100_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, int Lq, int Lk, int nQB, int nKB,
                       int nPair, float tau, const int32_t *__restrict__ kv_idx,
                       const int32_t *__restrict__ kv_cnt, int max_sel,
                       __nv_bfloat16 *__restrict__ out, float *__restrict__ lse,
                       int32_t *__restrict__ status, int withhold_kv) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base - raw_addr);
    Bars *bars = reinterpret_cast<Bars *>(smem + kOffBar);
    volatile int32_t *abort_flag = &bars->abort_flag;

    const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
    const int bh = blockIdx.x / nPair;
    const int qb0 = 2 * (blockIdx.x % nPair);  // query block A; B = qb0 + 1
    const bool hasB = qb0 + 1 < nQB;
    // Lists and counts of A (x = 0) and B (x = 1); an absent B has none.
    const int64_t rowA = (int64_t)bh * nQB + qb0;
    const int32_t *listA = kv_idx + rowA * max_sel;
    const int32_t *listB = kv_idx + (hasB ? rowA + 1 : rowA) * max_sel;
    int cntA = __ldg(kv_cnt + rowA), cntB = hasB ? __ldg(kv_cnt + rowA + 1) : 0;
    cntA = cntA < 0 ? 0 : (cntA > max_sel ? max_sel : cntA);
    cntB = cntB < 0 ? 0 : (cntB > max_sel ? max_sel : cntB);

    const uint32_t bar_q = smem_addr(&bars->q_full);
    // Ring slot e is use e / kStages of stage e % kStages; each stage has two
    // full barriers that alternate between its uses (see ring_parity).
    auto bar_full = [&](int e) {
        return smem_addr(&bars->st_full[e % kStages][(e / kStages) & 1]);
    };
    auto bar_empty = [&](int s) { return smem_addr(&bars->st_empty[s]); };
    auto bar_s = [&](int x) { return smem_addr(&bars->s_full[x]); };
    const uint32_t bar_sfree = smem_addr(&bars->s_free);
    auto bar_p = [&](int x, int h) { return smem_addr(&bars->p_full[x][h]); };
    auto bar_pv = [&](int x) { return smem_addr(&bars->pv_done[x]); };
    const uint32_t bar_drain = smem_addr(&bars->drain);

    // ---- set-up: barriers, valid-entry counts, TMEM
    if (warp == kProducerWarp) {
        if (lane == 0) {
            mbar_init(bar_q, 1);
            for (int s = 0; s < kStages; ++s) {
                mbar_init(smem_addr(&bars->st_full[s][0]), 1);
                mbar_init(smem_addr(&bars->st_full[s][1]), 1);
                mbar_init(bar_empty(s), 1);
            }
            mbar_init(bar_sfree, kSoftmaxThreads / 2);  // one block's softmax threads
            for (int x = 0; x < 2; ++x) {
                mbar_init(bar_s(x), 1);
                for (int h = 0; h < 2; ++h) mbar_init(bar_p(x, h), kSoftmaxThreads / 2);
                mbar_init(bar_pv(x), 1);
            }
            mbar_init(bar_drain, 2);  // one commit from each MMA warp
            bars->abort_flag = 0;
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmQ)));
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmK)));
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmV)));
        }
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            const int32_t *lx = x ? listB : listA;
            const int cx = x ? cntB : cntA;
            // Four loads in flight per lane: the entries are independent, and
            // this count is on the path from the CTA's start to its first S.
            int nv = 0;
            bool bad = false;
            int c = lane;
            for (; c + 96 < cx; c += 128) {
                const int j0 = __ldg(lx + c), j1 = __ldg(lx + c + 32);
                const int j2 = __ldg(lx + c + 64), j3 = __ldg(lx + c + 96);
                const bool v0 = j0 >= 0 && j0 < nKB, v1 = j1 >= 0 && j1 < nKB;
                const bool v2 = j2 >= 0 && j2 < nKB, v3 = j3 >= 0 && j3 < nKB;
                nv += (int)v0 + (int)v1 + (int)v2 + (int)v3;
                bad |= !(v0 && v1 && v2 && v3);
            }
            for (; c < cx; c += 32) {
                const int j = __ldg(lx + c);
                const bool v = j >= 0 && j < nKB;
                nv += (int)v;
                bad |= !v;
            }
            if (bad && status) atomicOr(status, SPARSTAR_STATUS_BAD_INDEX);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) nv += __shfl_xor_sync(0xffffffffu, nv, o);
            if (lane == 0) bars->n_valid[x] = nv;
        }
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
    const int nA = bars->n_valid[0], nB = bars->n_valid[1];
    const int nmax = nA > nB ? nA : nB;

    if (warp == kProducerWarp) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0 && nmax > 0) {
            const uint64_t pol_q = policy_evict_first(), pol_kv = policy_evict_normal();
            const int nq = nB > 0 ? 2 : 1;  // Q_B only when B has work
            mbar_expect_tx(bar_q, nq * kTileBytes);
            for (int x = 0; x < nq; ++x) {
                const uint32_t sQ = base + kOffQ + x * kTileBytes;
                const int qrow = (x == 0 ? qb0 : qb0 + 1) * kBlock;
                tma_load_3d(sQ, &tmQ, bar_q, 0, qrow, bh, pol_q);
                tma_load_3d(sQ + kPanelBytes, &tmQ, bar_q, 64, qrow, bh, pol_q);
            }
            int curKA = 0, curKB = 0, curVA = 0, curVB = 0;
            int e = 0;
            // withhold_kv (a test hook): no key or value tile is loaded, so
            // the first wait on the ring runs out and every role takes its
            // abort path.
            bool ok = !withhold_kv;
            // The next key (is_v false) or value tile of block x into ring
            // slot e.
            auto load = [&](bool is_v, int x) {
                if (!ok) return;
                const int stage = e % kStages;
                if (!wait1(bar_empty(stage), ((uint32_t)(e / kStages) & 1u) ^ 1u, abort_flag,
                           status)) {
                    ok = false;
                    return;
                }
                const int32_t *lx = x ? listB : listA;
                const int cx = x ? cntB : cntA;
                int &cr = is_v ? (x ? curVB : curVA) : (x ? curKB : curKA);
                const int kb = next_valid(lx, cx, cr, nKB);
                const uint32_t dst = base + kOffStage + stage * kTileBytes;
                const CUtensorMap *map = is_v ? &tmV : &tmK;
                mbar_expect_tx(bar_full(e), kTileBytes);
                tma_load_3d(dst, map, bar_full(e), 0, kb * kBlock, bh, pol_kv);
                tma_load_3d(dst + kPanelBytes, map, bar_full(e), 64, kb * kBlock, bh, pol_kv);
                ++e;
            };
            if (nA > 0) load(false, 0);
            if (nB > 0) load(false, 1);
            for (int j = 0; j < nmax && ok; ++j) {
                if (j + 1 < nA) load(false, 0);
                if (j < nA) load(true, 0);
                if (j + 1 < nB) load(false, 1);
                if (j < nB) load(true, 1);
            }
            // Copies in flight must land before the CTA may exit: wait for
            // Q and for the latest arming of every stage (no-ops normally).
            drain_wait(bar_q, 0);
            const int first = e > kStages ? e - kStages : 0;
            for (int i = first; i < e; ++i)
                drain_wait(bar_full(i), ring_parity(i));
        }
    } else if (warp == kMmaWarp) {
        // -------------------------------------------- S = Q K^T MMA issuer
        // Warp-uniform control flow; one elected lane issues.  Descriptors
        // are built once per operand and advanced by compile-time offsets.
        // The n-th product (order A(0), B(0), A(1), ...) overwrites S once
        // the reader of product n - 1 has its scores in registers.
        const uint64_t dQ0 = desc_k_major(base + kOffQ);
        const uint64_t dQ1 = desc_k_major(base + kOffQ + kTileBytes);
        bool ok = nmax > 0 && wait_warp(bar_q, 0, abort_flag, status);
        int n = 0;
        for (int j = 0; j < nmax && ok; ++j) {
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                if (!ok || j >= (x == 0 ? nA : nB)) continue;
                const int e = slot_k(x, j, nA, nB);
                const int stage = e % kStages;
                if (!wait_warp(bar_full(e), ring_parity(e), abort_flag, status)) {
                    ok = false;
                    break;
                }
                if (n >= 1) {
                    if (!wait_warp(bar_sfree, (uint32_t)(n - 1) & 1u, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                }
                const uint64_t dK = desc_k_major(base + kOffStage + stage * kTileBytes);
                const uint64_t dQ = x == 0 ? dQ0 : dQ1;
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < kHD / 16; ++kk) {
                        const uint64_t off =
                            (uint64_t)(((kk >> 2) * kPanelBytes + (kk & 3) * 32) >> 4);
                        mma_ss(tmem + kColS, dQ + off, dK + off, kIdescQK, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(bar_empty(stage));
                    mma_commit(bar_s(x));
                }
                __syncwarp();
                ++n;
            }
        }
        // Drain: every MMA this warp issued completes before TMEM is freed.
        if (nmax > 0) {
            if (elect_one()) mma_commit(bar_drain);
            __syncwarp();
        }
    } else if (warp == kPvWarp) {
        // ---------------------------------------------- O += P V MMA issuer
        // A = P_x in tensor memory (8 columns per K = 16 step), B = V.
        bool ok = nmax > 0;
        for (int j = 0; j < nmax && ok; ++j) {
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                if (!ok || j >= (x == 0 ? nA : nB)) continue;
                if (!wait_warp(bar_p(x, 0), (uint32_t)j & 1u, abort_flag, status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();  // orders the softmax's tcgen05.st (P, O rescale) first
                const int e = slot_v(x, j, nA, nB);
                const int stage = e % kStages;
                if (!wait_warp(bar_full(e), ring_parity(e), abort_flag, status)) {
                    ok = false;
                    break;
                }
                const uint64_t dV = desc_mn_major(base + kOffStage + stage * kTileBytes);
                const uint32_t aP = tmem + col_p(x);
                const uint32_t first = j > 0 ? 1u : 0u;
                // Each half of P (keys 64h .. 64h+63, columns 32h .. 32h+31)
                // is multiplied as soon as it is stored.
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if (h == 1) {
                        if (!wait_warp(bar_p(x, 1), (uint32_t)j & 1u, abort_flag, status)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                    }
                    if (elect_one()) {
#pragma unroll
                        for (int kq = 0; kq < 4; ++kq) {
                            const int kk = 4 * h + kq;
                            mma_ts(tmem + col_o(x), aP + 8u * kk,
                                   dV + (uint64_t)((kk * 16 * 128) >> 4), kIdescPV,
                                   kk > 0 ? 1u : first);
                        }
                        if (h == 1) {
                            mma_commit(bar_empty(stage));
                            mma_commit(bar_pv(x));
                        }
                    }
                    __syncwarp();
                }
            }
        }
        if (nmax > 0) {
            if (elect_one()) mma_commit(bar_drain);
            __syncwarp();
            // Both MMA warps have committed to the drain barrier; its phase
            // completes once every MMA of the CTA has.
            if (lane == 0) drain_wait(bar_drain, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------- softmax + epilogue (128 per block)
        const int x = warp >> 2;           // query block: 0 = A, 1 = B
        const int quarter = warp & 3;      // TMEM lane quarter
        const int row = quarter * 32 + lane;  // TMEM lane == tile row
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const uint32_t colO = col_o(x), colP = col_p(x);
        const int nx = x == 0 ? nA : nB;
        const float sc = tau * 1.4426950408889634f;  // scores in log2 units
        float m_ref = -INFINITY, l = 0.0f;
        bool ok = true;
        int cur = 0;
        const bool has_tail = (Lk % kBlock) != 0;
        for (int j = 0; j < nx; ++j) {
            // Only a partial last key block needs masking, so the list is
            // read only when Lk is not a multiple of the block size (else its
            // global load would sit on the path to the tile max).
            const int kb =
                has_tail ? next_valid(x ? listB : listA, x ? cntB : cntA, cur, nKB) : 0;
            if (!wait_warp(bar_s(x), (uint32_t)j & 1u, abort_flag, status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float s[128];
            {
                uint32_t r[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_base + kColS + 32 * c, r[c]);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 4; ++c) reg_fence(r[c]);
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int u = 0; u < 32; ++u) s[32 * c + u] = __uint_as_float(r[c][u]);
            }
            // The scores are in registers: the other block's S = Q K^T may
            // overwrite S.
            tc_fence_before();
            mbar_arrive(bar_sfree);
            const int valid = Lk - kb * kBlock;  // keys of this tile that exist
            if (has_tail && valid < kBlock) {
#pragma unroll
                for (int c = 0; c < kBlock; ++c)
                    if (c >= valid) s[c] = -INFINITY;
            }
            // four chains: s[0..3], then two quads per step (s[4..123]),
            // then the last quad
            float mx[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
            for (int c = 4; c + 8 <= kBlock; c += 8) {
#pragma unroll
                for (int t = 0; t < 4; ++t) mx[t] = max3f(mx[t], s[c + t], s[c + 4 + t]);
            }
#pragma unroll
            for (int t = 0; t < 4; ++t) mx[t] = fmaxf(mx[t], s[kBlock - 4 + t]);
            const float m_tile = max3f(mx[0], mx[1], fmaxf(mx[2], mx[3])) * sc;
            const float m_new = fmaxf(m_ref, m_tile);
            bool pv_seen = false;  // the O += P V of tile j - 1 is known complete
            if (__any_sync(0xffffffffu, m_new > m_ref + 8.0f)) {
                if (j > 0) {
                    if (!wait_warp(bar_pv(x), (uint32_t)(j - 1) & 1u, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    pv_seen = true;
                    const float f = m_new > -INFINITY ? ex2(m_ref - m_new) : 1.0f;
#pragma unroll 1
                    for (int c = 0; c < kHD / 8; ++c) {
                        uint32_t r[8];
                        tmem_ld8(tmem + lane_base + colO + 8 * c, r);
                        tmem_wait_ld();
                        asm volatile("" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]),
                                     "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]));
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            r[u] = __float_as_uint(__uint_as_float(r[u]) * f);
                        tmem_st8(tmem + lane_base + colO + 8 * c, r);
                    }
                    tmem_wait_st();
                }
                if (m_new > -INFINITY) {  // a row with no key yet keeps l = 0
                    l *= ex2(m_ref - m_new);
                    m_ref = m_new;
                }
            }
            // m_ref = -inf only while every key so far was masked: then
            // every p is 0 (a finite offset keeps -inf * sc + offset = -inf).
            const float neg_m = m_ref > -INFINITY ? -m_ref : 0.0f;
            // P_x is free once the O += P V of tile j - 1 has completed.
            if (j > 0 && !pv_seen) {
                if (!wait_warp(bar_pv(x), (uint32_t)(j - 1) & 1u, abort_flag, status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
            }
            // P (bf16) into tensor memory, keys 2u and 2u+1 in column u of
            // P_x, the layout of the A operand of O += P V.  Half h (keys
            // 64h .. 64h+63) is stored and released as soon as it is
            // computed.  The exponent arguments come from the packed fp32x2
            // FMA (the same rounded fma per element as the scalar form, half
            // the issues); the four running sums stay scalar adds.
            const float2 sc2 = make_float2(sc, sc), nm2 = make_float2(neg_m, neg_m);
            float ls[4] = {0.f, 0.f, 0.f, 0.f};
            uint32_t pk[64];  // P of keys 2u, 2u+1 in pk[u]
#pragma unroll
            for (int h = 0; h < 2; ++h) {
#pragma unroll
                for (int u = 32 * h; u < 32 * h + 32; u += 2) {
                    const int c = 2 * u;
                    const float2 x01 = __ffma2_rn(make_float2(s[c], s[c + 1]), sc2, nm2);
                    const float2 x23 = __ffma2_rn(make_float2(s[c + 2], s[c + 3]), sc2, nm2);
                    const float2 p01 = make_float2(ex2(x01.x), ex2(x01.y));
                    const float2 p23 = make_float2(ex2(x23.x), ex2(x23.y));
                    ls[0] += p01.x;
                    ls[1] += p01.y;
                    ls[2] += p23.x;
                    ls[3] += p23.y;
                    pk[u] = pack_bf16(p01.x, p01.y);
                    pk[u + 1] = pack_bf16(p23.x, p23.y);
                }
                // The store completes (wait::st) before the release; the
                // first release also orders any O rescale before the next
                // O += P V.
                tmem_st32(tmem + lane_base + colP + 32 * h, pk + 32 * h);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar_p(x, h));
            }
            l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
        }

        // ---- epilogue: O / l -> bf16, LSE
        const bool have = nx > 0 && ok &&
                          wait_warp(bar_pv(x), (uint32_t)(nx - 1) & 1u, abort_flag, status);
        const int qb = qb0 + x;
        const int64_t grow = (int64_t)qb * kBlock + row;
        const bool store = qb < nQB && grow < Lq;
        __nv_bfloat16 *orow = out + ((int64_t)bh * Lq + grow) * kHD;
        if (nx == 0) {
            if (store) {
                uint4 *o4 = reinterpret_cast<uint4 *>(orow);
#pragma unroll
                for (int c = 0; c < 16; ++c) o4[c] = make_uint4(0, 0, 0, 0);
                if (lse) lse[(int64_t)bh * Lq + grow] = -INFINITY;
            }
        } else if (have) {
            tc_fence_after();
            const float inv = 1.0f / l;
#pragma unroll
            for (int c = 0; c < 4; ++c) {  // output columns 32c .. 32c+31
                uint32_t r[32];
                tmem_ld32(tmem + lane_base + colO + 32 * c, r);
                tmem_wait_ld();
                reg_fence(r);
                if (store) {
                    uint4 *o4 = reinterpret_cast<uint4 *>(orow + 32 * c);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        uint4 wv;
                        wv.x = pack_bf16(__uint_as_float(r[8 * u + 0]) * inv,
                                         __uint_as_float(r[8 * u + 1]) * inv);
                        wv.y = pack_bf16(__uint_as_float(r[8 * u + 2]) * inv,
                                         __uint_as_float(r[8 * u + 3]) * inv);
                        wv.z = pack_bf16(__uint_as_float(r[8 * u + 4]) * inv,
                                         __uint_as_float(r[8 * u + 5]) * inv);
                        wv.w = pack_bf16(__uint_as_float(r[8 * u + 6]) * inv,
                                         __uint_as_float(r[8 * u + 7]) * inv);
                        __stcs(o4 + u, wv);  // O is not re-read: stream past L2
                    }
                }
            }
            if (store && lse)
                lse[(int64_t)bh * Lq + grow] = (m_ref + log2f(l)) * 0.6931471805599453f;
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
                           cudaStream_t stream, bool withhold_kv) {
    CUtensorMap mq, mk, mv;
    if (!encode(&mq, q, BH, Lq) || !encode(&mk, k, BH, Lk) || !encode(&mv, v, BH, Lk))
        return SPARSTAR_ECUDA;
    if (cudaFuncSetAttribute(attn_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemBytes) != cudaSuccess)
        return SPARSTAR_ECUDA;
    const int64_t nQB = ceil_div(Lq, kBlock), nKB = ceil_div(Lk, kBlock);
    const int64_t nPair = ceil_div(nQB, 2);
    attn_sm100_kernel<<<(unsigned)(BH * nPair), kThreads, kSmemBytes, stream>>>(
        mq, mk, mv, (int)Lq, (int)Lk, (int)nQB, (int)nKB, (int)nPair, tau, kv_idx, kv_cnt,
        (int)max_sel, static_cast<__nv_bfloat16 *>(out), lse, status, withhold_kv ? 1 : 0);
    return cudaGetLastError() == cudaSuccess ? SPARSTAR_OK : SPARSTAR_ECUDA;
}

}  // namespace sparstar
