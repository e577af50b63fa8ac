// Step 3, bf16 with head dim 128 — forward attention over the listed
// 128 x 128 tiles on the 5th-generation tensor cores (SparSTAR, pith.science
// review, "What carries the argument": the selected blocks run through a
// forward-only attention; the block list holds only forward fields).
//
// Work items are (b, h, pair of query blocks 2p, 2p+1), head-major.  The
// kernel is persistent: one CTA per SM walks the items w = blockIdx.x,
// + gridDim.x, ..., so the CTAs that run together hold consecutive pairs of
// one head and share its K/V in L2, and the next pair's list count, Q and
// first K/V loads overlap the current pair's last tiles and epilogue.  The
// two query blocks of a pair, A and B, have their own block lists and run
// as two interleaved pipelines: while the softmax of one works, the tensor
// core multiplies for the other.  Twelve warps:
//   warps 0-3  softmax + epilogue of block A, warps 4-7 of block B: warp w
//              serves TMEM lanes 32*(w%4)..+31, one query row per thread,
//              all 128 columns of each key tile;
//   warp 8     producer: counts each pair's valid list entries, publishes
//              them, writes the output of a block without tiles, loads Q_A
//              and Q_B, then K(0), K(1), V(0), K(2), V(1), ... (each for A
//              and B) through a 4-stage ring that runs on across pairs;
//   warp 9     TMEM allocation and the S = Q K^T MMAs (A then B per step),
//              with a record beside each S tile for the softmax;
//   warp 10    the O += P V MMAs (A then B per step);
//   warp 11    idle (it completes the producer warpgroup).
// The producer warpgroup runs on 136 registers a thread and gives the rest
// to the two softmax warpgroups (184 each: 128 x 136 + 256 x 184 = 384 x
// 168, the launch's share).
// TMEM (512 columns): S_A at 0, S_B at 128 (fp32 128 x 128), O_A at 256,
// O_B at 384.  The softmax frees S_X as soon as it has read it into
// registers, so S_X(j+1) = Q_X K(j+1)^T runs on the tensor core while the
// softmax of tile j computes its exponentials.  P (bf16) goes to shared
// memory as the K-major, 128-byte-swizzled A operand of O_X += P V; A and B
// hand their P tiles over through one buffer in turn, in the QK warp's
// issue order, each hand-off waiting for the O += P V of the one before it.
// Shared memory: Q_A, Q_B, P (32 KB each) and a 4-stage K/V ring whose
// keys run two steps ahead of its values.
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
constexpr int kStages = 4;                    // K/V ring depth
constexpr int kTileBytes = kBlock * kHD * 2;  // 32 KB: one Q, K or V tile
constexpr int kPanelBytes = kTileBytes / 2;   // 16 KB: 128 rows x 64 columns
constexpr int kSoftmaxThreads = 256;          // warps 0-7 (128 per query block)
constexpr int kThreads = kSoftmaxThreads + 128;  // + the producer warpgroup
constexpr int kProducerRegs = 136, kSoftmaxRegs = 184, kLaunchRegs = 168;
static_assert(128 * kProducerRegs + kSoftmaxThreads * kSoftmaxRegs == kThreads * kLaunchRegs,
              "the register split must balance the launch's registers");
constexpr int kProducerWarp = 8, kMmaWarp = 9, kPvWarp = 10;  // warp 11 idles
constexpr uint32_t kTmemCols = 512;
__host__ __device__ constexpr uint32_t col_s(int x) { return x ? 128u : 0u; }  // S_A, S_B
__host__ __device__ constexpr uint32_t col_o(int x) { return x ? 384u : 256u; }  // O_A, O_B
constexpr uint64_t kTimeoutNs = 2000000000ull;

// Shared-memory map (offsets from a 1024-byte aligned base).
constexpr int kOffQ = 0;                          // Q_A, then Q_B
constexpr int kOffP = 2 * kTileBytes;             // P (bf16, K-major, swizzled), A and B in turn
constexpr int kOffStage = 3 * kTileBytes;
constexpr int kOffBar = kOffStage + kStages * kTileBytes;
constexpr int kFullPerStage = 3;  // full barriers per ring stage (see ring_parity)
constexpr int kInfoReaders = 2;   // warps that read an item's tile counts: QK and PV
// Bits of a tile record (QK warp -> softmax): the item's first and last
// tile, a previous hand-off (its block in bit 2, the parity of that
// block's hand-off count in bit 3), the end of the stream; the key block
// in bits 16-31.
constexpr uint32_t kRecFirst = 1u, kRecLast = 2u, kRecPrev = 16u, kRecEnd = 32u;
struct Bars {
    uint64_t q_full;
    uint64_t q_free;  // the S products of the item that used Q are complete
    uint64_t st_full[kStages][kFullPerStage];  // [stage][use % kFullPerStage]
    uint64_t st_empty[kStages];
    uint64_t s_full[2];   // per query block: the S MMAs' commit and the tile record
    uint64_t s_free[2];
    uint64_t p_full[2][2];   // [block][half of P]: keys 64h .. 64h+63 written
    uint64_t pv_half[2][2];  // [block][half]: O += P_half V_half complete
    uint64_t info_full[2];   // [item & 1]: tile counts published
    uint64_t info_empty[2];  // [item & 1]: read by both reader warps
    uint64_t drain;
    uint32_t tmem_base;
    int32_t abort_flag;
    int32_t info[2][2];  // [item & 1][block]: valid tiles of A and B
    uint32_t rec[2][2][2];  // [block][S tile & 1]: record bits, item index
    int32_t slot_kb[kStages];  // key block of the tile in each stage
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
// another role already raised the abort flag.  The common case (phase
// already complete) costs one try_wait.  Every wait is inlined: the code
// after a register split (setmaxnreg) makes no calls.
__device__ __forceinline__ bool wait1_slow(uint32_t bar, uint32_t parity,
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
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
    if (mbar_test(bar, parity)) return;
    const uint64_t t0 = globaltimer();
    while (!mbar_test(bar, parity) && globaltimer() - t0 < kTimeoutNs) {
    }
}

// Warp-uniform bounded wait for warp-collective roles: the warp leaves
// together, so the .sync.aligned tcgen05 instructions after it stay
// converged.  The common case costs one try_wait per lane.
__device__ __forceinline__ bool wait_warp_slow(uint32_t bar, uint32_t parity,
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

// L2 eviction policies for TMA loads: Q tiles are read once
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

// Producer order within a pair: K(0), K(1), then for s = 0, 1, ...: V(s),
// K(s+2), where K(j) stands for K_A(j), K_B(j) and V(j) for V_A(j), V_B(j),
// each present while j is below that block's tile count.  Keys run two
// steps ahead of values, so the next S products never wait for a value
// tile's slot.  A pair's slots follow the previous pair's; within the pair
// the ring index of a tile is the number of the pair's tiles loaded before
// it, and steps_before(m) counts the tiles of steps before m.
__device__ __forceinline__ int steps_before(int m, int nA, int nB) {
    m = m < 0 ? 0 : m;
    return (m < nA ? m : nA) + (m < nB ? m : nB);
}
__device__ __forceinline__ int slot_k(int x, int j, int nA, int nB) {
    return steps_before(j, nA, nB) + steps_before(j - 1, nA, nB) + ((x == 1 && j < nA) ? 1 : 0);
}
__device__ __forceinline__ int slot_v(int x, int j, int nA, int nB) {
    return steps_before(j + 2, nA, nB) + steps_before(j, nA, nB) + ((x == 1 && j < nA) ? 1 : 0);
}
// Ring slot e is use u = e / kStages of stage e % kStages.  Each stage has
// kFullPerStage full barriers that take its uses in turn: slot e waits on
// barrier u % kFullPerStage for that barrier's phase u / kFullPerStage.  A
// parity test is exact while the barrier is at most one phase behind, so
// the barrier's previous use, slot e - kFullPerStage * kStages, must have
// landed when a consumer tests slot e.  It has.  A consumer tests slot e
// only after its own previous slot e' has landed.  The producer issues
// slots in order, so it had issued slot e - (kFullPerStage - 1) * kStages
// before e' whenever e - e' <= (kFullPerStage - 1) * kStages.  It issues
// a slot only after the stage's previous use (here e - kFullPerStage *
// kStages) has been consumed (its empty barrier), hence landed.
// Consecutive slots of one consumer are at most 5 apart: within a pair a
// key tile is followed by at most the other block's key tile and two value
// tiles, a value tile by two key tiles and the other block's value tile;
// across pairs, a pair's last key tile by up to four value tiles and its
// last value tile by the next pair's first four key tiles.  Two barriers
// per stage would allow a gap of 4, three allow 8.  A consumer's first slot
// (0 for keys, at most 4 for values) has no earlier use of its barrier.
__device__ __forceinline__ uint32_t ring_parity(int e) {
    return (uint32_t)((e / kStages) / kFullPerStage) & 1u;
}
// ------------------------------------------------------------------ kernel

// Work item w: (b*h, pair of query blocks 2p, 2p+1), with its two block
// lists and their (clamped) entry counts; an absent B has none.
struct ItemRef {
    int bh, qb0;
    const int32_t *listA, *listB;
    int cntA, cntB;
};
__device__ __forceinline__ ItemRef item_ref(int w, int nPair, int nQB, const int32_t *kv_idx,
                                            const int32_t *kv_cnt, int max_sel) {
    ItemRef r;
    r.bh = w / nPair;
    r.qb0 = 2 * (w % nPair);
    const bool hasB = r.qb0 + 1 < nQB;
    const int64_t rowA = (int64_t)r.bh * nQB + r.qb0;
    r.listA = kv_idx + rowA * max_sel;
    r.listB = kv_idx + (hasB ? rowA + 1 : rowA) * max_sel;
    int cA = __ldg(kv_cnt + rowA), cB = hasB ? __ldg(kv_cnt + rowA + 1) : 0;
    r.cntA = cA < 0 ? 0 : (cA > max_sel ? max_sel : cA);
    r.cntB = cB < 0 ? 0 : (cB > max_sel ? max_sel : cB);
    return r;
}

__global__ void __maxnreg__(kLaunchRegs)
attn_sm100_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, int Lq, int Lk, int nQB, int nKB,
                       int nPair, int nItems, float tau, const int32_t *__restrict__ kv_idx,
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

    const uint32_t bar_q = smem_addr(&bars->q_full);
    const uint32_t bar_qfree = smem_addr(&bars->q_free);
    auto bar_full = [&](int e) {
        return smem_addr(&bars->st_full[e % kStages][(e / kStages) % kFullPerStage]);
    };
    auto bar_empty = [&](int s) { return smem_addr(&bars->st_empty[s]); };
    auto bar_s = [&](int x) { return smem_addr(&bars->s_full[x]); };
    auto bar_sfree = [&](int x) { return smem_addr(&bars->s_free[x]); };
    auto bar_p = [&](int x, int h) { return smem_addr(&bars->p_full[x][h]); };
    auto bar_ph = [&](int x, int h) { return smem_addr(&bars->pv_half[x][h]); };
    // the whole O += P V of a block (its second half completes last)
    auto bar_pv = [&](int x) { return smem_addr(&bars->pv_half[x][1]); };
    auto bar_ifull = [&](int s) { return smem_addr(&bars->info_full[s]); };
    auto bar_iempty = [&](int s) { return smem_addr(&bars->info_empty[s]); };
    const uint32_t bar_drain = smem_addr(&bars->drain);

    // ---- set-up: barriers, TMEM
    if (warp == kProducerWarp) {
        if (lane == 0) {
            mbar_init(bar_q, 1);
            mbar_init(bar_qfree, 1);
            for (int s = 0; s < kStages; ++s) {
                for (int u = 0; u < kFullPerStage; ++u) mbar_init(smem_addr(&bars->st_full[s][u]), 1);
                mbar_init(bar_empty(s), 1);
            }
            for (int x = 0; x < 2; ++x) {
                mbar_init(bar_s(x), 2);  // the MMA commit and the record
                mbar_init(bar_sfree(x), kSoftmaxThreads / 2);
                for (int h = 0; h < 2; ++h) {
                    mbar_init(bar_p(x, h), kSoftmaxThreads / 2);
                    mbar_init(bar_ph(x, h), 1);
                }
                mbar_init(bar_ifull(x), 1);
                mbar_init(bar_iempty(x), kInfoReaders);
            }
            mbar_init(bar_drain, 2);  // one commit from each MMA warp
            bars->abort_flag = 0;
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmQ)));
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmK)));
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmV)));
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

    // The QK and PV warps read item it's tile counts (nA, nB) from the info
    // slot it & 1, published by the producer, and release the slot after
    // reading it; fail_ runs when the wait gives up.
#define READ_INFO(it_, nA_, nB_, fail_)                                                       \
    {                                                                                        \
        if (!wait_warp(bar_ifull((it_) & 1), (uint32_t)((it_) >> 1) & 1u, abort_flag, status)) \
            fail_;                                                                           \
        nA_ = bars->info[(it_) & 1][0];                                                      \
        nB_ = bars->info[(it_) & 1][1];                                                      \
        __syncwarp();                                                                        \
        if (lane == 0) mbar_arrive(bar_iempty((it_) & 1));                                  \
    }

    if (warp == kProducerWarp) {
        // ------------------------------------------------------ TMA producer
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs) : "memory");
        const uint64_t pol_q = policy_evict_first(), pol_kv = policy_evict_normal();
        int e = 0;   // ring slots issued so far
        int nq = 0;  // Q loads issued so far (items with work)
        bool ok = true;
        for (int it = 0, w = blockIdx.x; w < nItems && ok; ++it, w += gridDim.x) {
            const ItemRef I = item_ref(w, nPair, nQB, kv_idx, kv_cnt, max_sel);
            int nv2[2];
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const int32_t *lx = x ? I.listB : I.listA;
                const int cx = x ? I.cntB : I.cntA;
                // Four loads in flight per lane: the entries are independent.
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
                nv2[x] = nv;
            }
            const int nA = nv2[0], nB = nv2[1];
            const int nmax = nA > nB ? nA : nB;
            // A block without tiles gets its output here: zeros, LSE -inf.
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const int qb = I.qb0 + x;
                if ((x ? nB : nA) != 0 || qb >= nQB) continue;
                for (int i = lane; i < kBlock * (kHD / 8); i += 32) {
                    const int64_t grow = (int64_t)qb * kBlock + i / (kHD / 8);
                    if (grow < Lq)
                        reinterpret_cast<uint4 *>(out + ((int64_t)I.bh * Lq + grow) * kHD)[i % (kHD / 8)] =
                            make_uint4(0, 0, 0, 0);
                }
                if (lse) {
                    for (int r = lane; r < kBlock; r += 32) {
                        const int64_t grow = (int64_t)qb * kBlock + r;
                        if (grow < Lq) lse[(int64_t)I.bh * Lq + grow] = -INFINITY;
                    }
                }
            }
            if (lane == 0) {
                // publish the counts (the slot's previous item has been read)
                const int slot = it & 1;
                if (it >= 2 &&
                    !wait1(bar_iempty(slot), (uint32_t)((it >> 1) - 1) & 1u, abort_flag, status)) {
                    ok = false;
                } else {
                    bars->info[slot][0] = nA;
                    bars->info[slot][1] = nB;
                    mbar_arrive(bar_ifull(slot));
                }
                // Q of this item once the previous item's last S = Q K^T is done
                if (ok && nmax > 0) {
                    if (nq >= 1 && !wait1(bar_qfree, (uint32_t)(nq - 1) & 1u, abort_flag, status)) {
                        ok = false;
                    } else {
                        const int nqt = nB > 0 ? 2 : 1;  // Q_B only when B has work
                        mbar_expect_tx(bar_q, nqt * kTileBytes);
                        for (int x = 0; x < nqt; ++x) {
                            const uint32_t sQ = base + kOffQ + x * kTileBytes;
                            const int qrow = (I.qb0 + x) * kBlock;
                            tma_load_3d(sQ, &tmQ, bar_q, 0, qrow, I.bh, pol_q);
                            tma_load_3d(sQ + kPanelBytes, &tmQ, bar_q, 64, qrow, I.bh, pol_q);
                        }
                        ++nq;
                    }
                }
                int curKA = 0, curKB = 0, curVA = 0, curVB = 0;
                // Groups K(0), K(1), V(0), K(2), V(1), K(3), ...: group g > 0
                // is K((g+1)/2) when odd, V(g/2-1) when even.
                // withhold_kv (a test hook): no key or value tile is loaded, so
                // the first wait on the ring runs out and every role takes its
                // abort path.
                for (int g = 0; g <= 2 * nmax && ok && nmax > 0 && !withhold_kv; ++g) {
                    const bool is_v = g > 0 && (g & 1) == 0;
                    const int j = g == 0 ? 0 : (is_v ? g / 2 - 1 : (g + 1) / 2);
                    for (int x = 0; x < 2 && ok; ++x) {
                        if (j >= (x == 0 ? nA : nB)) continue;
                        const int stage = e % kStages;
                        if (!wait1(bar_empty(stage), ((uint32_t)(e / kStages) & 1u) ^ 1u,
                                   abort_flag, status)) {
                            ok = false;
                            break;
                        }
                        const int32_t *lx = x ? I.listB : I.listA;
                        const int cx = x ? I.cntB : I.cntA;
                        int &cr = is_v ? (x ? curVB : curVA) : (x ? curKB : curKA);
                        const int kb = next_valid(lx, cx, cr, nKB);
                        const uint32_t dst = base + kOffStage + stage * kTileBytes;
                        const CUtensorMap *map = is_v ? &tmV : &tmK;
                        bars->slot_kb[stage] = kb;  // published by the arrive below
                        mbar_expect_tx(bar_full(e), kTileBytes);
                        tma_load_3d(dst, map, bar_full(e), 0, kb * kBlock, I.bh, pol_kv);
                        tma_load_3d(dst + kPanelBytes, map, bar_full(e), 64, kb * kBlock, I.bh,
                                    pol_kv);
                        ++e;
                    }
                }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        }
        // Copies in flight must land before the CTA may exit: wait for
        // the last Q and for the latest arming of every stage (no-ops
        // normally).
        if (lane == 0) {
            if (nq > 0) drain_wait(bar_q, (uint32_t)(nq - 1) & 1u);
            const int first = e > kStages ? e - kStages : 0;
            for (int i = first; i < e; ++i) drain_wait(bar_full(i), ring_parity(i));
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // -------------------------------------------- S = Q K^T MMA issuer
        // Warp-uniform control flow; one elected lane issues.  Descriptors
        // are built once per operand and advanced by compile-time offsets.
        // Beside each S tile it writes the tile's record for the softmax:
        // first / last tile of the item, the previous P hand-off (the tile
        // it issued just before: the hand-off order is this warp's order),
        // the key block (for masking) and the item.
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs) : "memory");
        const uint64_t dQ0 = desc_k_major(base + kOffQ);
        const uint64_t dQ1 = desc_k_major(base + kOffQ + kTileBytes);
        int e0 = 0, nq = 0;        // slots and Q loads of the items before
        int tA = 0, tB = 0;        // S tiles of A and B so far
        uint32_t prev = 0;         // record bits of the previous hand-off
        bool ok = true;
        for (int it = 0, w = blockIdx.x; w < nItems && ok; ++it, w += gridDim.x) {
            int nA, nB;
            READ_INFO(it, nA, nB, break);
            const int nmax = nA > nB ? nA : nB;
            if (nmax == 0) continue;
            if (!wait_warp(bar_q, (uint32_t)nq & 1u, abort_flag, status)) break;
            for (int j = 0; j < nmax && ok; ++j) {
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    const int nxx = x == 0 ? nA : nB;
                    if (!ok || j >= nxx) continue;
                    const int e = e0 + slot_k(x, j, nA, nB);
                    const int stage = e % kStages;
                    if (!wait_warp(bar_full(e), ring_parity(e), abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    const int t = x == 0 ? tA : tB;  // this block's S tiles before
                    if (t >= 1) {
                        // S_x is free once the softmax has read the previous S_x.
                        if (!wait_warp(bar_sfree(x), (uint32_t)(t - 1) & 1u, abort_flag, status)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                    }
                    const uint32_t rec = ((uint32_t)bars->slot_kb[stage] << 16) |
                                         (j == 0 ? kRecFirst : 0u) |
                                         (j == nxx - 1 ? kRecLast : 0u) | prev;
                    if (lane == 0) {
                        bars->rec[x][t & 1][0] = rec;
                        bars->rec[x][t & 1][1] = (uint32_t)w;
                    }
                    const uint64_t dK = desc_k_major(base + kOffStage + stage * kTileBytes);
                    const uint64_t dQ = x == 0 ? dQ0 : dQ1;
                    const uint32_t dS = tmem + col_s(x);
                    if (elect_one()) {
#pragma unroll
                        for (int kk = 0; kk < kHD / 16; ++kk) {
                            const uint64_t off =
                                (uint64_t)(((kk >> 2) * kPanelBytes + (kk & 3) * 32) >> 4);
                            mma_ss(dS, dQ + off, dK + off, kIdescQK, kk > 0 ? 1u : 0u);
                        }
                        mma_commit(bar_empty(stage));
                        mma_commit(bar_s(x));
                    }
                    __syncwarp();
                    // second arrival on S_x's barrier: the record is written
                    // (the previous phase is complete: the softmax has read
                    // the previous S_x)
                    if (lane == 0) mbar_arrive(bar_s(x));
                    prev = kRecPrev | ((uint32_t)x << 2) | ((uint32_t)(t & 1) << 3);
                    if (x == 0) ++tA; else ++tB;
                }
            }
            if (!ok) break;
            // Q may be replaced once this item's S products are complete.
            if (elect_one()) mma_commit(bar_qfree);
            __syncwarp();
            ++nq;
            e0 += 2 * (nA + nB);
        }
        // End of the stream for each softmax warpgroup: once it has read its
        // last S, an end record completes the next phase of its barrier.
        if (ok) {
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const int t = x == 0 ? tA : tB;
                if (t >= 1 && !wait_warp(bar_sfree(x), (uint32_t)(t - 1) & 1u, abort_flag, status))
                    break;
                if (lane == 0) {
                    bars->rec[x][t & 1][0] = kRecEnd;
                    mbar_arrive(bar_s(x));
                    mbar_arrive(bar_s(x));
                }
                __syncwarp();
            }
        }
        // Drain: every MMA this warp issued completes before TMEM is freed.
        if (elect_one()) mma_commit(bar_drain);
        __syncwarp();
    } else if (warp == kPvWarp) {
        // ---------------------------------------------- O += P V MMA issuer
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs) : "memory");
        int e0 = 0, cA = 0, cB = 0;  // slots, hand-offs of A and B so far
        bool ok = true;
        const uint64_t dP = desc_k_major(base + kOffP);
        for (int it = 0, w = blockIdx.x; w < nItems && ok; ++it, w += gridDim.x) {
            int nA, nB;
            READ_INFO(it, nA, nB, break);
            const int nmax = nA > nB ? nA : nB;
            for (int j = 0; j < nmax && ok; ++j) {
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    if (!ok || j >= (x == 0 ? nA : nB)) continue;
                    const uint32_t par = (uint32_t)((x == 0 ? cA : cB) + j) & 1u;
                    if (!wait_warp(bar_p(x, 0), par, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();  // orders an O rescale or read (tcgen05) before the MMA
                    const int e = e0 + slot_v(x, j, nA, nB);
                    const int stage = e % kStages;
                    if (!wait_warp(bar_full(e), ring_parity(e), abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    const uint64_t dV = desc_mn_major(base + kOffStage + stage * kTileBytes);
                    const uint32_t first = j > 0 ? 1u : 0u;
                    // Each half of P (keys 64h .. 64h+63, one 16 KB panel) is
                    // multiplied as soon as it is written.
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (h == 1 && !wait_warp(bar_p(x, 1), par, abort_flag, status)) {
                            ok = false;
                            break;
                        }
                        if (elect_one()) {
#pragma unroll
                            for (int kq = 0; kq < 4; ++kq) {
                                const int kk = 4 * h + kq;
                                mma_ss(tmem + col_o(x),
                                       dP + (uint64_t)((h * kPanelBytes + kq * 32) >> 4),
                                       dV + (uint64_t)((kk * 16 * 128) >> 4), kIdescPV,
                                       kk > 0 ? 1u : first);
                            }
                            if (h == 1) mma_commit(bar_empty(stage));
                            mma_commit(bar_ph(x, h));
                        }
                        __syncwarp();
                    }
                }
            }
            e0 += 2 * (nA + nB);
            cA += nA;
            cB += nB;
        }
        if (elect_one()) mma_commit(bar_drain);
        __syncwarp();
        // Both MMA warps have committed to the drain barrier; its phase
        // completes once every MMA of the CTA has.
        if (lane == 0) drain_wait(bar_drain, 0);
        __syncwarp();
    } else if (warp < 8) {
        // ------------------------------- softmax + epilogue (128 per block)
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs) : "memory");
        // The softmax follows the stream of its block's S tiles over all
        // items; each tile's record (written by the QK warp) says where an
        // item starts and ends and which hand-off precedes it.
        const int x = warp >> 2;           // query block: 0 = A, 1 = B
        const int quarter = warp & 3;      // TMEM lane quarter
        const int row = quarter * 32 + lane;  // TMEM lane == tile row
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const uint32_t colS = col_s(x), colO = col_o(x);
        const float sc = tau * 1.4426950408889634f;  // scores in log2 units
        const bool has_tail = (Lk % kBlock) != 0;
        float m_ref = -INFINITY, l = 0.0f;
        for (uint32_t t = 0;; ++t) {
            if (!wait_warp(bar_s(x), t & 1u, abort_flag, status)) break;
            const uint32_t rec = *reinterpret_cast<volatile uint32_t *>(&bars->rec[x][t & 1][0]);
            if (rec & kRecEnd) break;
            tc_fence_after();
            float s[128];
            {
                uint32_t r[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_base + colS + 32 * c, r[c]);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 4; ++c) reg_fence(r[c]);
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int u = 0; u < 32; ++u) s[32 * c + u] = __uint_as_float(r[c][u]);
            }
            // S_x(t) is in registers: the next S = Q K^T may overwrite it.
            tc_fence_before();
            mbar_arrive(bar_sfree(x));
            if (rec & kRecFirst) {  // a new item: a fresh row state
                m_ref = -INFINITY;
                l = 0.0f;
            }
            // Only a partial last key block needs masking.
            const int valid = Lk - (int)(rec >> 16) * kBlock;  // keys of this tile that exist
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
                for (int q = 0; q < 4; ++q) mx[q] = max3f(mx[q], s[c + q], s[c + 4 + q]);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) mx[q] = fmaxf(mx[q], s[kBlock - 4 + q]);
            const float m_tile = max3f(mx[0], mx[1], fmaxf(mx[2], mx[3])) * sc;
            const float m_new = fmaxf(m_ref, m_tile);
            bool ok = true;
            if (__any_sync(0xffffffffu, m_new > m_ref + 8.0f)) {
                if (!(rec & kRecFirst)) {
                    // O_x holds this item's earlier tiles: rescale it once
                    // the previous O += P V of this block is complete.
                    if (!wait_warp(bar_pv(x), (t - 1) & 1u, abort_flag, status)) break;
                    tc_fence_after();
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
            uint32_t pk[64];  // P of keys 2u, 2u+1 in pk[u]
            // The exponent arguments come from the packed fp32x2 FMA (the
            // same rounded fma per element as the scalar form, half the
            // issues); the four running sums stay scalar adds.
            const float2 sc2 = make_float2(sc, sc), nm2 = make_float2(neg_m, neg_m);
            float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int u = 0; u < 64; u += 2) {
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
            l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
            // P (bf16) in shared memory as the K-major, 128-byte-swizzled A
            // operand of O += P V: panel h holds keys 64h..64h+63, row r at
            // r * 128 bytes, 16-byte chunk c (keys 8c..8c+7) at c ^ (r & 7).
            // The blocks take the one buffer in the QK warp's issue order; a
            // hand-off waits for the O += P V of the one before it, named by
            // the record (its block and the parity of that block's count).
            // Hand P over half by half: half h waits for the previous
            // hand-off's O += P_h V_h, is stored, and is released to the MMA
            // warp (after the proxy fence that orders the generic-proxy
            // stores before the tensor core's reads; the first release also
            // orders any O rescale or output read before the next MMA).
            uint8_t *prow = smem + kOffP + row * 128;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if (rec & kRecPrev) {
                    if (!wait_warp(bar_ph((rec >> 2) & 1, h), (rec >> 3) & 1u, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                }
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<uint4 *>(prow + h * kPanelBytes + ((c ^ (row & 7)) << 4)) =
                        make_uint4(pk[32 * h + 4 * c], pk[32 * h + 4 * c + 1],
                                   pk[32 * h + 4 * c + 2], pk[32 * h + 4 * c + 3]);
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                if (h == 0) tc_fence_before();
                mbar_arrive(bar_p(x, h));
            }
            if (!ok) break;
            if (rec & kRecLast) {
                // ---- epilogue of the item: O / l -> bf16, LSE
                if (!wait_warp(bar_pv(x), t & 1u, abort_flag, status)) break;
                const int w = (int)bars->rec[x][t & 1][1];
                const int bh = w / nPair;
                const int qb = 2 * (w % nPair) + x;
                const int64_t grow = (int64_t)qb * kBlock + row;
                const bool store = grow < Lq;
                __nv_bfloat16 *orow = out + ((int64_t)bh * Lq + grow) * kHD;
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
    }

    else {
        // idle warp of the producer warpgroup: it gives up its registers too
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs) : "memory");
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
    // The register split (setmaxnreg) balances only when the kernel is
    // launched with exactly kLaunchRegs registers a thread.
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, attn_sm100_kernel) != cudaSuccess || fa.numRegs != kLaunchRegs)
        return SPARSTAR_ECUDA;
    const int64_t nQB = ceil_div(Lq, kBlock), nKB = ceil_div(Lk, kBlock);
    const int64_t nPair = ceil_div(nQB, 2);
    const int64_t nItems = BH * nPair;
    int dev = 0, nsm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || nsm <= 0)
        return SPARSTAR_ECUDA;
    // tile records hold the key block in 16 bits; items are counted in int
    if (nKB > 65535 || nItems > INT32_MAX) return SPARSTAR_ESIZE;
    const int64_t grid = nItems < nsm ? nItems : nsm;  // one CTA per SM walks the items
    attn_sm100_kernel<<<(unsigned)grid, kThreads, kSmemBytes, stream>>>(
        mq, mk, mv, (int)Lq, (int)Lk, (int)nQB, (int)nKB, (int)nPair, (int)nItems, tau, kv_idx, kv_cnt,
        (int)max_sel, static_cast<__nv_bfloat16 *>(out), lse, status, withhold_kv ? 1 : 0);
    return cudaGetLastError() == cudaSuccess ? SPARSTAR_OK : SPARSTAR_ECUDA;
}

}  // namespace sparstar

