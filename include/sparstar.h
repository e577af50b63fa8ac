/*
 * sparstar.h — C ABI of libsparstar: SparSTAR's per-scale block-sparse
 * attention forward on B200 (sm_100a).
 *
 * The operation (SparSTAR, arXiv 2608.10519; pith.science review of the
 * paper, "What carries the argument"): at one expensive scale, per attention
 * head,
 *   1. average Q and K over contiguous 128-token blocks;
 *   2. score every (query block i, key block j) pair as
 *      S_ij = tau * qbar_i^T kbar_j, tau = D^-1/2 (the paper's Eq. 2), keep
 *      every block holding text (and, in Clip 1, the last image-pyramid
 *      reference) whatever its score, and keep the top ceil(density * C) of the remaining C
 *      reference and current-scale blocks, ranked jointly;
 *   3. run a forward-only attention over the selected 128 x 128 tiles only,
 *      described by a forward block list (per-row count + key-block index
 *      list) without any reverse index.
 *
 * Sources cited below:
 *   [R-carry]  pith.science review of SparSTAR (arXiv 2608.10519), section
 *              "What carries the argument": block-averaged q and k over
 *              contiguous 128-token blocks, the score S_ij = tau qbar_i^T
 *              kbar_j (Eq. 2), the block-average identity, text / Clip-1
 *              reference always kept, one ranking shared by reference and
 *              current blocks under the density schedule, forward-only
 *              mask fields (FastFlex).
 *   abstract   SparSTAR abstract (mlsanity.com/paper/2608.10519): the
 *              block scores are computed anew at each scale and head from
 *              that scale's own Q and K, and only the chosen blocks go
 *              through the (forward-only) sparse attention.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors are [B, H, L, D] row-major, D contiguous, with no padding.
 *    Key order inside L_k: [text | image_ref | ref | cur]; queries are the
 *    current-scale tokens.  Blocks are 128 tokens; the last block of a grid
 *    may be partial and then holds L - 128 * (nblocks - 1) real tokens.
 *  - Pointers passed to kernels are DEVICE pointers (cudaMalloc'd or
 *    equivalent), owned by the caller; the library allocates no memory,
 *    keeps no state between calls and never synchronises (the one
 *    exception, sparstar_forward_static, is described at its declaration).  `stream` is a
 *    cudaStream_t handle (NULL = the legacy default stream); every call is
 *    asynchronous on it.
 *  - dtype codes: SPARSTAR_BF16 = 0 (bfloat16 stored as 16-bit words),
 *    SPARSTAR_F32 = 1.  Head dim D is 64 or 128.
 *  - Return value: SPARSTAR_OK (0) or an error code below.  Argument errors
 *    are detected on the host before anything is launched; SPARSTAR_ECUDA
 *    reports a launch failure (cudaGetLastError after the launch).
 *  - Device pointers to q, k, v, out and the pooled / score buffers must be
 *    16-byte aligned (cudaMalloc gives 256).
 *  - The library is built for sm_100a only; calls on another device return
 *    SPARSTAR_ENODEV.
 */
#ifndef SPARSTAR_H
#define SPARSTAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SPARSTAR_BLOCK 128

enum sparstar_dtype { SPARSTAR_BF16 = 0, SPARSTAR_F32 = 1 };

enum sparstar_status {
    SPARSTAR_OK = 0,
    SPARSTAR_EINVAL = 1,  /* bad size, null pointer, misalignment, density outside (0,1] */
    SPARSTAR_EDTYPE = 2,  /* unknown dtype code */
    SPARSTAR_ECUDA = 3,   /* a CUDA runtime call or launch failed */
    SPARSTAR_ESIZE = 4,   /* max_sel < selected count, or a call too big for the static arena */
    SPARSTAR_ENODEV = 5   /* no usable sm_100 device for this call */
};

/* Bits the attention kernels OR into *status (when status is non-NULL). */
#define SPARSTAR_STATUS_BAD_INDEX 0x1 /* a kv_idx entry outside [0, nKB) was skipped */
#define SPARSTAR_STATUS_TIMEOUT 0x2   /* a pipeline wait gave up; output is invalid */

/*
 * sparstar_block_pool — step 1, block mean pooling.
 * Source: [R-carry] — queries and keys are averaged over contiguous 128-token
 * blocks, taken in the order the attention kernel walks them.
 *   x     [B,H,L,D] of `dtype` (device)
 *   xbar  [B,H,ceil(L/128),D] fp32 (device, written)
 * xbar[b,h,blk,d] is the mean of the block's real tokens, summed in this
 * fixed fp32 order: stripe r = 0..7 adds the tokens t = r, r+8, r+16, ...
 * of the block in ascending t, starting from +0; the total is
 * ((s0+s1)+(s2+s3))+((s4+s5)+(s6+s7)); the mean is one IEEE
 * round-to-nearest division by the real token count n.
 * Call once for Q (L = Lq) and once for K (L = Lk).
 */
int sparstar_block_pool(const void *x, int dtype, int64_t B, int64_t H, int64_t L,
                        int64_t D, float *xbar, void *stream);

/*
 * sparstar_block_score — step 2a, the aggregated block score (Eq. 2).
 * Source: [R-carry] — S_ij = tau qbar_i^T kbar_j with tau = D^-1/2; the dot
 * product of two block means is the mean of the pairwise query-key dot
 * products between the two blocks.
 *   qbar [B,H,nQB,D] fp32, kbar [B,H,nKB,D] fp32 (device)
 *   tau  fp32 scale, normally (float)(1/sqrt((double)D))
 *   S    [B,H,nQB,nKB] fp32 (device, written)
 * S = (acc) * tau, one IEEE multiply, where acc starts at +0 and takes
 * acc = fma(qbar[d], kbar[d], acc) for d = 0..D-1 in ascending order.
 * Every pair is scored, forced blocks included.  Results are bit-identical
 * to any implementation of that order.
 */
int sparstar_block_score(const float *qbar, const float *kbar, int64_t B, int64_t H,
                         int64_t nQB, int64_t nKB, int64_t D, float tau, float *S,
                         void *stream);

/*
 * sparstar_forced_blocks — host only.  Number of leading key blocks that
 * hold at least one text or Clip-1 image-reference token:
 * ceil((text_len + image_ref_len) / 128).  Source: [R-carry] — the text
 * tokens, and in Clip 1 the last image-pyramid reference, always take part
 * in the attention.  Returns -1 for negative lengths.
 */
int64_t sparstar_forced_blocks(int64_t text_len, int64_t image_ref_len);

/*
 * sparstar_select_count — host only.  Selected blocks per query block:
 * n_forced_blocks + k with k = ceil(density * C), C = nKB - n_forced_blocks,
 * computed in fp64 and clamped to [0, C].  Passage: the per-scale density
 * schedule ([R-carry]).  Returns -1 when nKB <= 0, n_forced_blocks is
 * outside [0, nKB] or density is outside (0, 1].
 */
int64_t sparstar_select_count(int64_t nKB, int64_t n_forced_blocks, double density);

/*
 * sparstar_select — step 2b, clip-aware block Top-K into a forward-only
 * block list.  Source: [R-carry] — text and the Clip-1 reference are kept;
 * the remaining blocks of the preceding-clip reference and of the current
 * scale compete in one ranking under the density budget; the mask keeps
 * only its forward fields and builds no reverse index.
 *   S       [B,H,nQB,nKB] fp32 (device); must be finite
 *   kv_idx  [B,H,nQB,max_sel] int32 (device, written): for every row,
 *           0..nF-1, then the chosen candidates in ascending order, then -1
 *           in the unused slots
 *   kv_cnt  [B,H,nQB] int32 (device, written): sel = sparstar_select_count
 * Candidates j in [nF, nKB) are ranked by S descending, equal scores
 * (with -0 == +0) going to the lower j.  Returns SPARSTAR_ESIZE when
 * max_sel < sel.
 */
int sparstar_select(const float *S, int64_t B, int64_t H, int64_t nQB, int64_t nKB,
                    int64_t n_forced_blocks, double density, int32_t *kv_idx,
                    int32_t *kv_cnt, int64_t max_sel, void *stream);

/*
 * sparstar_attn_fwd — step 3, forward attention over the listed tiles.
 * Source: abstract and [R-carry] — only the selected blocks are computed,
 * by a forward-only sparse attention.
 *   q [B,H,Lq,D], k and v [B,H,Lk,D] of `dtype` (device)
 *   tau      softmax scale (normally D^-1/2)
 *   kv_idx   [B,H,ceil(Lq/128),max_sel] int32, kv_cnt [B,H,ceil(Lq/128)]
 *            int32 (device): the block list of each query block.  Entries
 *            past kv_cnt are ignored; an entry outside [0, ceil(Lk/128)) is
 *            skipped and flagged in *status.
 *   out      [B,H,Lq,D] of `dtype` (device, written)
 *   lse      [B,H,Lq] fp32 natural-log sum-exp of the scaled scores over
 *            the visible keys (device, written), or NULL
 *   status   one int32 (device) that kernels OR SPARSTAR_STATUS_* bits into,
 *            or NULL; the caller zeroes it
 * For query row r of block i: out_r = sum_t softmax_t(tau q_r.k_t) v_t over
 * the tokens t < Lk of the listed key blocks.  No causal mask.  A row whose
 * list is empty gets out = 0 and lse = -inf.  bf16 with D = 128 runs on the
 * tcgen05 tensor-core kernel (fp32 accumulation and softmax, P rounded to
 * bf16 for the second product); fp32 inputs and D = 64 run on an fp32 SIMT
 * kernel.
 */
int sparstar_attn_fwd(const void *q, const void *k, const void *v, int dtype, int64_t B,
                      int64_t H, int64_t Lq, int64_t Lk, int64_t D, float tau,
                      const int32_t *kv_idx, const int32_t *kv_cnt, int64_t max_sel,
                      void *out, float *lse, int32_t *status, void *stream);

/*
 * sparstar_forward — the four steps in order on one stream, for one scale.
 * Segments: text_len, image_ref_len (Clip 1 only, else 0), ref_len, cur_len;
 * Lk = their sum, Lq = cur_len.  Workspace (device, caller-owned):
 *   qbar [B,H,nQB,D] fp32, kbar [B,H,nKB,D] fp32, S [B,H,nQB,nKB] fp32,
 *   kv_idx [B,H,nQB,max_sel] int32, kv_cnt [B,H,nQB] int32.
 * tau = (float)(1/sqrt(D)).  Returns the first error of the chain.
 */
int sparstar_forward(const void *q, const void *k, const void *v, int dtype, int64_t B,
                     int64_t H, int64_t D, int64_t text_len, int64_t image_ref_len,
                     int64_t ref_len, int64_t cur_len, double density, float *qbar,
                     float *kbar, float *S, int32_t *kv_idx, int32_t *kv_cnt,
                     int64_t max_sel, void *out, float *lse, int32_t *status, void *stream);

/*
 * sparstar_forward_static — sparstar_forward for callers that cannot
 * allocate device memory.  The paper has no counterpart: it is an
 * allocation-free way into the same four steps.
 *
 * Some callers have no way to allocate device memory of their own: a host
 * program that hands the library only its input and output buffers, or a
 * plugin whose host forbids device allocations outside its own pool.  This
 * entry point takes the same arguments as sparstar_forward minus the
 * workspace and keeps the intermediates (block means, scores, block lists)
 * in a fixed arena of SPARSTAR_STATIC_ARENA_BYTES that the library itself
 * reserves on every GPU that loads it, for the life of the process.  It
 * calls no cudaMalloc, cudaFree or allocating library routine.
 *   - Size limit: the intermediates of one call, 4 * B * H * (nQB * D +
 *     nKB * D + nQB * nKB + nQB * sel + nQB) bytes plus alignment, must fit
 *     in the arena (the 72,000-token scale with 16 heads needs about
 *     59 MB); larger calls return SPARSTAR_ESIZE and launch nothing.
 *   - The first call on each device looks the arena's address up
 *     (cudaGetSymbolAddress) with that device current and caches it; make
 *     that first call before any stream capture.  The cached address is
 *     tied to the CUDA context it was taken in: a call in another context
 *     (a non-primary context, or the new primary context after
 *     cudaDeviceReset) looks it up again, so that call too should come
 *     before any capture.
 *   - All calls share the arena.  Calls whose GPU work overlaps (other
 *     streams, other host threads) race on it; serialise them.
 * The caller still owns q, k, v, out, lse and status.  Errors are those of
 * sparstar_forward, plus SPARSTAR_ESIZE for a call that does not fit.
 */
#define SPARSTAR_STATIC_ARENA_BYTES ((size_t)64 << 20)

int sparstar_forward_static(const void *q, const void *k, const void *v, int dtype, int64_t B,
                            int64_t H, int64_t D, int64_t text_len, int64_t image_ref_len,
                            int64_t ref_len, int64_t cur_len, double density, void *out,
                            float *lse, int32_t *status, void *stream);

/*
 * Fused selection front-end.  Source: [R-carry] — the block selection
 * (pooling, scoring, Top-K) is a small cost beside the sparse attention it
 * prepares; these calls make it three launches instead of five and keep S
 * out of device memory.  Results are bit-identical to the separate calls:
 * the same fixed fp32 orders, the same ranking and tie rule.
 *
 * sparstar_block_pool_qk — sparstar_block_pool of q (length Lq) into qbar
 * and of k (length Lk) into kbar, in one launch.  Same arguments, layouts
 * and errors as two sparstar_block_pool calls.
 */
int sparstar_block_pool_qk(const void *q, const void *k, int dtype, int64_t B, int64_t H,
                           int64_t Lq, int64_t Lk, int64_t D, float *qbar, float *kbar,
                           void *stream);

/*
 * sparstar_score_select — sparstar_block_score followed by sparstar_select
 * in one launch, without the S buffer: each CTA scores 16 query blocks
 * against every key block into shared memory and selects from there.
 *   qbar, kbar, tau as for sparstar_block_score;
 *   n_forced_blocks, density, kv_idx, kv_cnt, max_sel as for sparstar_select;
 *   status   one int32 (device) that the kernel ORs SPARSTAR_STATUS_TIMEOUT
 *            into if a copy wait gives up (the lists of that CTA's rows are
 *            then empty: kv_cnt = 0), or NULL; the caller zeroes it.
 * The score rows of 16 query blocks must fit in one CTA's shared memory:
 * nKB <= sparstar_score_select_max_nkb(D) (2432 for D = 128, 2944 for
 * D = 64, i.e. about 311k / 377k keys), else SPARSTAR_ESIZE and nothing is
 * launched; the separate calls have no such limit.  Up to nKB = 1536 the
 * key means arrive by TMA as d-chunks of every key column (8 rows x up to 6
 * columns per thread); up to 1664 as 256-key tiles (4 x 4 per thread);
 * larger nKB use a register-staged tiling that needs less shared memory per
 * key block.  Other errors as for the separate calls.
 */
int sparstar_score_select(const float *qbar, const float *kbar, int64_t B, int64_t H,
                          int64_t nQB, int64_t nKB, int64_t D, float tau,
                          int64_t n_forced_blocks, double density, int32_t *kv_idx,
                          int32_t *kv_cnt, int64_t max_sel, int32_t *status, void *stream);

/* Largest nKB sparstar_score_select accepts for head dim D; -1 for a bad D. */
int64_t sparstar_score_select_max_nkb(int64_t D);

/*
 * sparstar_forward_fused — sparstar_forward over the fused front-end:
 * sparstar_block_pool_qk, sparstar_score_select, sparstar_attn_fwd, three
 * launches on one stream.  Same arguments as sparstar_forward without S;
 * same results.  The whole chain is checked before anything is launched
 * (SPARSTAR_ESIZE for max_sel < sel or nKB above the fused limit).  It
 * calls no synchronising CUDA routine, so it can be recorded into a CUDA
 * graph by stream capture once a first call on that device has run outside
 * the capture.
 */
int sparstar_forward_fused(const void *q, const void *k, const void *v, int dtype, int64_t B,
                           int64_t H, int64_t D, int64_t text_len, int64_t image_ref_len,
                           int64_t ref_len, int64_t cur_len, double density, float *qbar,
                           float *kbar, int32_t *kv_idx, int32_t *kv_cnt, int64_t max_sel,
                           void *out, float *lse, int32_t *status, void *stream);

/*
 * sparstar_retained_mass — diagnostic: how much dense attention mass the
 * block lists keep, and the most that any token-level choice with the same
 * budget could keep.  Source: pith.science review of SparSTAR, "Extended
 * reading notes / Core claim" (block-wise Top-K recomputed at every scale
 * stays close to the token-wise upper bound in retained attention mass) and
 * "What would settle it" (the exact token-wise Top-K at the same densities
 * as the comparison).  Not part of the attention forward; it reads all of K
 * for every sampled row.
 *   q, k       [B,H,Lq,D], [B,H,Lk,D] of `dtype` (device)
 *   tau        softmax scale (normally D^-1/2)
 *   n_forced_blocks, kv_idx, kv_cnt, max_sel: the block lists, as written
 *              by sparstar_select (device)
 *   rows       [n_rows] int64 (device): flat query rows b*H*Lq + h*Lq + r;
 *              a row outside [0, B*H*Lq) gets NaN results
 *   scratch    [n_rows, Lk] fp32 (device, overwritten): the rows' scores
 *   lse_dense, mass_block, mass_tok, mass_forced  [n_rows] fp64 (device,
 *              written), for each row with dense weights
 *              p_t = softmax_t(tau q.k_t) over every key t < Lk:
 *                lse_dense   = log sum_t exp(tau q.k_t);
 *                mass_block  = sum of p_t over the tokens of the listed blocks;
 *                mass_forced = sum of p_t over the tokens of blocks 0..nF-1;
 *                mass_tok    = mass_forced + the M largest p_t among the
 *                              candidate tokens t >= 128 nF, where M = the
 *                              real tokens of the listed blocks j >= nF.
 * Scores are fp32 (q.k accumulated with fp32 FMAs), every sum fp64.
 * mass_block also equals exp(lse_sparse - lse_dense) with the lse of
 * sparstar_attn_fwd.  Errors: SPARSTAR_EINVAL for bad sizes or pointers,
 * n_forced_blocks outside [0, nKB] or nKB > 2^20.
 */
int sparstar_retained_mass(const void *q, const void *k, int dtype, int64_t B, int64_t H,
                           int64_t Lq, int64_t Lk, int64_t D, float tau, int64_t n_forced_blocks,
                           const int32_t *kv_idx, const int32_t *kv_cnt, int64_t max_sel,
                           const int64_t *rows, int64_t n_rows, float *scratch,
                           double *lse_dense, double *mass_block, double *mass_tok,
                           double *mass_forced, void *stream);

/*
 * sparstar_transfer_lists — diagnostic: the block lists of a source scale
 * carried by token position to a target scale, i.e. the mask reuse across
 * scales that the method argues against.  Source: pith.science review of
 * SparSTAR, "Extended reading notes / Core claim" (a selection carried from
 * one scale to another keeps less attention mass than a fresh one, so the
 * method selects anew at every scale) and Figure 1 (a carried-over mask can leave
 * out blocks that matter at the new scale).  The pages give no map between two scales' token
 * positions; this call resamples the block mask by nearest neighbour
 * along the token order, the plainest reading:
 *   - keys at both scales are the segments [text | image_ref | ref | cur];
 *     src_len[g] / dst_len[g] are their lengths at the source / target
 *     scale (host arrays of 4 int64; queries are the cur segment);
 *   - the target token at offset p of segment g has as image the source
 *     token at offset floor(p * src_len[g] / dst_len[g]) of segment g (none
 *     when src_len[g] = 0);
 *   - the centre of a block of n real tokens starting at token a is token
 *     a + (n - 1) / 2;
 *   - target query block i uses the list of the source query block holding
 *     the image of i's centre query token;
 *   - target key block j is kept when j < ceil((dst_len[0] + dst_len[1]) /
 *     128) (forced at the target), or when the image of j's centre token
 *     lies in a block of that list.
 *   src_idx, src_cnt, src_max_sel: the source lists as written by
 *            sparstar_select ([B,H,nQB_s,src_max_sel], [B,H,nQB_s] int32,
 *            device); entries outside [0, nKB_s) are ignored and a count
 *            above src_max_sel is read as src_max_sel
 *   dst_idx  [B,H,nQB_t,dst_max_sel] int32 (device, written): kept blocks
 *            ascending, unused slots -1
 *   dst_cnt  [B,H,nQB_t] int32 (device, written)
 * The transferred list has no budget of its own (it keeps about the source
 * scale's density); dst_max_sel must be at least
 * sparstar_transfer_max_sel(src_len, dst_len, src_max_sel), the longest
 * row any source lists can produce.
 * Errors: SPARSTAR_EINVAL for null pointers, B or H < 1, a negative length,
 * src_len[3] = 0 < dst_len[3], src_max_sel < 1 or more than 2^31 - 1
 * source or target keys; SPARSTAR_ESIZE for dst_max_sel below that bound or
 * a source or target with more than 32768 key blocks.  Nothing is launched on an
 * error, or when dst_len[3] = 0 (no target rows).  The host computes the
 * bound on every call (a pass over the target's key blocks).
 */
/*
 * Longest transferred row that source lists of stride src_max_sel can give
 * (host-only; src_len, dst_len as for sparstar_transfer_lists): the
 * target's forced blocks plus the src_max_sel largest counts of non-forced
 * target blocks whose centre token has its image in one source block.
 * Returns -1 for bad arguments (as sparstar_transfer_lists would reject).
 */
int64_t sparstar_transfer_max_sel(const int64_t *src_len, const int64_t *dst_len,
                                  int64_t src_max_sel);

int sparstar_transfer_lists(const int32_t *src_idx, const int32_t *src_cnt, int64_t src_max_sel,
                            int64_t B, int64_t H, const int64_t *src_len, const int64_t *dst_len,
                            int32_t *dst_idx, int32_t *dst_cnt, int64_t dst_max_sel,
                            void *stream);

/*
 * sparstar_test_attn_timeout — TEST HOOK for failure detection, not part of
 * the attention forward.  Runs the bf16 D = 128 attention kernel with every
 * key and value copy withheld: the kernel's first wait on its K/V ring can
 * never complete, gives up after about two seconds, ORs
 * SPARSTAR_STATUS_TIMEOUT into *status, and every role leaves through its
 * abort path (copies in flight drained, TMEM freed), so the CUDA context
 * stays usable.  `out` is left undefined.  Arguments as for sparstar_attn_fwd
 * (bf16, D = 128; status required).  Returns a launch status; the timeout is
 * reported in *status once the stream has run.
 */
int sparstar_test_attn_timeout(const void *q, const void *k, const void *v, int64_t B, int64_t H,
                               int64_t Lq, int64_t Lk, const int32_t *kv_idx,
                               const int32_t *kv_cnt, int64_t max_sel, void *out,
                               int32_t *status, void *stream);

/* Message for a status code (static storage). */
const char *sparstar_strerror(int code);

/* ABI version: major * 10000 + minor * 100 + patch. */
int sparstar_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SPARSTAR_H */
