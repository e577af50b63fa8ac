// Internal launch interface between the C ABI layer (sparstar_api.cu) and
// the kernels.  Not installed; the public interface is include/sparstar.h.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace sparstar {

constexpr int kBlock = 128;  // tokens per block (query and key grids)

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Step 1: block means, fixed fp32 order.  x is bf16 (dtype 0) or fp32 (1).
cudaError_t launch_pool(const void *x, int dtype, int64_t BH, int64_t L, int D, float *xbar,
                        cudaStream_t stream);

// Step 1 for Q and K in one launch (same order, same results).
cudaError_t launch_pool2(const void *x0, int64_t L0, float *out0, const void *x1, int64_t L1,
                         float *out1, int dtype, int64_t BH, int D, cudaStream_t stream);

// Step 2a: S = fl(tau * sequential-fma dot) for every block pair.
cudaError_t launch_score(const float *qbar, const float *kbar, int64_t BH, int64_t nQB,
                         int64_t nKB, int D, float tau, float *S, cudaStream_t stream);

// Step 2b: per-row clip-aware top-k into kv_idx / kv_cnt.
cudaError_t launch_select(const float *S, int64_t rows, int64_t nKB, int64_t nF, int64_t k,
                          int32_t *kv_idx, int32_t *kv_cnt, int64_t max_sel,
                          cudaStream_t stream);

// Steps 2a + 2b fused: the scores of 16 query blocks kept in shared memory
// and selected from there (S never written to global memory); same bits as
// launch_score followed by launch_select.  nKB <= score_select_tiled_max_nkb()
// runs the TMA-tiled kernel, larger nKB up to score_select_max_nkb(D) the
// wide kernel; beyond that cudaErrorInvalidValue.  A timed-out TMA wait sets
// SPARSTAR_STATUS_TIMEOUT in *status (if given) and empties the CTA's lists.
cudaError_t launch_score_select(const float *qbar, const float *kbar, int64_t BH, int64_t nQB,
                                int64_t nKB, int D, float tau, int64_t nF, int64_t k,
                                int32_t *kv_idx, int32_t *kv_cnt, int64_t max_sel,
                                int32_t *status, cudaStream_t stream);
int64_t score_select_max_nkb(int D);
int64_t score_select_tiled_max_nkb();
int64_t score_select_ctas(int64_t BH, int64_t nQB);

// Step 3, bf16 D=128: TMA + tcgen05 + TMEM kernel (sm_100a), two query blocks
// per CTA as interleaved pipelines.
// withhold_kv: a test hook that loads no key or value tile, so that the
// kernel's first ring wait runs out (SPARSTAR_STATUS_TIMEOUT).
int launch_attn_sm100(const void *q, const void *k, const void *v, int64_t BH, int64_t Lq,
                      int64_t Lk, float tau, const int32_t *kv_idx, const int32_t *kv_cnt,
                      int64_t max_sel, void *out, float *lse, int32_t *status,
                      cudaStream_t stream, bool withhold_kv = false);

// Step 3, fp32 inputs (D 64/128) and bf16 D=64: fp32 SIMT kernel.
cudaError_t launch_attn_simt(const void *q, const void *k, const void *v, int dtype,
                             int64_t BH, int64_t Lq, int64_t Lk, int D, float tau,
                             const int32_t *kv_idx, const int32_t *kv_cnt, int64_t max_sel,
                             void *out, float *lse, int32_t *status, cudaStream_t stream);

// Diagnostic: retained attention mass of block lists and the token-wise
// bound, one CTA per sampled row (scratch: n_rows * Lk fp32).
cudaError_t launch_retained_mass(const void *q, const void *k, int dtype, int64_t BH, int64_t Lq,
                                 int64_t Lk, int D, float tau, int64_t nF, const int32_t *kv_idx,
                                 const int32_t *kv_cnt, int64_t max_sel, const int64_t *rows,
                                 int64_t n_rows, float *scratch, double *lse_dense,
                                 double *mass_block, double *mass_tok, double *mass_forced,
                                 cudaStream_t stream);
int64_t mass_max_nkb();

// Diagnostic: block lists carried from a source scale to a target scale by
// proportional token position (segments text, image_ref, ref, cur).
struct TransferLayout {
    int64_t len_s[4], len_t[4];  // segment lengths at the source and target scale
    int64_t off_s[4], off_t[4];  // segment starts in the key sequence
    int64_t Lk_t;                // keys at the target scale
    int32_t nKB_s, nKB_t, nQB_s, nQB_t, nF_t;
};
TransferLayout make_transfer_layout(const int64_t *len_s, const int64_t *len_t);
cudaError_t launch_transfer_lists(const int32_t *src_idx, const int32_t *src_cnt,
                                  int64_t src_max_sel, int64_t BH, const TransferLayout &ly,
                                  int32_t *dst_idx, int32_t *dst_cnt, int64_t dst_max_sel,
                                  cudaStream_t stream);
int64_t transfer_max_nkb();
int64_t transfer_max_sel(const TransferLayout &ly, int64_t src_max_sel);  // host

}  // namespace sparstar
