// C ABI of libsparstar (declared in include/sparstar.h): argument checks,
// device check and dispatch to the kernels.  Every argument error is found
// here, on the host, before anything is launched.  The library allocates
// no memory and keeps no state between calls.
#include <cmath>
#include <cstdint>

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>  // header-only: ranges cost nothing without a tool attached

#include "sparstar.h"
#include "sparstar_internal.h"

#define SPARSTAR_API extern "C" __attribute__((visibility("default")))

using sparstar::ceil_div;
using sparstar::kBlock;

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool dtype_ok(int dtype) { return dtype == SPARSTAR_BF16 || dtype == SPARSTAR_F32; }

bool head_dim_ok(int64_t D) { return D == 64 || D == 128; }

// The kernels are built for sm_100a only.
int device_check() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return SPARSTAR_ENODEV;
    }
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cudaGetLastError();
        return SPARSTAR_ENODEV;
    }
    return (major == 10 && minor == 0) ? SPARSTAR_OK : SPARSTAR_ENODEV;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? SPARSTAR_OK : SPARSTAR_ECUDA; }

// An NVTX range over one ABI call (host side: argument checks and launches),
// named after the call, for profilers that group work by NVTX range.
struct TraceRange {
    explicit TraceRange(const char *name) { nvtxRangePushA(name); }
    ~TraceRange() { nvtxRangePop(); }
    TraceRange(const TraceRange &) = delete;
    TraceRange &operator=(const TraceRange &) = delete;
};

// Largest sizes the kernels index with 32-bit grid or coordinate values.
constexpr int64_t kMaxGrid = 0x7fffffffLL;
constexpr int64_t kMaxTokens = 0x7fffffffLL - kBlock;

}  // namespace

SPARSTAR_API int sparstar_version(void) { return 10000; }

SPARSTAR_API const char *sparstar_strerror(int code) {
    switch (code) {
    case SPARSTAR_OK: return "ok";
    case SPARSTAR_EINVAL: return "invalid argument (size, null pointer, alignment or density)";
    case SPARSTAR_EDTYPE: return "unsupported dtype code";
    case SPARSTAR_ECUDA: return "CUDA runtime error";
    case SPARSTAR_ESIZE:
        return "size limit: max_sel below the selected count, the intermediates exceed the "
               "static arena (SPARSTAR_STATIC_ARENA_BYTES), or nKB above "
               "sparstar_score_select_max_nkb(D)";
    case SPARSTAR_ENODEV: return "no sm_100 device available for this call";
    default: return "unknown status";
    }
}

SPARSTAR_API int64_t sparstar_forced_blocks(int64_t text_len, int64_t image_ref_len) {
    if (text_len < 0 || image_ref_len < 0) return -1;
    return ceil_div(text_len + image_ref_len, kBlock);
}

SPARSTAR_API int64_t sparstar_select_count(int64_t nKB, int64_t n_forced_blocks, double density) {
    if (nKB <= 0 || n_forced_blocks < 0 || n_forced_blocks > nKB) return -1;
    if (!(density > 0.0) || !(density <= 1.0)) return -1;
    const int64_t C = nKB - n_forced_blocks;
    int64_t k = (int64_t)std::ceil(density * (double)C);
    if (k < 0) k = 0;
    if (k > C) k = C;
    return n_forced_blocks + k;
}

SPARSTAR_API int sparstar_block_pool(const void *x, int dtype, int64_t B, int64_t H, int64_t L,
                                     int64_t D, float *xbar, void *stream) {
    TraceRange trace("sparstar_block_pool");
    if (!dtype_ok(dtype)) return SPARSTAR_EDTYPE;
    if (!x || !xbar || B <= 0 || H <= 0 || L <= 0 || !head_dim_ok(D)) return SPARSTAR_EINVAL;
    if (!aligned16(x) || !aligned16(xbar)) return SPARSTAR_EINVAL;
    if (L > kMaxTokens || B * H * ceil_div(L, kBlock) > kMaxGrid) return SPARSTAR_EINVAL;
    if (int rc = device_check()) return rc;
    return cuda_status(sparstar::launch_pool(x, dtype, B * H, L, (int)D, xbar,
                                             static_cast<cudaStream_t>(stream)));
}

SPARSTAR_API int sparstar_block_score(const float *qbar, const float *kbar, int64_t B, int64_t H,
                                      int64_t nQB, int64_t nKB, int64_t D, float tau, float *S,
                                      void *stream) {
    TraceRange trace("sparstar_block_score");
    if (!qbar || !kbar || !S || B <= 0 || H <= 0 || nQB <= 0 || nKB <= 0 || !head_dim_ok(D))
        return SPARSTAR_EINVAL;
    if (!std::isfinite(tau)) return SPARSTAR_EINVAL;
    if (!aligned16(qbar) || !aligned16(kbar)) return SPARSTAR_EINVAL;
    // grid: x = key-block tiles, y = query-block tiles, z = B*H
    if (B * H > 65535 || ceil_div(nQB, 64) > 65535 || ceil_div(nKB, 64) > kMaxGrid)
        return SPARSTAR_EINVAL;
    if (int rc = device_check()) return rc;
    return cuda_status(sparstar::launch_score(qbar, kbar, B * H, nQB, nKB, (int)D, tau, S,
                                              static_cast<cudaStream_t>(stream)));
}

SPARSTAR_API int sparstar_select(const float *S, int64_t B, int64_t H, int64_t nQB, int64_t nKB,
                                 int64_t n_forced_blocks, double density, int32_t *kv_idx,
                                 int32_t *kv_cnt, int64_t max_sel, void *stream) {
    TraceRange trace("sparstar_select");
    if (!S || !kv_idx || !kv_cnt || B <= 0 || H <= 0 || nQB <= 0 || nKB <= 0)
        return SPARSTAR_EINVAL;
    if (nKB > 0x7fffffffLL) return SPARSTAR_EINVAL;
    const int64_t sel = sparstar_select_count(nKB, n_forced_blocks, density);
    if (sel < 0) return SPARSTAR_EINVAL;
    if (max_sel < sel) return SPARSTAR_ESIZE;
    const int64_t rows = B * H * nQB;
    if (ceil_div(rows, 4) > kMaxGrid) return SPARSTAR_EINVAL;
    if (int rc = device_check()) return rc;
    return cuda_status(sparstar::launch_select(S, rows, nKB, n_forced_blocks,
                                               sel - n_forced_blocks, kv_idx, kv_cnt, max_sel,
                                               static_cast<cudaStream_t>(stream)));
}

SPARSTAR_API int sparstar_attn_fwd(const void *q, const void *k, const void *v, int dtype,
                                   int64_t B, int64_t H, int64_t Lq, int64_t Lk, int64_t D,
                                   float tau, const int32_t *kv_idx, const int32_t *kv_cnt,
                                   int64_t max_sel, void *out, float *lse, int32_t *status,
                                   void *stream) {
    TraceRange trace("sparstar_attn_fwd");
    if (!dtype_ok(dtype)) return SPARSTAR_EDTYPE;
    if (!q || !k || !v || !out || !kv_cnt || B <= 0 || H <= 0 || Lq <= 0 || Lk <= 0 ||
        !head_dim_ok(D) || max_sel < 0)
        return SPARSTAR_EINVAL;
    if (max_sel > 0 && !kv_idx) return SPARSTAR_EINVAL;
    if (!std::isfinite(tau)) return SPARSTAR_EINVAL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
        return SPARSTAR_EINVAL;
    if (Lq > kMaxTokens || Lk > kMaxTokens || max_sel > 0x7fffffffLL) return SPARSTAR_EINVAL;
    const int64_t nQB = ceil_div(Lq, kBlock);
    if (B * H * nQB > kMaxGrid) return SPARSTAR_EINVAL;
    if (int rc = device_check()) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dtype == SPARSTAR_BF16 && D == 128) {
        if (B * H > 0x7fffffffLL) return SPARSTAR_EINVAL;  // TMA coordinate
        return sparstar::launch_attn_sm100(q, k, v, B * H, Lq, Lk, tau, kv_idx, kv_cnt, max_sel,
                                           out, lse, status, s);
    }
    return cuda_status(sparstar::launch_attn_simt(q, k, v, dtype, B * H, Lq, Lk, (int)D, tau,
                                                  kv_idx, kv_cnt, max_sel, out, lse, status, s));
}

SPARSTAR_API int sparstar_block_pool_qk(const void *q, const void *k, int dtype, int64_t B,
                                        int64_t H, int64_t Lq, int64_t Lk, int64_t D,
                                        float *qbar, float *kbar, void *stream) {
    TraceRange trace("sparstar_block_pool_qk");
    if (!dtype_ok(dtype)) return SPARSTAR_EDTYPE;
    if (!q || !k || !qbar || !kbar || B <= 0 || H <= 0 || Lq <= 0 || Lk <= 0 ||
        !head_dim_ok(D))
        return SPARSTAR_EINVAL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(qbar) || !aligned16(kbar))
        return SPARSTAR_EINVAL;
    if (Lq > kMaxTokens || Lk > kMaxTokens ||
        B * H * (ceil_div(Lq, kBlock) + ceil_div(Lk, kBlock)) > kMaxGrid)
        return SPARSTAR_EINVAL;
    if (int rc = device_check()) return rc;
    return cuda_status(sparstar::launch_pool2(q, Lq, qbar, k, Lk, kbar, dtype, B * H, (int)D,
                                              static_cast<cudaStream_t>(stream)));
}

SPARSTAR_API int64_t sparstar_score_select_max_nkb(int64_t D) {
    if (!head_dim_ok(D)) return -1;
    return sparstar::score_select_max_nkb((int)D);
}

SPARSTAR_API int sparstar_score_select(const float *qbar, const float *kbar, int64_t B,
                                       int64_t H, int64_t nQB, int64_t nKB, int64_t D, float tau,
                                       int64_t n_forced_blocks, double density, int32_t *kv_idx,
                                       int32_t *kv_cnt, int64_t max_sel, int32_t *status,
                                       void *stream) {
    TraceRange trace("sparstar_score_select");
    if (!qbar || !kbar || !kv_idx || !kv_cnt || B <= 0 || H <= 0 || nQB <= 0 || nKB <= 0 ||
        !head_dim_ok(D))
        return SPARSTAR_EINVAL;
    if (!std::isfinite(tau)) return SPARSTAR_EINVAL;
    if (!aligned16(qbar) || !aligned16(kbar)) return SPARSTAR_EINVAL;
    const int64_t sel = sparstar_select_count(nKB, n_forced_blocks, density);
    if (sel < 0) return SPARSTAR_EINVAL;
    if (max_sel < sel) return SPARSTAR_ESIZE;
    if (nKB > sparstar::score_select_max_nkb((int)D)) return SPARSTAR_ESIZE;
    if (sparstar::score_select_ctas(B * H, nQB) > kMaxGrid) return SPARSTAR_EINVAL;
    if (int rc = device_check()) return rc;
    return cuda_status(sparstar::launch_score_select(
        qbar, kbar, B * H, nQB, nKB, (int)D, tau, n_forced_blocks, sel - n_forced_blocks, kv_idx,
        kv_cnt, max_sel, status, static_cast<cudaStream_t>(stream)));
}

SPARSTAR_API int sparstar_forward(const void *q, const void *k, const void *v, int dtype,
                                  int64_t B, int64_t H, int64_t D, int64_t text_len,
                                  int64_t image_ref_len, int64_t ref_len, int64_t cur_len,
                                  double density, float *qbar, float *kbar, float *S,
                                  int32_t *kv_idx, int32_t *kv_cnt, int64_t max_sel, void *out,
                                  float *lse, int32_t *status, void *stream) {
    TraceRange trace("sparstar_forward");
    if (text_len < 0 || image_ref_len < 0 || ref_len < 0 || cur_len <= 0 || !head_dim_ok(D))
        return SPARSTAR_EINVAL;
    const int64_t Lq = cur_len, Lk = text_len + image_ref_len + ref_len + cur_len;
    const int64_t nQB = ceil_div(Lq, kBlock), nKB = ceil_div(Lk, kBlock);
    const int64_t nF = sparstar_forced_blocks(text_len, image_ref_len);
    const float tau = (float)(1.0 / std::sqrt((double)D));
    // Check the whole chain before launching any of it.
    const int64_t sel = sparstar_select_count(nKB, nF, density);
    if (sel < 0) return SPARSTAR_EINVAL;
    if (max_sel < sel) return SPARSTAR_ESIZE;
    int rc = sparstar_block_pool(q, dtype, B, H, Lq, D, qbar, stream);
    if (rc) return rc;
    if ((rc = sparstar_block_pool(k, dtype, B, H, Lk, D, kbar, stream))) return rc;
    if ((rc = sparstar_block_score(qbar, kbar, B, H, nQB, nKB, D, tau, S, stream))) return rc;
    if ((rc = sparstar_select(S, B, H, nQB, nKB, nF, density, kv_idx, kv_cnt, max_sel, stream)))
        return rc;
    return sparstar_attn_fwd(q, k, v, dtype, B, H, Lq, Lk, D, tau, kv_idx, kv_cnt, max_sel, out,
                             lse, status, stream);
}

SPARSTAR_API int sparstar_forward_fused(const void *q, const void *k, const void *v, int dtype,
                                        int64_t B, int64_t H, int64_t D, int64_t text_len,
                                        int64_t image_ref_len, int64_t ref_len, int64_t cur_len,
                                        double density, float *qbar, float *kbar,
                                        int32_t *kv_idx, int32_t *kv_cnt, int64_t max_sel,
                                        void *out, float *lse, int32_t *status, void *stream) {
    TraceRange trace("sparstar_forward_fused");
    if (text_len < 0 || image_ref_len < 0 || ref_len < 0 || cur_len <= 0 || !head_dim_ok(D))
        return SPARSTAR_EINVAL;
    const int64_t Lq = cur_len, Lk = text_len + image_ref_len + ref_len + cur_len;
    const int64_t nQB = ceil_div(Lq, kBlock), nKB = ceil_div(Lk, kBlock);
    const int64_t nF = sparstar_forced_blocks(text_len, image_ref_len);
    const float tau = (float)(1.0 / std::sqrt((double)D));
    const int64_t sel = sparstar_select_count(nKB, nF, density);
    if (sel < 0) return SPARSTAR_EINVAL;
    if (max_sel < sel) return SPARSTAR_ESIZE;
    if (nKB > sparstar::score_select_max_nkb((int)D)) return SPARSTAR_ESIZE;
    int rc = sparstar_block_pool_qk(q, k, dtype, B, H, Lq, Lk, D, qbar, kbar, stream);
    if (rc) return rc;
    if ((rc = sparstar_score_select(qbar, kbar, B, H, nQB, nKB, D, tau, nF, density, kv_idx,
                                    kv_cnt, max_sel, status, stream)))
        return rc;
    return sparstar_attn_fwd(q, k, v, dtype, B, H, Lq, Lk, D, tau, kv_idx, kv_cnt, max_sel, out,
                             lse, status, stream);
}

SPARSTAR_API int sparstar_retained_mass(const void *q, const void *k, int dtype, int64_t B,
                                        int64_t H, int64_t Lq, int64_t Lk, int64_t D, float tau,
                                        int64_t n_forced_blocks, const int32_t *kv_idx,
                                        const int32_t *kv_cnt, int64_t max_sel,
                                        const int64_t *rows, int64_t n_rows, float *scratch,
                                        double *lse_dense, double *mass_block, double *mass_tok,
                                        double *mass_forced, void *stream) {
    TraceRange trace("sparstar_retained_mass");
    if (!dtype_ok(dtype)) return SPARSTAR_EDTYPE;
    if (!q || !k || !kv_cnt || !rows || !scratch || !lse_dense || !mass_block || !mass_tok ||
        !mass_forced || B <= 0 || H <= 0 || Lq <= 0 || Lk <= 0 || !head_dim_ok(D) ||
        n_rows <= 0 || max_sel < 0)
        return SPARSTAR_EINVAL;
    if (max_sel > 0 && !kv_idx) return SPARSTAR_EINVAL;
    if (!std::isfinite(tau) || !aligned16(q) || !aligned16(k)) return SPARSTAR_EINVAL;
    const int64_t nKB = ceil_div(Lk, kBlock);
    if (n_forced_blocks < 0 || n_forced_blocks > nKB) return SPARSTAR_EINVAL;
    if (Lq > kMaxTokens || Lk > kMaxTokens || nKB > sparstar::mass_max_nkb() ||
        n_rows > kMaxGrid || max_sel > 0x7fffffffLL)
        return SPARSTAR_EINVAL;
    if (int rc = device_check()) return rc;
    return cuda_status(sparstar::launch_retained_mass(
        q, k, dtype, B * H, Lq, Lk, (int)D, tau, n_forced_blocks, kv_idx, kv_cnt, max_sel, rows,
        n_rows, scratch, lse_dense, mass_block, mass_tok, mass_forced,
        static_cast<cudaStream_t>(stream)));
}

namespace {

// Checks shared by the transfer and its stride helper; fills the layout.
int transfer_layout(const int64_t *src_len, const int64_t *dst_len, int64_t src_max_sel,
                    sparstar::TransferLayout *ly) {
    if (!src_len || !dst_len || src_max_sel < 1 || src_max_sel > 0x7fffffffLL)
        return SPARSTAR_EINVAL;
    int64_t Ls = 0, Lt = 0;
    for (int g = 0; g < 4; ++g) {
        if (src_len[g] < 0 || dst_len[g] < 0 || src_len[g] > kMaxTokens ||
            dst_len[g] > kMaxTokens)
            return SPARSTAR_EINVAL;
        Ls += src_len[g];
        Lt += dst_len[g];
    }
    if (Ls > kMaxTokens || Lt > kMaxTokens) return SPARSTAR_EINVAL;
    if (dst_len[3] > 0 && src_len[3] == 0) return SPARSTAR_EINVAL;
    if (ceil_div(Ls, kBlock) > sparstar::transfer_max_nkb() ||
        ceil_div(Lt, kBlock) > sparstar::transfer_max_nkb())
        return SPARSTAR_ESIZE;
    *ly = sparstar::make_transfer_layout(src_len, dst_len);
    return SPARSTAR_OK;
}

}  // namespace

SPARSTAR_API int64_t sparstar_transfer_max_sel(const int64_t *src_len, const int64_t *dst_len,
                                               int64_t src_max_sel) {
    sparstar::TransferLayout ly;
    if (transfer_layout(src_len, dst_len, src_max_sel, &ly) != SPARSTAR_OK) return -1;
    return sparstar::transfer_max_sel(ly, src_max_sel);
}

SPARSTAR_API int sparstar_transfer_lists(const int32_t *src_idx, const int32_t *src_cnt,
                                         int64_t src_max_sel, int64_t B, int64_t H,
                                         const int64_t *src_len, const int64_t *dst_len,
                                         int32_t *dst_idx, int32_t *dst_cnt, int64_t dst_max_sel,
                                         void *stream) {
    TraceRange trace("sparstar_transfer_lists");
    if (!src_idx || !src_cnt || !dst_idx || !dst_cnt || B <= 0 || H <= 0 ||
        dst_max_sel > 0x7fffffffLL)
        return SPARSTAR_EINVAL;
    sparstar::TransferLayout ly;
    if (int rc = transfer_layout(src_len, dst_len, src_max_sel, &ly)) return rc;
    if (dst_max_sel < sparstar::transfer_max_sel(ly, src_max_sel)) return SPARSTAR_ESIZE;
    if (dst_len[3] == 0) return SPARSTAR_OK;
    // list sizes in elements (in double: the product of four checked
    // sizes may not fit in int64)
    if (B > kMaxGrid || H > kMaxGrid ||
        (double)B * H * ceil_div(src_len[3], kBlock) * src_max_sel > 1e12 ||
        (double)B * H * ceil_div(dst_len[3], kBlock) * dst_max_sel > 1e12)
        return SPARSTAR_EINVAL;
    if (int rc = device_check()) return rc;
    return cuda_status(sparstar::launch_transfer_lists(src_idx, src_cnt, src_max_sel, B * H, ly,
                                                       dst_idx, dst_cnt, dst_max_sel,
                                                       static_cast<cudaStream_t>(stream)));
}

SPARSTAR_API int sparstar_test_attn_timeout(const void *q, const void *k, const void *v,
                                            int64_t B, int64_t H, int64_t Lq, int64_t Lk,
                                            const int32_t *kv_idx, const int32_t *kv_cnt,
                                            int64_t max_sel, void *out, int32_t *status,
                                            void *stream) {
    TraceRange trace("sparstar_test_attn_timeout");
    if (!q || !k || !v || !out || !kv_cnt || !status || B <= 0 || H <= 0 || Lq <= 0 ||
        Lk <= 0 || max_sel < 0 || (max_sel > 0 && !kv_idx))
        return SPARSTAR_EINVAL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
        return SPARSTAR_EINVAL;
    if (Lq > kMaxTokens || Lk > kMaxTokens || max_sel > 0x7fffffffLL ||
        B * H * ceil_div(Lq, kBlock) > kMaxGrid || B * H > 0x7fffffffLL)
        return SPARSTAR_EINVAL;
    if (int rc = device_check()) return rc;
    return sparstar::launch_attn_sm100(q, k, v, B * H, Lq, Lk, 0.0883883476f, kv_idx, kv_cnt,
                                       max_sel, out, nullptr, status,
                                       static_cast<cudaStream_t>(stream), true);
}
