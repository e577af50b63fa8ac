// sparstar_forward_static: the four steps of one scale (pool Q, pool K,
// score, select, attention) with the intermediate buffers (block means,
// scores, block lists) held in a fixed arena of device memory that belongs
// to the library, instead of in workspace the caller allocates.
//
// It exists for callers that cannot allocate device memory themselves: a
// host program that only hands this library its input and output buffers,
// or a plugin whose host forbids any device allocation outside its own
// pool.  Nothing here calls cudaMalloc, cudaFree or an allocating library
// routine.
//
// The arena is one file-scope __device__ array of kArenaBytes.  Every GPU
// that loads the library reserves it when the module is loaded and keeps
// it until the process exits.  Host code cannot use the array's name as a
// device address (on the host it names a stand-in), so the first call on
// each device, with that device current, looks the address up once with
// cudaGetSymbolAddress and caches it; that first call should be made
// before any stream capture starts.  The cache entry remembers the unique
// id of the CUDA context it was taken in (cuCtxGetId): a call made in
// another context (a non-primary one, or a new primary context after
// cudaDeviceReset, where the module may be loaded at another address)
// looks the address up again instead of using a stale one.  All calls
// share the arena: calls whose work overlaps on the GPU (different
// streams, or different host threads) race on it and must be serialised
// by the caller.  Every byte a call reads from the arena is written
// earlier in the same call, so no clearing is needed.
#include <cmath>
#include <cstddef>
#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "sparstar.h"
#include "sparstar_internal.h"

#define SPARSTAR_API extern "C" __attribute__((visibility("default")))

namespace {

constexpr size_t kArenaBytes = SPARSTAR_STATIC_ARENA_BYTES;  // 64 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_arena[kArenaBytes];

std::mutex g_setup_mutex;
struct ArenaEntry {
    unsigned long long ctx_id;  // unique id of the context the address belongs to
    void *addr;                 // device address of g_arena in that context
};
ArenaEntry g_arena_cache[kMaxDevices];

// Unique id of the calling thread's current CUDA context, or 0 when none
// is current yet.  The driver entry points are looked up through the
// runtime, so the library keeps loading on hosts without a driver.
int current_context_id(unsigned long long *id) {
    using GetCurrent = CUresult (*)(CUcontext *);
    using GetId = CUresult (*)(CUcontext, unsigned long long *);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    if (!get_current || !get_id) {
        void *a = nullptr, *b = nullptr;
        cudaDriverEntryPointQueryResult qa, qb;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) != cudaSuccess ||
            cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) != cudaSuccess ||
            qa != cudaDriverEntryPointSuccess || qb != cudaDriverEntryPointSuccess) {
            cudaGetLastError();
            return SPARSTAR_ECUDA;
        }
        get_current = reinterpret_cast<GetCurrent>(a);
        get_id = reinterpret_cast<GetId>(b);
    }
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS) return SPARSTAR_ECUDA;
    *id = 0;
    if (ctx && get_id(ctx, id) != CUDA_SUCCESS) return SPARSTAR_ECUDA;
    return SPARSTAR_OK;
}

// Device address of the arena on the current device, in the current
// context (looked up once per device and context).
int arena_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return SPARSTAR_ENODEV;
    }
    if (dev < 0 || dev >= kMaxDevices) return SPARSTAR_ENODEV;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    unsigned long long id = 0;
    if (int rc = current_context_id(&id)) return rc;
    ArenaEntry &entry = g_arena_cache[dev];
    if (id != 0 && entry.addr && entry.ctx_id == id) {
        *out = entry.addr;
        return SPARSTAR_OK;
    }
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_arena) != cudaSuccess || !p) {
        cudaGetLastError();
        return SPARSTAR_ECUDA;
    }
    // The lookup makes the device's primary context current when none was.
    if (id == 0) {
        if (int rc = current_context_id(&id)) return rc;
    }
    entry.ctx_id = id;
    entry.addr = p;
    *out = p;
    return SPARSTAR_OK;
}

size_t round256(size_t n) { return (n + 255) & ~size_t(255); }

}  // namespace

namespace {

int forward_static_impl(const void *q, const void *k, const void *v, int dtype, int64_t B,
                        int64_t H, int64_t D, int64_t text_len, int64_t image_ref_len,
                        int64_t ref_len, int64_t cur_len, double density, void *out, float *lse,
                        int32_t *status, void *stream) {
    if (B <= 0 || H <= 0 || (D != 64 && D != 128) || text_len < 0 || image_ref_len < 0 ||
        ref_len < 0 || cur_len <= 0)
        return SPARSTAR_EINVAL;
    const int64_t Lk = text_len + image_ref_len + ref_len + cur_len;
    const int64_t nQB = sparstar::ceil_div(cur_len, sparstar::kBlock);
    const int64_t nKB = sparstar::ceil_div(Lk, sparstar::kBlock);
    const int64_t nF = sparstar_forced_blocks(text_len, image_ref_len);
    const int64_t sel = sparstar_select_count(nKB, nF, density);
    if (sel < 0) return SPARSTAR_EINVAL;
    // Arena layout: qbar | kbar | S | kv_idx | kv_cnt, each 256-byte aligned.
    const double need_d = 4.0 * (double)B * (double)H *
                          ((double)nQB * D + (double)nKB * D + (double)nQB * nKB +
                           (double)nQB * sel + (double)nQB) + 5 * 256.0;
    if (need_d > (double)kArenaBytes) return SPARSTAR_ESIZE;
    const size_t BH = (size_t)(B * H);
    const size_t s_qbar = round256(BH * nQB * D * sizeof(float));
    const size_t s_kbar = round256(BH * nKB * D * sizeof(float));
    const size_t s_S = round256(BH * nQB * nKB * sizeof(float));
    const size_t s_idx = round256(BH * nQB * sel * sizeof(int32_t));
    const size_t s_cnt = round256(BH * nQB * sizeof(int32_t));
    if (s_qbar + s_kbar + s_S + s_idx + s_cnt > kArenaBytes) return SPARSTAR_ESIZE;

    void *arena = nullptr;
    if (int rc = arena_address(&arena)) return rc;
    unsigned char *a = static_cast<unsigned char *>(arena);
    float *qbar = reinterpret_cast<float *>(a);
    float *kbar = reinterpret_cast<float *>(a + s_qbar);
    float *S = reinterpret_cast<float *>(a + s_qbar + s_kbar);
    int32_t *kv_idx = reinterpret_cast<int32_t *>(a + s_qbar + s_kbar + s_S);
    int32_t *kv_cnt = reinterpret_cast<int32_t *>(a + s_qbar + s_kbar + s_S + s_idx);
    return sparstar_forward(q, k, v, dtype, B, H, D, text_len, image_ref_len, ref_len, cur_len,
                            density, qbar, kbar, S, kv_idx, kv_cnt, sel, out, lse, status, stream);
}

}  // namespace

SPARSTAR_API int sparstar_forward_static(const void *q, const void *k, const void *v, int dtype,
                                         int64_t B, int64_t H, int64_t D, int64_t text_len,
                                         int64_t image_ref_len, int64_t ref_len, int64_t cur_len,
                                         double density, void *out, float *lse, int32_t *status,
                                         void *stream) {
    nvtxRangePushA("sparstar_forward_static");  // one NVTX range per ABI call
    const int rc = forward_static_impl(q, k, v, dtype, B, H, D, text_len, image_ref_len, ref_len,
                                       cur_len, density, out, lse, status, stream);
    nvtxRangePop();
    return rc;
}
