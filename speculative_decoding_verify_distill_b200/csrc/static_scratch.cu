// static_scratch.cu -- svd_verify_distill_noalloc: the fused verify-and-distill call with its
// scratch in a fixed, file-scope device array instead of a caller-provided workspace.
//
// Who needs it: callers that cannot allocate device memory on their path -- a plain C host
// program with no device allocator of its own, or an embedding runtime that claims nearly all
// HBM for its own pools at start-up (a serving engine's KV-cache pool) and forbids cudaMalloc
// afterwards, since cudaMalloc may synchronise the device and fails once the memory is claimed.
// Such a caller cannot provide the workspace svd_verify_distill asks for; this entry point
// brings its own, of a fixed maximum size, created with the library's device image.
//
// Nothing here allocates: no cudaMalloc / cudaFree, no allocating library.  The scratch is a
// static __device__ array.  Its device address belongs to the CUDA context that loaded the
// library's device image, not to the device number: a caller on the driver API may run under a
// context of its own, and a context destroyed and re-created (cudaDeviceReset) maps the array
// again, possibly elsewhere.  So the address is looked up (cudaGetSymbolAddress, with that
// context current) once per context, keyed by the context's unique id, under a lock, and
// cached.  Every call first checks all arguments, then clears the bytes it uses with one
// cudaMemsetAsync on the caller's stream, runs the same kernels as svd_verify_distill on that
// scratch, and (optionally) copies the device status word to a caller-owned device location.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "svd_internal.h"

namespace {

// Largest workspace the static scratch can stand in for: 4 MiB per device.  At k = 16 and a
// 256-unit length head this covers batches of several hundred sequences (about 1.7 MiB at
// B = 128); larger calls are rejected with SVD_ERR_WORKSPACE before anything is launched.
constexpr size_t kScratchBytes = size_t(4) << 20;
static_assert(kScratchBytes == SVD_NOALLOC_SCRATCH_BYTES, "header and library agree on the size");

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// Context ids come from the driver (cuCtxGetCurrent + cuCtxGetId, CUDA 12.0), reached through
// the runtime's entry-point query so that the library does not link the driver library itself.
using CtxGetCurrentFn = int (*)(void** ctx);
using CtxGetIdFn = int (*)(void* ctx, unsigned long long* id);

struct CacheEntry {
    unsigned long long ctx_id;   // 0: empty
    void* ptr;
};
constexpr int kCacheEntries = 64;
std::mutex g_setup_lock;
CacheEntry g_cache[kCacheEntries] = {};
int g_cache_next = 0;            // round-robin slot for a new context once the cache is full
bool g_driver_tried = false;
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;

// Unique id of the current context; 0 if no context is current yet on this thread (the runtime
// binds its primary context on the first call that needs one) or the driver cannot say.  With
// id 0 the address is looked up without caching it.
unsigned long long current_context_id() {
    if (!g_driver_tried) {
        g_driver_tried = true;
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 12000, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(f);
        f = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &f, 12000, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(f);
    }
    if (!g_ctx_get_current || !g_ctx_get_id) return 0;
    void* ctx = nullptr;
    unsigned long long id = 0;
    if (g_ctx_get_current(&ctx) != 0 || ctx == nullptr) return 0;
    if (g_ctx_get_id(ctx, &id) != 0) return 0;
    return id;
}

// Device address of g_scratch in the current context: looked up once per context.
svd_status scratch_for_current_context(void** out) {
    std::lock_guard<std::mutex> guard(g_setup_lock);
    const unsigned long long id = current_context_id();
    if (id != 0) {
        for (int e = 0; e < kCacheEntries; ++e) {
            if (g_cache[e].ctx_id == id) {
                *out = g_cache[e].ptr;
                return SVD_OK;
            }
        }
    }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) return SVD_ERR_CUDA;
    if ((reinterpret_cast<uintptr_t>(p) & 255u) != 0) return SVD_ERR_ALIGNMENT;
    if (id != 0) {
        g_cache[g_cache_next] = CacheEntry{id, p};
        g_cache_next = (g_cache_next + 1) % kCacheEntries;
    }
    *out = p;
    return SVD_OK;
}

}  // namespace

extern "C" svd_status svd_verify_distill_noalloc(const svd_verify_distill_args* a,
                                                 uint32_t* status_out, void* stream) {
    // every argument check first: a rejected call touches neither the scratch nor the device
    svd_status s = svd::check_verify_distill_args(a);
    if (s != SVD_OK || a->B == 0) return s;
    const int M = a->h != nullptr ? a->M : 0;
    const size_t need = svd_workspace_bytes(a->B, a->k, a->kt, M);
    if (need == 0) return SVD_ERR_INVALID_ARG;
    if (need > kScratchBytes) return SVD_ERR_WORKSPACE;
    void* ws = nullptr;
    s = scratch_for_current_context(&ws);
    if (s != SVD_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the kernels expect an all-zero workspace; clearing it here also drops a status word or
    // ticket left behind by an earlier call that ended in a device error
    if (cudaMemsetAsync(ws, 0, need, st) != cudaSuccess) return SVD_ERR_CUDA;
    s = svd_verify_distill(a, ws, kScratchBytes, stream);
    if (s != SVD_OK) return s;
    if (status_out != nullptr &&
        cudaMemcpyAsync(status_out, ws, sizeof(uint32_t), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return SVD_ERR_CUDA;
    return SVD_OK;
}
