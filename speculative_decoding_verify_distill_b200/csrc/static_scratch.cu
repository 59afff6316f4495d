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
// static __device__ array; its address is looked up once per device (cudaGetSymbolAddress with
// that device current) under a lock and cached.  Each call clears the bytes it uses with one
// cudaMemsetAsync on the caller's stream, runs the same kernels as svd_verify_distill on that
// scratch, and (optionally) copies the device status word to a caller-owned device location.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "svd_internal.h"

namespace {

// Largest workspace the static scratch can stand in for: 4 MiB per device.  At k = 16 and a
// 256-unit length head this covers batches of several hundred sequences (about 1.4 MiB at
// B = 128); larger calls are rejected with SVD_ERR_WORKSPACE before anything is launched.
constexpr size_t kScratchBytes = size_t(4) << 20;
static_assert(kScratchBytes == SVD_NOALLOC_SCRATCH_BYTES, "header and library agree on the size");

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_lock;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_scratch on the current device; looked up on the first call per device.
svd_status scratch_for_current_device(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return SVD_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return SVD_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> guard(g_setup_lock);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) return SVD_ERR_CUDA;
        if ((reinterpret_cast<uintptr_t>(p) & 255u) != 0) return SVD_ERR_ALIGNMENT;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return SVD_OK;
}

}  // namespace

extern "C" svd_status svd_verify_distill_noalloc(const svd_verify_distill_args* a,
                                                 uint32_t* status_out, void* stream) {
    if (a == nullptr) return SVD_ERR_INVALID_ARG;
    const int M = a->h != nullptr ? a->M : 0;
    const size_t need = svd_workspace_bytes(a->B, a->k, a->kt, M);
    // need == 0: a shape svd_verify_distill rejects; B == 0: nothing to launch.  Both return
    // before the workspace is touched, so no scratch is set up for them.
    if (need == 0 || a->B == 0) return svd_verify_distill(a, nullptr, 0, stream);
    if (need > kScratchBytes) return SVD_ERR_WORKSPACE;
    void* ws = nullptr;
    svd_status s = scratch_for_current_device(&ws);
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
