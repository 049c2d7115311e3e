// simple_gla_fwd_noalloc: the dense forward with library-owned scratch memory.
//
// Some callers cannot hand the library a workspace, because they are not allowed
// to allocate device memory at all: a plugin running inside another runtime that
// owns the whole GPU memory pool and forbids foreign cudaMalloc/cudaFree, or a
// latency-critical loop where an allocation (which may synchronise the device)
// is not acceptable after start-up.  For them this entry point takes its scratch
// from a fixed array compiled into the library instead of from a caller buffer.
// It is a thin front of simple_gla_fwd: same kernels, same results.
//
// Cost and limits:
//   * the array (kStaticScratchBytes = 16 MiB) exists on every GPU that loads the
//     library and stays allocated until the process exits;
//   * a problem whose workspace (simple_gla_fwd_workspace_size) exceeds it is
//     refused with SGLA_ERR_WORKSPACE;
//   * every call on a device shares the one array: calls whose work can overlap on
//     the GPU (different streams without ordering) race on it.  Whatever must
//     start at zero is cleared by the forward itself (its status word); the rest
//     of the scratch is always written before it is read;
//   * the first call on each device looks up the device address of the array
//     (cudaGetSymbolAddress, with that device current); make that first call
//     before any stream capture begins.  The address is kept for the life of the
//     process: after cudaDeviceReset (or anything else that destroys the device's
//     primary context) it is stale, and the entry point must not be used again;
//   * the forward's device status word (a time-out of a bounded device wait, for
//     instance) sits at the head of the array, where the caller cannot name it:
//     sgla_noalloc_status reads it back.
#include <mutex>

#include "launch_status.h"
#include "simple_gla.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 128;
void *g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mutex;

// Device address of g_static_scratch on the current device.  In host code the
// array's name only stands in for the symbol; it is not a device address, so it is
// resolved here once per device and cached.
sgla_status static_scratch(void **out) {
    int dev = -1;
    const cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return sgla::cuda_failure(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return sgla::cuda_failure(cudaErrorInvalidDevice, "cudaGetDevice");
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        const cudaError_t es = cudaGetSymbolAddress(&p, g_static_scratch);
        if (es != cudaSuccess) return sgla::cuda_failure(es, "cudaGetSymbolAddress");
        if (p == nullptr) return sgla::cuda_failure(cudaErrorInvalidSymbol, "cudaGetSymbolAddress");
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return SGLA_OK;
}

}  // namespace

extern "C" sgla_status simple_gla_fwd_noalloc(const void *q, const void *k, const void *v, const float *g,
                                              const float *g_gamma, float scale, const float *initial_state,
                                              void *o, float *final_state, int64_t B, int64_t T, int64_t H,
                                              int64_t K, int64_t V, int chunk_size, sgla_dtype dtype,
                                              void *stream) {
    const size_t need = simple_gla_fwd_workspace_size(B, T, H, K, V, chunk_size, dtype);
    if (need > kStaticScratchBytes) return SGLA_ERR_WORKSPACE;
    void *scratch = nullptr;
    const sgla_status st = static_scratch(&scratch);
    if (st != SGLA_OK) return st;
    // need == 0 means invalid sizes: simple_gla_fwd reports which error.
    return simple_gla_fwd(q, k, v, g, g_gamma, scale, initial_state, o, final_state, B, T, H, K, V, chunk_size,
                          dtype, scratch, kStaticScratchBytes, stream);
}

extern "C" sgla_status sgla_noalloc_status(int *device_status, void *stream) {
    if (!device_status) return SGLA_ERR_INVALID_ARGUMENT;
    void *scratch = nullptr;
    const sgla_status st = static_scratch(&scratch);
    if (st != SGLA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int host = -1;
    cudaError_t e = cudaMemcpyAsync(&host, scratch, sizeof(int), cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return sgla::cuda_failure(e, "noalloc status read");
    e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return sgla::cuda_failure(e, "noalloc status sync");
    *device_status = host;
    return SGLA_OK;
}
