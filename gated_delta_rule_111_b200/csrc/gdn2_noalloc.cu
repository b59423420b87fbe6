// gdn2_chunk_bwd_noalloc: the chunkwise backward for callers that cannot
// allocate device memory when they call it.
//
// Who cannot allocate: code running inside another runtime's memory manager (a
// framework's caching allocator that must own every device allocation, an
// embedded engine with a fixed memory budget decided at start-up), and host
// threads on a latency-critical path, where cudaMalloc and cudaFree may
// synchronise the device.  Such callers pass inputs and outputs only; the
// workspace of the backward is a fixed array in this library's own device
// memory instead of a caller buffer.
//
// That array is reserved on every GPU on which this library's device code is
// loaded and stays reserved until the process exits.  All calls share it, and
// it keeps what the last call left there: nothing in it needs to start at zero
// (every workspace element is written before it is read within one call), but
// two calls whose kernels overlap on the GPU (different streams, or different
// host threads, without ordering between them) race on it and corrupt each
// other's results.
#include <stdio.h>

#include <mutex>

#include "common.cuh"

namespace gdn2 {
void set_last_error(const char *message);
}

namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;     // 32 MiB, the largest workspace served

// The scratch array.  In host code this name only stands for the device symbol;
// its device address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void *g_scratch_address[kMaxDevices];   // device address of g_scratch per device; null until looked up

// Device address of g_scratch on the current device, looked up on the first call
// there (which also makes the runtime load this library's device code on that
// device, if nothing else has yet).
cudaError_t scratch_address(void **out) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_address[dev]) {
        void *p = nullptr;
        err = cudaGetSymbolAddress(&p, g_scratch);
        if (err != cudaSuccess) return err;
        g_scratch_address[dev] = p;
    }
    *out = g_scratch_address[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" gdn2_status gdn2_chunk_bwd_noalloc(const void *q, const void *k, const void *v, const float *alpha,
                                              const float *b, const float *w, const float *S0, const void *dO,
                                              const float *dST, void *dq, void *dk, void *dv, float *dalpha,
                                              float *db, float *dw, float *dS0, int B, int T, int H, int d_k,
                                              int d_v, gdn2_dtype dt, void *stream) {
    const size_t need = gdn2_chunk_bwd_workspace_size(B, T, H, d_k, d_v);
    if (need > kScratchBytes) {
        char msg[200];
        snprintf(msg, sizeof(msg),
                 "gdn2_chunk_bwd_noalloc: these sizes need %zu bytes of workspace, more than its fixed %zu "
                 "(use gdn2_chunk_bwd with a caller buffer)", need, kScratchBytes);
        gdn2::set_last_error(msg);
        return GDN2_ERR_INVALID_ARG;
    }
    void *ws = nullptr;
    const cudaError_t err = scratch_address(&ws);
    if (err != cudaSuccess) {
        char msg[200];
        snprintf(msg, sizeof(msg), "gdn2_chunk_bwd_noalloc: looking up the scratch array: %s",
                 cudaGetErrorString(err));
        gdn2::set_last_error(msg);
        return GDN2_ERR_CUDA;
    }
    return gdn2_chunk_bwd(q, k, v, alpha, b, w, S0, dO, dST, dq, dk, dv, dalpha, db, dw, dS0, ws, kScratchBytes, B, T,
                          H, d_k, d_v, dt, stream);
}
