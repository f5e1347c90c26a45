// pdr_render_fwd_noalloc: the forward render for callers that cannot allocate
// device memory themselves -- for example a plugin whose host application owns
// every byte of device memory through its own pool, or a real-time loop that
// must not allocate once it has started.  Such a caller has its inputs and
// outputs but no way to provide the workspace that pdr_render_fwd needs, so
// this entry point uses a fixed scratch array compiled into the library
// instead.  It calls no cudaMalloc, cudaFree or allocating library routine.
//
// The paper has no counterpart: this is a convenience of the library's
// interface, not a step of the method.
#include <mutex>

#include "common.cuh"
#include "pdr.h"

namespace {

// The scratch that replaces the caller's workspace.  Every GPU that loads
// libpdr.so holds PDR_STATIC_SCRATCH_BYTES of it until the process exits.  In
// host code `g_scratch` only names the variable: its device address comes from
// cudaGetSymbolAddress, looked up once per device.
static __device__ __align__(256) unsigned char g_scratch[PDR_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void *g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mutex;

// Device address of g_scratch on the current device (looked up on the first
// call made with that device current, then cached).
cudaError_t scratch_address(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" pdr_status pdr_render_fwd_noalloc(const float *params, int B, int N, int C, int H,
                                             int W, int k, float *image, void *stream) {
    if (B < 1 || N < 0 || C < 1 || H < 1 || W < 1 || k < 1 || (k & 1) == 0 ||
        (N > 0 && !params) || !image)
        return PDR_ERR_INVALID_ARG;
    const size_t need = pdr_workspace_bytes(B, N, C, H, W, k);
    if (need == 0 || need > PDR_STATIC_SCRATCH_BYTES) return PDR_ERR_TOO_LARGE;
    void *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return PDR_ERR_CUDA;
    // The bins are rebuilt on every call, and every word of the scratch that
    // the kernels read is written earlier in the same call (the error word is
    // cleared before the first kernel), so the previous call's leftovers never
    // leak.
    return pdr_render_fwd(params, B, N, C, H, W, k, image, scratch, PDR_STATIC_SCRATCH_BYTES,
                          /*workspace_holds_bins=*/0, stream);
}

extern "C" pdr_status pdr_check_device_error_noalloc(void *stream) {
    void *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return PDR_ERR_CUDA;
    // The error word is the first word of any workspace layout.
    return pdr_check_device_error(scratch, stream);
}
