// iabn_noalloc.cu -- iabn_forward_static_ws: the training forward of
// iabn_forward with its scratch taken from a fixed array of device memory
// that this library owns, for callers that cannot allocate device memory.
//
// Who needs it: a plugin layer inside a host framework whose own allocator
// owns the device memory and hands the plugin only the tensors it works on;
// and real-time loops that forbid device allocation after start-up
// (cudaMalloc can synchronise the device and stall).  Such callers still
// pass their inputs and outputs; only the scratch comes from here.
//
// The array is file-scope device memory of kStaticWsBytes, held on every GPU
// that loads this library until the process exits.  Host code may not use
// the symbol itself as a device address, so the first call on each device
// (with that device current) looks the address up with cudaGetSymbolAddress
// and caches it for the life of the process (a cudaDeviceReset discards the
// array, so callers must not use this entry point on that device after one).
// Every call on a device shares the array: calls that overlap on the GPU race.
#include <cuda_runtime.h>

#include <mutex>

#include "iabn.h"
#include "iabn_device.cuh"

namespace {

constexpr size_t kStaticWsBytes = (size_t)8 << 20;   // 8 MiB

// Scratch shared by every call of iabn_forward_static_ws on a device.
static __device__ __align__(256) unsigned char g_static_ws[kStaticWsBytes];

std::mutex g_ws_mu;
void* g_ws_addr[64] = {nullptr};

// Device address of g_static_ws on the current device (looked up once).
cudaError_t static_ws_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_ws_mu);
    if (g_ws_addr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_ws);
        if (e != cudaSuccess) return e;
        g_ws_addr[dev] = p;
    }
    *out = g_ws_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" iabn_status iabn_forward_static_ws(const iabn_desc* d, void* x_inout,
                                              const float* gamma, const float* beta, float eps,
                                              int32_t act, float act_param, float* save_mean,
                                              float* save_var, void* stream) {
    // Every argument check of iabn_forward runs before its workspace check,
    // so a call without a workspace reports any other problem first and
    // launches nothing.
    const iabn_status probe = iabn_forward(d, x_inout, gamma, beta, eps, act, act_param,
                                           save_mean, save_var, nullptr, 0, stream);
    if (probe != IABN_ERR_WORKSPACE) return probe;
    const size_t need = iabn_workspace_size(d);
    if (need == 0 || need > kStaticWsBytes) return IABN_ERR_WORKSPACE;
    void* ws = nullptr;
    if (static_ws_address(&ws) != cudaSuccess) {
        cudaGetLastError();
        return IABN_ERR_CUDA;
    }
    // The control block (sticky status, grid-barrier counters) must start at
    // zero; the rest of the scratch is written before it is read.
    if (cudaMemsetAsync(ws, 0, sizeof(iabn::Control), static_cast<cudaStream_t>(stream)) !=
        cudaSuccess) {
        cudaGetLastError();
        return IABN_ERR_CUDA;
    }
    return iabn_forward(d, x_inout, gamma, beta, eps, act, act_param, save_mean, save_var, ws,
                        kStaticWsBytes, stream);
}

extern "C" iabn_status iabn_get_static_ws_status(void* stream) {
    void* ws = nullptr;
    if (static_ws_address(&ws) != cudaSuccess) {
        cudaGetLastError();
        return IABN_ERR_CUDA;
    }
    return iabn_get_device_status(ws, stream);
}
