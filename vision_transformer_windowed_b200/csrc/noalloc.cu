// Backward entry point that allocates nothing.
//
// fs_winattn_bwd needs a device workspace from its caller.  Some callers
// cannot provide one: code that runs where a device allocation is not allowed
// or not possible at that moment (inside a fixed memory pool that is already
// fully handed out, a runtime that forbids cudaMalloc after start-up, or a
// framework hook that may not touch the allocator).  For them this file keeps
// one scratch array in the library itself, a file-scope __device__ array of
// kNoAllocScratchBytes (64 MiB).  Every GPU that loads this library holds that
// array until the process exits.
//
// The array is shared by every call on a device and keeps the last call's
// contents; the backward clears what must start at zero itself (its dQ
// accumulator).  Calls whose kernels overlap on the GPU (different streams, or
// host threads, without ordering between them) race on the array.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/fswin.h"
#include "geometry.cuh"
#include "kernels.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
constexpr int kMaxDevices = 64;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  The array's name
// in host code is only a stand-in for the symbol, so its address is looked up
// once per device (with that device current) and cached.
fs_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FS_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return FS_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return FS_OK;
}

}  // namespace

extern "C" {

size_t fs_winattn_bwd_noalloc_max_bytes(void) { return kNoAllocScratchBytes; }

fs_status fs_winattn_bwd_noalloc(const fs_winattn_shape* shape, const void* q, const void* k, const void* v,
                                 const void* o, const void* dout, const float* lse, const float* theta, void* dq,
                                 void* dk, void* dv, float* dtheta, fs_stream_t stream) {
    fs_status st = fs_winattn_check_shape(shape);
    if (st != FS_OK) return st;
    if (fs_winattn_bwd_workspace_bytes(shape) > kNoAllocScratchBytes) return FS_ERR_WORKSPACE;
    // the device check first: on another architecture the symbol lookup below
    // would fail with a CUDA error instead of FS_ERR_ARCH
    if ((st = static_cast<fs_status>(fswin::device_ready())) != FS_OK) return st;
    void* scratch = nullptr;
    if ((st = scratch_address(&scratch)) != FS_OK) return st;
    return fs_winattn_bwd(shape, q, k, v, o, dout, lse, theta, dq, dk, dv, dtheta, scratch, kNoAllocScratchBytes,
                          stream);
}

}  // extern "C"
