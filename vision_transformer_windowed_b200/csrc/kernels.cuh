// Host-side launch entry points of the kernels, shared by api.cu.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <mutex>

#include "geometry.cuh"

namespace fswin {

// Opts a kernel into more than the default 48 KB of dynamic shared memory.  The
// attribute is per device, so it is set once for every device the kernel is
// launched on (the first launch there, with that device current), under a lock
// because several host threads may launch at once.
class SmemOptIn {
   public:
    cudaError_t ensure(const void* func, int bytes) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= kDevices)
            return cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        std::lock_guard<std::mutex> lk(mu_);
        if (!done_[dev]) {
            e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
            if (e != cudaSuccess) return e;
            done_[dev] = true;
        }
        return cudaSuccess;
    }

   private:
    static constexpr int kDevices = 64;
    std::mutex mu_;
    bool done_[kDevices] = {};
};

// Checks that the current device can run the kernels (sm_100) and sets up the
// library's per-device state; returns an fs_status code (0 when usable).
int device_ready();

long long fwd_items(const Geo& g);
// train_ws: NULL, or the backward's workspace (windows of >= 128 tokens): the
// forward then first writes the rotated q', k' tile images there (the images
// the backward's prep would write) and reads Q', K' from them, instead of
// rotating every K tile again for each query tile of its window.
cudaError_t launch_fwd(const Geo& g, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                       const CUtensorMap& mo, const void* q, const void* k, const void* v, void* o,
                       const float* theta, float* lse, unsigned int* status,
                       unsigned long long limit_ns, int num_sms, cudaStream_t stream, cudaEvent_t const* events,
                       uint8_t* train_ws = nullptr);

struct BwdPtrs {
    const void *q, *k, *v, *o, *dout;
    const float *lse, *theta;
    void *dq, *dk, *dv;
    float* dtheta;
    uint8_t* ws;
};

// TMA maps (window boxes) of the backward's token tensors.
struct BwdMaps {
    CUtensorMap q, k, v, o, dout, dq, dk, dv;
};

long long bwd_items(const Geo& g);
size_t bwd_workspace_bytes(const Geo& g);
// Offsets of the rotated q', k' tile images in the backward's workspace, and
// the launch that writes them (windows of >= 128 tokens).
void bwd_image_offsets(const Geo& g, size_t* qimg, size_t* kimg);
cudaError_t launch_rope_images(const Geo& g, const void* q, const void* k, const float* theta, uint8_t* ws,
                               cudaStream_t stream);
// events: NULL, or 5 events recorded before the first and after each of the
// four launches (prep, main, post, d theta; windows of fewer than 128 tokens
// run one kernel in the place of the first three).
// images_ready: the workspace already holds the q', k' images of these inputs
// (written by a training forward, windows of >= 128 tokens): prep skips them.
cudaError_t launch_bwd(const Geo& g, const BwdPtrs& p, const BwdMaps& maps, unsigned int* status,
                       unsigned long long limit_ns, int num_sms, cudaStream_t stream, cudaEvent_t const* events,
                       bool images_ready = false);

// Windows of fewer than 128 tokens (the tile holds whole windows): the whole
// backward of a tile in one kernel (d theta partials, 4 x 16 per (head, tile),
// into `part`), and the forward.
cudaError_t launch_small_bwd(const Geo& g, const BwdPtrs& p, float* part, unsigned int* dtheta_cnt,
                             unsigned int* status, unsigned long long limit_ns, int num_sms, cudaStream_t stream);
cudaError_t launch_small_fwd(const Geo& g, const void* q, const void* k, const void* v, const float* theta, void* o,
                             float* lse, unsigned int* status, unsigned long long limit_ns, int num_sms,
                             cudaStream_t stream);

// Heads of d = 64 channels, every window size (plain one-tile pipelines).  The
// backward's workspace holds an fp32 dQ' accumulator of 256 bytes per
// token-head row and the d theta partials.
size_t wide_bwd_workspace_bytes(const Geo& g);
// events: NULL, or (forward) 2 events recorded before and after the kernel,
// (backward) 5 events recorded before the first and after each of prep, main,
// post and the d theta sum.
cudaError_t launch_wide_fwd(const Geo& g, const void* q, const void* k, const void* v, const float* theta, void* o,
                            float* lse, unsigned int* status, unsigned long long limit_ns, int num_sms,
                            cudaStream_t stream, cudaEvent_t const* events);
cudaError_t launch_wide_bwd(const Geo& g, const BwdPtrs& p, unsigned int* status, unsigned long long limit_ns,
                            int num_sms, cudaStream_t stream, cudaEvent_t const* events);

// Windowed attention with a low-rank additive bias U_h W_h^T (heads of 32
// channels, every window size; theta may be null: no rotation, no d theta).
struct LrbPtrs {
    const void *q, *k, *v, *o, *dout;  // bf16 [B, H, W, heads, 32]
    const float *lse, *theta;           // theta: [heads][2][8] or null
    const float *u, *w;                 // [heads][M*M][16]
    void *o_out, *dq, *dk, *dv;         // o_out: the forward's O
    float *lse_out, *dtheta, *du, *dw;
    uint8_t* ws;
};
size_t lrbias_bwd_workspace_bytes(const Geo& g);
// events as for the 64-channel kernels (the backward's last mark follows the
// d theta and dU / dW sums).
cudaError_t launch_lrbias_fwd(const Geo& g, const LrbPtrs& p, unsigned int* status, unsigned long long limit_ns,
                              int num_sms, cudaStream_t stream, cudaEvent_t const* events);
cudaError_t launch_lrbias_bwd(const Geo& g, const LrbPtrs& p, unsigned int* status, unsigned long long limit_ns,
                              int num_sms, cudaStream_t stream, cudaEvent_t const* events);

// Fixed-order d theta sum: part [heads][per_head][16] -> dtheta [heads][16] (one
// launch; cnt: heads counters that are zero when it starts).
namespace bwdk {
cudaError_t launch_dtheta(const float* part, long long per_head, int heads, float* scratch, unsigned int* cnt,
                          float* dtheta, cudaStream_t stream);
}

// The attention block with its projections (inference), windows of fewer than
// 128 tokens, at most three heads: y = attention(x W_qkv^T + b_qkv) W_o^T + b_o.
struct BlockPtrs {
    const void *x, *w_qkv, *w_o;  // bf16 [B,H,W,C], [3C,C], [C,C]
    const float *b_qkv, *b_o, *theta;
    void* y;  // bf16 [B,H,W,C]
};
cudaError_t launch_block_fwd(const Geo& g, const BlockPtrs& p, unsigned int* status, unsigned long long limit_ns,
                             int num_sms, cudaStream_t stream);

}  // namespace fswin
