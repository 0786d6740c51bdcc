// C ABI of the library: argument validation, TMA descriptor encoding and
// kernel launches on the caller's stream.  Declared in include/fswin.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/fswin.h"
#include "geometry.cuh"
#include "kernels.cuh"
#include "ptx.cuh"


using namespace fswin;

namespace {

__device__ unsigned int g_status_word;

std::mutex g_mu;
unsigned long long g_limit_ns = 10ull * 1000 * 1000 * 1000;
constexpr int kMaxDev = 64;
unsigned int* g_status_ptr[kMaxDev] = {};
int g_num_sms[kMaxDev] = {};
int g_arch_ok[kMaxDev] = {};  // 0 unknown, 1 ok, -1 not sm_100
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
cudaEvent_t g_phase_events[8] = {};
int g_phase_n = 0;

fs_status device_state(unsigned int** status, int* num_sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return FS_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_arch_ok[dev] == 0) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return FS_ERR_CUDA;
        g_arch_ok[dev] = (major == 10 && minor == 0) ? 1 : -1;
        g_num_sms[dev] = sms;
    }
    if (g_arch_ok[dev] < 0) return FS_ERR_ARCH;
    if (!g_status_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return FS_ERR_CUDA;
        g_status_ptr[dev] = static_cast<unsigned int*>(p);
    }
    if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return FS_ERR_CUDA;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    *status = g_status_ptr[dev];
    *num_sms = g_num_sms[dev];
    return FS_OK;
}

fs_status make_geo(const fs_winattn_shape* sh, Geo* g) {
    if (!sh) return FS_ERR_NULL;
    return geo_init(g, sh->B, sh->H, sh->W, sh->heads, sh->d, sh->M, sh->s) ? FS_ERR_SHAPE : FS_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 5-D view [d, heads, W, H, B] of a bf16 [B, H, W, heads, d] tensor, box = one
// geometry box of one head, 64-byte swizzle (one 64-byte token row per line).
fs_status encode_box_map(CUtensorMap* m, const void* base, const Geo& g) {
    const cuuint64_t d = kHeadDim;
    cuuint64_t dims[5] = {d, static_cast<cuuint64_t>(g.heads), static_cast<cuuint64_t>(g.W),
                          static_cast<cuuint64_t>(g.H), static_cast<cuuint64_t>(g.B)};
    cuuint64_t strides[4] = {d * 2, d * 2 * g.heads, d * 2 * g.heads * g.W, d * 2 * g.heads * g.W * g.H};
    cuuint32_t box[5] = {static_cast<cuuint32_t>(d), 1, static_cast<cuuint32_t>(g.bw), static_cast<cuuint32_t>(g.bh),
                         1};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FS_OK : FS_ERR_CUDA;
}

__global__ void bounded_wait_selftest_kernel(unsigned int* status, unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const Ctl ctl{status, &abort_flag, limit_ns};
    // Nobody arrives on `bar`: the wait must give up after limit_ns and report.
    mbar_wait(&bar, 0, ctl, 0xABC);
    __syncthreads();
    if (threadIdx.x == 0) mbar_arrive(&bar);  // complete the phase before the CTA exits
}

__global__ void zero_f32_kernel(float* p, int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) p[i] = 0.f;
}

}  // namespace

int fswin::device_ready() {
    unsigned int* status = nullptr;
    int sms = 0;
    return static_cast<int>(device_state(&status, &sms));
}

extern "C" {

fs_status fs_winattn_check_shape(const fs_winattn_shape* shape) {
    Geo g;
    return make_geo(shape, &g);
}

const char* fs_status_string(fs_status st) {
    switch (st) {
        case FS_OK: return "FS_OK";
        case FS_ERR_NULL: return "FS_ERR_NULL: a required pointer is NULL";
        case FS_ERR_SHAPE: return "FS_ERR_SHAPE: unsupported or inconsistent shape";
        case FS_ERR_ALIGN: return "FS_ERR_ALIGN: a pointer is not 16-byte aligned";
        case FS_ERR_WORKSPACE: return "FS_ERR_WORKSPACE: workspace missing, misaligned or too small";
        case FS_ERR_CUDA: return "FS_ERR_CUDA: a CUDA call failed";
        case FS_ERR_TIMEOUT: return "FS_ERR_TIMEOUT: a device-side wait ran out of time";
        case FS_ERR_ARCH: return "FS_ERR_ARCH: the current device is not sm_100";
    }
    return "unknown fs_status";
}

}  // extern "C"

namespace {

// The forward; train_ws: NULL, or the backward's workspace (already checked),
// which then receives the rotated q', k' images for the training backward.
fs_status forward(const fs_winattn_shape* shape, const void* q, const void* k, const void* v, const float* theta,
                  void* o, float* lse, uint8_t* train_ws, fs_stream_t stream) {
    Geo g;
    fs_status st = make_geo(shape, &g);
    if (st != FS_OK) return st;
    if (g.B == 0) return FS_OK;
    if (!q || !k || !v || !theta || !o) return FS_ERR_NULL;  // lse may be NULL (inference)
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
        (reinterpret_cast<uintptr_t>(theta) & 3u) || (reinterpret_cast<uintptr_t>(lse) & 3u))
        return FS_ERR_ALIGN;
    unsigned int* status = nullptr;
    int sms = 0;
    if ((st = device_state(&status, &sms)) != FS_OK) return st;
    if (g.d == 64) {  // heads of 64 channels: the wide kernels (no tensor maps)
        unsigned long long lim;
        {
            std::lock_guard<std::mutex> lk(g_mu);
            lim = g_limit_ns;
        }
        const cudaError_t e = launch_wide_fwd(g, q, k, v, theta, o, lse, status, lim, sms,
                                              reinterpret_cast<cudaStream_t>(stream),
                                              g_phase_n >= 2 ? g_phase_events : nullptr);
        return e == cudaSuccess ? FS_OK : FS_ERR_CUDA;
    }
    CUtensorMap mq, mk, mv, mo;
    if (encode_box_map(&mq, q, g) || encode_box_map(&mk, k, g) || encode_box_map(&mv, v, g) ||
        encode_box_map(&mo, o, g))
        return FS_ERR_CUDA;
    unsigned long long lim;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        lim = g_limit_ns;
    }
    cudaError_t e = launch_fwd(g, mq, mk, mv, mo, q, k, v, o, theta, lse, status, lim, sms,
                               reinterpret_cast<cudaStream_t>(stream),
                               g_phase_n >= 2 ? g_phase_events : nullptr, g.N >= kTile ? train_ws : nullptr);
    return e == cudaSuccess ? FS_OK : FS_ERR_CUDA;
}

}  // namespace

extern "C" {

fs_status fs_winattn_fwd(const fs_winattn_shape* shape, const void* q, const void* k, const void* v,
                         const float* theta, void* o, float* lse, fs_stream_t stream) {
    return forward(shape, q, k, v, theta, o, lse, nullptr, stream);
}

fs_status fs_winattn_fwd_train(const fs_winattn_shape* shape, const void* q, const void* k, const void* v,
                               const float* theta, void* o, float* lse, void* workspace, size_t workspace_bytes,
                               fs_stream_t stream) {
    Geo g;
    fs_status st = make_geo(shape, &g);
    if (st != FS_OK) return st;
    if (g.B == 0) return FS_OK;
    if (!lse) return FS_ERR_NULL;  // the backward needs it
    const size_t need = g.d == 64 ? wide_bwd_workspace_bytes(g) : bwd_workspace_bytes(g);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need)
        return FS_ERR_WORKSPACE;
    return forward(shape, q, k, v, theta, o, lse, g.d == 32 ? static_cast<uint8_t*>(workspace) : nullptr, stream);
}

fs_status fs_winattn_block_fwd(const fs_winattn_shape* shape, const void* x, const void* w_qkv,
                               const float* b_qkv, const void* w_o, const float* b_o, const float* theta,
                               void* y, fs_stream_t stream) {
    Geo g;
    fs_status st = make_geo(shape, &g);
    if (st != FS_OK) return st;
    if (g.N >= kTile || g.heads > 3 || g.d != 32) return FS_ERR_SHAPE;  // windows inside one tile, C <= 96
    if (g.B == 0) return FS_OK;
    if (!x || !w_qkv || !b_qkv || !w_o || !b_o || !theta || !y) return FS_ERR_NULL;
    if (!aligned16(x) || !aligned16(w_qkv) || !aligned16(w_o) || !aligned16(y) ||
        (reinterpret_cast<uintptr_t>(b_qkv) & 3u) || (reinterpret_cast<uintptr_t>(b_o) & 3u) ||
        (reinterpret_cast<uintptr_t>(theta) & 3u))
        return FS_ERR_ALIGN;
    unsigned int* status = nullptr;
    int sms = 0;
    if ((st = device_state(&status, &sms)) != FS_OK) return st;
    unsigned long long lim;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        lim = g_limit_ns;
    }
    const BlockPtrs p{x, w_qkv, w_o, b_qkv, b_o, theta, y};
    const cudaError_t e = launch_block_fwd(g, p, status, lim, sms, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? FS_OK : FS_ERR_CUDA;
}

size_t fs_winattn_bwd_workspace_bytes(const fs_winattn_shape* shape) {
    Geo g;
    if (make_geo(shape, &g) != FS_OK) return 0;
    return g.d == 64 ? wide_bwd_workspace_bytes(g) : bwd_workspace_bytes(g);
}

}  // extern "C"

namespace {

fs_status backward(const fs_winattn_shape* shape, const void* q, const void* k, const void* v, const void* o,
                   const void* dout, const float* lse, const float* theta, void* dq, void* dk, void* dv,
                   float* dtheta, void* workspace, size_t workspace_bytes, bool images_ready, fs_stream_t stream) {
    Geo g;
    fs_status st = make_geo(shape, &g);
    if (st != FS_OK) return st;
    if (!theta || !dtheta) return FS_ERR_NULL;
    unsigned int* status = nullptr;
    int sms = 0;
    if (g.B == 0) {
        // Empty batch: gradients of theta are zero.
        if ((st = device_state(&status, &sms)) != FS_OK) return st;
        const int n = g.heads * 2 * (g.d / 4);
        zero_f32_kernel<<<(n + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(dtheta, n);
        return cudaGetLastError() == cudaSuccess ? FS_OK : FS_ERR_CUDA;
    }
    if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return FS_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(dq) ||
        !aligned16(dk) || !aligned16(dv) || (reinterpret_cast<uintptr_t>(lse) & 3u) ||
        (reinterpret_cast<uintptr_t>(theta) & 3u) || (reinterpret_cast<uintptr_t>(dtheta) & 3u))
        return FS_ERR_ALIGN;
    const size_t need = g.d == 64 ? wide_bwd_workspace_bytes(g) : bwd_workspace_bytes(g);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need)
        return FS_ERR_WORKSPACE;
    if ((st = device_state(&status, &sms)) != FS_OK) return st;
    if (g.d == 64) {  // heads of 64 channels: the wide kernels
        unsigned long long lim;
        {
            std::lock_guard<std::mutex> lk(g_mu);
            lim = g_limit_ns;
        }
        BwdPtrs p{q, k, v, o, dout, lse, theta, dq, dk, dv, dtheta, static_cast<uint8_t*>(workspace)};
        const cudaError_t e = launch_wide_bwd(g, p, status, lim, sms, reinterpret_cast<cudaStream_t>(stream),
                                              g_phase_n >= 5 ? g_phase_events : nullptr);
        return e == cudaSuccess ? FS_OK : FS_ERR_CUDA;
    }
    BwdMaps maps;
    if (encode_box_map(&maps.q, q, g) || encode_box_map(&maps.k, k, g) || encode_box_map(&maps.v, v, g) ||
        encode_box_map(&maps.o, o, g) || encode_box_map(&maps.dout, dout, g) || encode_box_map(&maps.dq, dq, g) ||
        encode_box_map(&maps.dk, dk, g) || encode_box_map(&maps.dv, dv, g))
        return FS_ERR_CUDA;
    unsigned long long lim;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        lim = g_limit_ns;
    }
    BwdPtrs p{q, k, v, o, dout, lse, theta, dq, dk, dv, dtheta, static_cast<uint8_t*>(workspace)};
    cudaError_t e = launch_bwd(g, p, maps, status, lim, sms, reinterpret_cast<cudaStream_t>(stream),
                               g_phase_n >= 5 ? g_phase_events : nullptr, images_ready);
    return e == cudaSuccess ? FS_OK : FS_ERR_CUDA;
}

}  // namespace

extern "C" {

fs_status fs_winattn_bwd(const fs_winattn_shape* shape, const void* q, const void* k, const void* v,
                         const void* o, const void* dout, const float* lse, const float* theta, void* dq,
                         void* dk, void* dv, float* dtheta, void* workspace, size_t workspace_bytes,
                         fs_stream_t stream) {
    return backward(shape, q, k, v, o, dout, lse, theta, dq, dk, dv, dtheta, workspace, workspace_bytes, false,
                    stream);
}

fs_status fs_winattn_bwd_train(const fs_winattn_shape* shape, const void* q, const void* k, const void* v,
                               const void* o, const void* dout, const float* lse, const float* theta, void* dq,
                               void* dk, void* dv, float* dtheta, void* workspace, size_t workspace_bytes,
                               fs_stream_t stream) {
    return backward(shape, q, k, v, o, dout, lse, theta, dq, dk, dv, dtheta, workspace, workspace_bytes, true,
                    stream);
}

fs_status fs_winattn_lrbias_fwd(const fs_winattn_shape* shape, const void* q, const void* k, const void* v,
                                const float* theta, const float* u, const float* w, int rank, void* o, float* lse,
                                fs_stream_t stream) {
    Geo g;
    fs_status st = make_geo(shape, &g);
    if (st != FS_OK) return st;
    if (g.d != 32 || rank != 16) return FS_ERR_SHAPE;
    if (g.B == 0) return FS_OK;
    if (!q || !k || !v || !u || !w || !o) return FS_ERR_NULL;  // theta and lse may be NULL
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(u) || !aligned16(w) ||
        (reinterpret_cast<uintptr_t>(theta) & 3u) || (reinterpret_cast<uintptr_t>(lse) & 3u))
        return FS_ERR_ALIGN;
    unsigned int* status = nullptr;
    int sms = 0;
    if ((st = device_state(&status, &sms)) != FS_OK) return st;
    unsigned long long lim;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        lim = g_limit_ns;
    }
    LrbPtrs p{};
    p.q = q;
    p.k = k;
    p.v = v;
    p.theta = theta;
    p.u = u;
    p.w = w;
    p.o_out = o;
    p.lse_out = lse;
    const cudaError_t e = launch_lrbias_fwd(g, p, status, lim, sms, reinterpret_cast<cudaStream_t>(stream),
                                            g_phase_n >= 2 ? g_phase_events : nullptr);
    return e == cudaSuccess ? FS_OK : FS_ERR_CUDA;
}

size_t fs_winattn_lrbias_bwd_workspace_bytes(const fs_winattn_shape* shape) {
    Geo g;
    if (make_geo(shape, &g) != FS_OK || g.d != 32) return 0;
    return lrbias_bwd_workspace_bytes(g);
}

fs_status fs_winattn_lrbias_bwd(const fs_winattn_shape* shape, const void* q, const void* k, const void* v,
                                const void* o, const void* dout, const float* lse, const float* theta,
                                const float* u, const float* w, int rank, void* dq, void* dk, void* dv,
                                float* dtheta, float* du, float* dw, void* workspace, size_t workspace_bytes,
                                fs_stream_t stream) {
    Geo g;
    fs_status st = make_geo(shape, &g);
    if (st != FS_OK) return st;
    if (g.d != 32 || rank != 16) return FS_ERR_SHAPE;
    if (!du || !dw || (theta && !dtheta)) return FS_ERR_NULL;
    if (!aligned16(du) || !aligned16(dw) || (reinterpret_cast<uintptr_t>(dtheta) & 3u)) return FS_ERR_ALIGN;
    unsigned int* status = nullptr;
    int sms = 0;
    const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    if (g.B == 0) {
        // Empty batch: the parameter gradients are empty sums.
        if ((st = device_state(&status, &sms)) != FS_OK) return st;
        const int nb = g.heads * g.N * 16;
        zero_f32_kernel<<<(nb + 255) / 256, 256, 0, cs>>>(du, nb);
        zero_f32_kernel<<<(nb + 255) / 256, 256, 0, cs>>>(dw, nb);
        if (theta) zero_f32_kernel<<<(g.heads * 16 + 255) / 256, 256, 0, cs>>>(dtheta, g.heads * 16);
        return cudaGetLastError() == cudaSuccess ? FS_OK : FS_ERR_CUDA;
    }
    if (!q || !k || !v || !o || !dout || !lse || !u || !w || !dq || !dk || !dv) return FS_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(dq) ||
        !aligned16(dk) || !aligned16(dv) || !aligned16(u) || !aligned16(w) ||
        (reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(theta) & 3u))
        return FS_ERR_ALIGN;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
        workspace_bytes < lrbias_bwd_workspace_bytes(g))
        return FS_ERR_WORKSPACE;
    if ((st = device_state(&status, &sms)) != FS_OK) return st;
    unsigned long long lim;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        lim = g_limit_ns;
    }
    LrbPtrs p{};
    p.q = q;
    p.k = k;
    p.v = v;
    p.o = o;
    p.dout = dout;
    p.lse = lse;
    p.theta = theta;
    p.u = u;
    p.w = w;
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    p.dtheta = theta ? dtheta : nullptr;
    p.du = du;
    p.dw = dw;
    p.ws = static_cast<uint8_t*>(workspace);
    const cudaError_t e = launch_lrbias_bwd(g, p, status, lim, sms, cs, g_phase_n >= 5 ? g_phase_events : nullptr);
    return e == cudaSuccess ? FS_OK : FS_ERR_CUDA;
}

fs_status fs_device_status(unsigned int* code) {
    if (!code) return FS_ERR_NULL;
    unsigned int* status = nullptr;
    int sms = 0;
    fs_status st = device_state(&status, &sms);
    if (st != FS_OK) return st;
    unsigned int v = 0;
    if (cudaMemcpy(&v, status, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return FS_ERR_CUDA;
    const unsigned int zero = 0;
    if (cudaMemcpy(status, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess) return FS_ERR_CUDA;
    *code = v;
    return FS_OK;
}

fs_status fs_set_phase_events(void* const* events, int n) {
    if (n < 0 || n > 8) return FS_ERR_SHAPE;
    if (n > 0 && !events) return FS_ERR_NULL;
    for (int i = 0; i < n; ++i)
        if (!events[i]) return FS_ERR_NULL;
    for (int i = 0; i < 8; ++i) g_phase_events[i] = i < n ? static_cast<cudaEvent_t>(events[i]) : nullptr;
    g_phase_n = n;
    return FS_OK;
}

fs_status fs_set_wait_limit_ns(uint64_t limit_ns) {
    if (limit_ns == 0) return FS_ERR_SHAPE;
    std::lock_guard<std::mutex> lk(g_mu);
    g_limit_ns = limit_ns;
    return FS_OK;
}

fs_status fs_selftest_bounded_wait(uint64_t limit_ns, fs_stream_t stream) {
    unsigned int* status = nullptr;
    int sms = 0;
    fs_status st = device_state(&status, &sms);
    if (st != FS_OK) return st;
    bounded_wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(status, limit_ns);
    return cudaGetLastError() == cudaSuccess ? FS_OK : FS_ERR_CUDA;
}

}  // extern "C"
