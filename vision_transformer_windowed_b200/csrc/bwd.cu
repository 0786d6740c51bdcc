// Backward of fused shifted-window attention with window-local 2D RoPE.
//
// Recompute-based (the probabilities are rebuilt from the forward's
// log-sum-exp, never stored), in five launches on the caller's stream:
//   1. prep:   per token row, rotate q and k (RoPE) into swizzled fp16 tile
//              images, D = rowsum(dO * O), lse in log2 units, and zero the
//              fp32 dQ accumulator; per tile, the largest |dO row| and |v row|;
//      scale:  per window, the gradient scaling 2^e from those maxima (see
//              grad_scale_exp in rows.cuh): lse2 -= e, so that the main kernel's
//              probabilities, dS and dV carry 2^e;
//   2. main:   persistent, warp-specialised tcgen05 kernel; a work item is one
//              128-key tile, iterating over the query tiles it attends to:
//                S^T = K' Q'^T, dP^T = V dO^T            (TMEM)
//                P^T = exp2(S^T * c - lse2), dS^T = P^T (dP^T - D)
//                dV += P^T dO, dK' += dS^T Q'            (TMEM accumulators)
//                dQ' = dS K'  -> bulk reduce-add into the fp32 accumulator
//              and, per item, dk (dK' un-rotated) and dv, with the key side
//              of d theta (2^-e undoes the scaling of dQ', dK', dV);
//   3. post:   per token row, undo the rotation of dQ', write dq, and the
//              query side of d theta;
//   4. reduce: fixed-order sum of the partials into dtheta (it adds no
//              run-to-run variation; the query-side partials carry that of
//              dQ', whose reduce-adds land in any order).
#include <cuda.h>
#include <cuda_runtime.h>

#include "geometry.cuh"
#include "kernels.cuh"
#include "ptx.cuh"
#include "schedule.cuh"
#include "tile_io.cuh"
#include "dgeo.cuh"
#include "rows.cuh"

namespace fswin {

namespace bwdk {

// ------------------------------------------------------------------ workspace
struct WsLayout {
    size_t qimg, kimg, lse2, dvec, dqacc, nrm, wexp, part, part2, cnt, total;
};

__host__ __device__ inline size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

__host__ __device__ inline WsLayout ws_layout(const Geo& g) {
    const size_t ht = static_cast<size_t>(g.heads) * static_cast<size_t>(g.tiles);
    WsLayout L;
    size_t o = 0;
    L.qimg = o;  o += round256(ht * kTileBytes);
    L.kimg = o;  o += round256(ht * kTileBytes);
    L.lse2 = o;  o += round256(ht * kTile * 4);
    L.dvec = o;  o += round256(ht * kTile * 4);
    L.dqacc = o; o += round256(ht * kTile * kHeadDim * 4);
    L.nrm = o;   o += round256(ht * 8);  // per (head, tile): max |dO row|^2, max |v row|^2
    L.wexp = o;  o += round256(ht * 4);  // per (head, tile): e of the tile's window
    L.part = o;  o += round256(ht * 8 * 16 * 4);  // up to 8 x 16 partials per (head, tile)
    L.part2 = o; o += round256(static_cast<size_t>(g.heads) * 64 * 16 * 4);  // level-1 d theta sums
    L.cnt = o;   o += round256(static_cast<size_t>(g.heads) * 4);            // level-1 blocks done, per head
    L.total = o;
    return L;
}

// What a prep launch does: everything (the backward on its own); only the
// rotated q', k' images (the training forward, which reads them); everything
// but the images (the backward after such a forward, whose images are still
// in the workspace).
enum PrepMode : int { kPrepFull = 0, kPrepImages = 1, kPrepReuse = 2 };

struct PrepParams {
    Geo g;
    const uint4 *q, *k, *v, *o, *dout;
    const float *lse, *theta;
    uint8_t* ws;
    WsLayout L;
    int mode;
};

struct PostParams {
    Geo g;  // windows of >= 128 tokens
    const uint4* q;
    const float* theta;
    uint4* dq;
    const uint8_t* ws;
    WsLayout L;
    float scale;
};

// cos/sin of pos * theta[h][ax][k] for pos < M, in shared memory: [2][64][8],
// built by threads t < nt.
__device__ __forceinline__ void build_table(float2* tab, const float* theta_h, int M, int t, int nt) {
    for (int e = t; e < 2 * M * 8; e += nt) {
        const int ax = e / (M * 8), rem = e - ax * M * 8, pos = rem >> 3, k = rem & 7;
        float sn, cs;
        sincosf(static_cast<float>(pos) * theta_h[ax * 8 + k], &sn, &cs);
        tab[(ax * 64 + pos) * 8 + k] = make_float2(cs, sn);
    }
}

// Rotate (inv = false) or un-rotate (inv = true) 32 channel values of a token
// at in-window position (i, j).
__device__ __forceinline__ void rope32(float (&x)[32], int i, int j, const float2* tab, bool inv) {
#pragma unroll
    for (int ax = 0; ax < 2; ++ax) {
        const float2* t = tab + (ax * 64 + (ax ? i : j)) * 8;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const float2 cs = t[k];
            const float sn = inv ? -cs.y : cs.y;
            const float a = x[ax * 16 + 2 * k], b = x[ax * 16 + 2 * k + 1];
            x[ax * 16 + 2 * k] = a * cs.x - b * sn;
            x[ax * 16 + 2 * k + 1] = a * sn + b * cs.x;
        }
    }
}

__device__ __forceinline__ void load_row_bf16(const uint4* src, float (&x)[32]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint4 v = src[c];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            x[8 * c + 2 * e] = bf16lo_to_f32(w[e]);
            x[8 * c + 2 * e + 1] = bf16hi_to_f32(w[e]);
        }
    }
}

// ------------------------------------------------------------------ 1. prep
__global__ void __launch_bounds__(128) prep_kernel(const PrepParams p) {
    __shared__ float2 tab[2 * 64 * 8];
    __shared__ float2 nrm_w[4];
    const Geo& g = p.g;
    const bool images = p.mode != kPrepReuse, extras = p.mode != kPrepImages;  // uniform over the launch
    // blocks take the heads of a tile in turn (a token's heads share memory
    // lines); ht indexes the workspace images, [head][tile]
    const long long T = blockIdx.x / g.heads;
    const int h = static_cast<int>(blockIdx.x - T * g.heads);
    const long long ht = static_cast<long long>(h) * g.tiles + T;
    if (extras && blockIdx.x == 0)  // the d theta reduction's counters, for its launch after this one
        for (int i = threadIdx.x; i < g.heads; i += blockDim.x) reinterpret_cast<unsigned int*>(p.ws + p.L.cnt)[i] = 0u;
    if (images) {
        build_table(tab, p.theta + h * 16, g.M, threadIdx.x, blockDim.x);
        __syncthreads();
    }
    const int r = threadIdx.x;
    const Slot sl = slot_of(g, T, r);
    float q[32], k[32], dO[32], o[32];
    float D = 0.f, lse2 = INFINITY, ndo = 0.f, nv = 0.f;
    if (sl.valid) {
        const long long tok = ((static_cast<long long>(sl.box.b) * g.H + sl.row) * g.W + sl.col) * g.heads + h;
        if (images) {
            load_row_bf16(p.q + tok * 4, q);
            load_row_bf16(p.k + tok * 4, k);
            rope32(q, sl.i, sl.j, tab, false);
            rope32(k, sl.i, sl.j, tab, false);
        }
        if (extras) {
            load_row_bf16(p.dout + tok * 4, dO);
            load_row_bf16(p.o + tok * 4, o);
            float acc[4] = {0.f, 0.f, 0.f, 0.f}, n4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                acc[e & 3] = fmaf(dO[e], o[e], acc[e & 3]);
                n4[e & 3] = fmaf(dO[e], dO[e], n4[e & 3]);
            }
            D = (acc[0] + acc[1]) + (acc[2] + acc[3]);
            ndo = (n4[0] + n4[1]) + (n4[2] + n4[3]);
            load_row_bf16(p.v + tok * 4, o);  // o is done with: v's row
#pragma unroll
            for (int e = 0; e < 4; ++e) n4[e] = 0.f;
#pragma unroll
            for (int e = 0; e < 32; ++e) n4[e & 3] = fmaf(o[e], o[e], n4[e & 3]);
            nv = (n4[0] + n4[1]) + (n4[2] + n4[3]);
            lse2 = p.lse[tok] * 1.4426950408889634f;
        }
    } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) q[e] = k[e] = 0.f;
    }
    if (images) {
        store_row_swz(p.ws + p.L.qimg + ht * kTileBytes, r, q, true);
        store_row_swz(p.ws + p.L.kimg + ht * kTileBytes, r, k, true);
    }
    if (!extras) return;
    reinterpret_cast<float*>(p.ws + p.L.lse2)[ht * kTile + r] = lse2;
    reinterpret_cast<float*>(p.ws + p.L.dvec)[ht * kTile + r] = D;
    uint4* acc = reinterpret_cast<uint4*>(p.ws + p.L.dqacc + (ht * kTile + r) * kHeadDim * 4);
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = make_uint4(0, 0, 0, 0);
    // the tile's largest squared norms of dO and v rows
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        ndo = fmaxf(ndo, __shfl_xor_sync(0xFFFFFFFFu, ndo, o));
        nv = fmaxf(nv, __shfl_xor_sync(0xFFFFFFFFu, nv, o));
    }
    if ((r & 31) == 0) nrm_w[r >> 5] = make_float2(ndo, nv);
    __syncthreads();
    if (r == 0)
        reinterpret_cast<float2*>(p.ws + p.L.nrm)[ht] =
            make_float2(fmaxf(fmaxf(nrm_w[0].x, nrm_w[1].x), fmaxf(nrm_w[2].x, nrm_w[3].x)),
                        fmaxf(fmaxf(nrm_w[0].y, nrm_w[1].y), fmaxf(nrm_w[2].y, nrm_w[3].y)));
}

// ------------------------------------------------------------------ 1b. scale
// One block per (head, window) of >= 128 tokens: the gradient scaling exponent
// e of the window from its tiles' largest |dO row|^2 and |v row|^2 (every row
// of the window: a key tile's products reach all of the window's queries, and
// D_t = dO_t . O_t mixes all of its v rows), lse2 -= e for the window's rows,
// and e kept for each of its tiles (per tile, so that the workspace does not
// depend on the window size).
__global__ void __launch_bounds__(128) scale_kernel(const Geo g, uint8_t* ws, const WsLayout L) {
    const long long hw = blockIdx.x;  // head-major: h * wins + window
    const int h = static_cast<int>(hw / g.wins);
    const long long w = hw - static_cast<long long>(h) * g.wins;
    const size_t t0 = static_cast<size_t>(h) * g.tiles + static_cast<size_t>(w) * g.tpw;
    const float2* nrm = reinterpret_cast<const float2*>(ws + L.nrm) + t0;
    float a = 0.f, b = 0.f;
    for (int i = 0; i < g.tpw; ++i) {
        const float2 t = nrm[i];
        a = fmaxf(a, t.x);
        b = fmaxf(b, t.y);
    }
    const int e = grad_scale_exp(a, b);
    float* lse2 = reinterpret_cast<float*>(ws + L.lse2) + t0 * kTile;
    for (int i = threadIdx.x; i < g.tpw * kTile; i += blockDim.x) lse2[i] -= static_cast<float>(e);
    for (int i = threadIdx.x; i < g.tpw; i += blockDim.x) reinterpret_cast<int*>(ws + L.wexp)[t0 + i] = e;
}

// ------------------------------------------------------------------ 2. main
// A work item is one 128-key tile u and the query tiles of its window that
// attend it; a step is one (u, query tile) pair, done in two half-steps of 64
// queries.  Per half-step h (counter hc, TMEM buffer b = hc & 1):
//   MMA warp:      S^T_h = K' Q'_h^T and dP^T_h = V dO_h^T (N = 64) into buffer b
//   compute warps: P^T = exp2(S^T c - lse2), dS^T = P^T (dP^T - D) into the
//                  buffer's P^T, dS^T columns, and dS into shared memory
//   MMA warp:      dV += P^T dO_h, dK' += dS^T Q'_h; after both halves
//                  dQ' = dS K' (a double-buffered accumulator); then the
//                  S^T, dP^T of the half-step two ahead into the same buffer
// so the compute warps work on one buffer while the tensor core fills the
// other and never wait for the previous gradients.
//   epilogue warps: dQ' of each step to the fp32 accumulator (bulk
//                   reduce-add); at the end of each item dk (dK' un-rotated),
//                   the key side of d theta, and dv (TMA stores).
constexpr int kThreads = 448;
constexpr int kQStages = 3;
constexpr int kWarpTma = 12, kWarpMma = 13;  // warps 0-7: P/dS, 8-11: epilogue

constexpr int kQStageBytes = 2 * kTileBytes + 2 * kTile * 4;  // Q', dO, lse2, D
constexpr int kKVOff = 0;                                      // 2 slots x (K', V)
constexpr int kQOff = kKVOff + 2 * 2 * kTileBytes;
constexpr int kDSOff = kQOff + kQStages * kQStageBytes;        // 2 x dS, MN-major 128B swizzle
constexpr int kDSBytes = 4 * kTileBytes;
constexpr int kDQStOff = kDSOff + 2 * kDSBytes;                // 2 x fp32 [128][32]
constexpr int kDKStOff = kDQStOff + 2 * 4 * kTile * kHeadDim;  // bf16 tile
constexpr int kTabOff = kDKStOff + kTileBytes;                  // cos / sin [2][64][8]
constexpr int kDVStOff = kTabOff + 2 * 64 * 8 * 8;              // bf16 tile
constexpr int kBarOff = kDVStOff + kTileBytes;
constexpr int kSmemBytes = kBarOff + 1024 + 1024;
static_assert(kDSOff % 1024 == 0, "128-byte swizzled operand must be 1024-byte aligned");

// TMEM columns (all 512): half-step buffer b: S^T at 128 b, dP^T at 128 b + 64
// (64 columns each); its P^T (bf16) at 256 + 64 b and dS^T (fp16) at
// 256 + 64 b + 32 (32 columns each, 8 per K step of 16 queries), apart from
// S^T and dP^T, so that the next S^T, dP^T of the buffer never overwrite what
// pending gradient MMAs read; dQ' accumulators at 384 + 32 c (step parity c);
// dV at 448, dK' at 480.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColDQ = 384, kColDV = 448, kColDK = 480;
__device__ __forceinline__ uint32_t col_buf(uint32_t b) { return 128u * b; }
__device__ __forceinline__ uint32_t col_pb(uint32_t b) { return 256u + 64u * b; }

struct Bars {
    uint64_t kv_full[2], kv_empty[2];
    uint64_t q_full[kQStages], q_empty[kQStages];
    uint64_t s_full[2], p_full[2];
    uint64_t dq_full[2], dq_free[2], dkv_full, dkv_free;
    uint64_t done;
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Bars) <= 1024, "barrier block overflows its slot");

struct MainParams {
    Geo g;
    uint8_t* ws;
    WsLayout L;
    const float* theta;
    float* part;  // [heads][tiles][8][16] d theta partials
    unsigned int* status;
    unsigned long long limit_ns;
    long long items;
    float scale;
};

using Item = BwdItem;
__device__ __forceinline__ Item item_of(const Geo& g, long long it) { return d_bwd_item(g, it); }
__device__ __forceinline__ bool q_active(const Geo& g, const Item& I, int n) { return bwd_active(g, I, n); }

__global__ void __launch_bounds__(kThreads, 1)
    main_kernel(const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_dv,
                const __grid_constant__ CUtensorMap map_do, const __grid_constant__ CUtensorMap map_dk,
                const __grid_constant__ MainParams prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars* bars = reinterpret_cast<Bars*>(smem + kBarOff);
    const Geo& g = prm.g;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t tiles = static_cast<size_t>(g.tiles);

    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->kv_full[i], 1);
            mbar_init(&bars->kv_empty[i], 5);  // the item's last MMAs, and each epilogue warp's read of its k' rows
            mbar_init(&bars->s_full[i], 1);
            mbar_init(&bars->p_full[i], 8);
            mbar_init(&bars->dq_full[i], 1);
            mbar_init(&bars->dq_free[i], 4);
        }
        for (int i = 0; i < kQStages; ++i) {
            mbar_init(&bars->q_full[i], 1);
            mbar_init(&bars->q_empty[i], 1);
        }
        mbar_init(&bars->dkv_full, 1);
        mbar_init(&bars->dkv_free, 4);
        mbar_init(&bars->done, 1);
        bars->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&bars->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const Ctl ctl{prm.status, &bars->abort_flag, prm.limit_ns};
    const uint8_t* ws = prm.ws;

    if (warp == kWarpTma) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&map_v);
            prefetch_tmap(&map_do);
            int it = 0;
            uint32_t qc = 0;
            bool ok = true;
            for (long long item = blockIdx.x; item < prm.items && ok; item += gridDim.x, ++it) {
                const Item I = item_of(g, item);
                const int ks = it & 1;
                if (!mbar_wait(&bars->kv_empty[ks], ((it >> 1) & 1) ^ 1, ctl, 0x1101)) break;
                uint8_t* kv = smem + kKVOff + ks * 2 * kTileBytes;
                const size_t hu = static_cast<size_t>(I.h) * tiles + static_cast<size_t>(I.u);
                mbar_arrive_expect_tx(&bars->kv_full[ks], 2 * kTileBytes);
                bulk_load(kv, ws + prm.L.kimg + hu * kTileBytes, kTileBytes, &bars->kv_full[ks]);
                tile_tma(g, &map_v, kv + kTileBytes, &bars->kv_full[ks], I.u, I.h, false);
                for (int n = 0; n < I.nq; ++n) {
                    if (!q_active(g, I, n)) continue;
                    const int st = qc % kQStages;
                    const uint32_t ph = (qc / kQStages) & 1;
                    ++qc;
                    if (!mbar_wait(&bars->q_empty[st], ph ^ 1, ctl, 0x1102)) { ok = false; break; }
                    uint8_t* qs = smem + kQOff + st * kQStageBytes;
                    const size_t hv = static_cast<size_t>(I.h) * tiles + static_cast<size_t>(I.q0 + n);
                    mbar_arrive_expect_tx(&bars->q_full[st], kQStageBytes);
                    bulk_load(qs, ws + prm.L.qimg + hv * kTileBytes, kTileBytes, &bars->q_full[st]);
                    tile_tma(g, &map_do, qs + kTileBytes, &bars->q_full[st], I.q0 + n, I.h, false);
                    bulk_load(qs + 2 * kTileBytes, ws + prm.L.lse2 + hv * kTile * 4, kTile * 4, &bars->q_full[st]);
                    bulk_load(qs + 2 * kTileBytes + kTile * 4, ws + prm.L.dvec + hv * kTile * 4, kTile * 4,
                              &bars->q_full[st]);
                }
            }
        }
    } else if (warp == kWarpMma) {
        // ------------------------------------------------------------ MMA issue
        if (lane == 0) {
            // operand types: Q', K', dS in fp16; V, dO, P in bf16
            const uint32_t id_s = make_idesc(kTile, 64, false, false, true);
            const uint32_t id_dp = make_idesc(kTile, 64, false, false, false);
            const uint32_t id_dv = make_idesc(kTile, kHeadDim, false, true, false);
            const uint32_t id_dk = make_idesc(kTile, kHeadDim, false, true, true);
            const uint32_t id_dq = make_idesc(kTile, kHeadDim, true, true, true);
            // cursor over this CTA's steps: items and their attending query tiles
            struct Step {
                bool valid, first, last;
                int it, ks, st;
                uint32_t qph;
            };
            long long c_item = blockIdx.x;
            int c_it = 0, c_n = -1;
            uint32_t c_qc = 0;
            bool c_loaded = false;
            Item CI{};
            auto next_step = [&]() -> Step {
                Step s{};
                while (c_item < prm.items) {
                    if (!c_loaded) {
                        CI = item_of(g, c_item);
                        c_loaded = true;
                        c_n = -1;
                    }
                    int n = c_n + 1;
                    while (n < CI.nq && !q_active(g, CI, n)) ++n;
                    if (n < CI.nq) {
                        int n2 = n + 1;
                        while (n2 < CI.nq && !q_active(g, CI, n2)) ++n2;
                        s.valid = true;
                        s.first = c_n < 0;
                        s.last = n2 >= CI.nq;
                        s.it = c_it;
                        s.ks = c_it & 1;
                        s.st = static_cast<int>(c_qc % kQStages);
                        s.qph = (c_qc / kQStages) & 1;
                        ++c_qc;
                        c_n = n;
                        return s;
                    }
                    c_loaded = false;  // item done
                    c_item += gridDim.x;
                    ++c_it;
                }
                return s;
            };
            auto wait_inputs = [&](const Step& s) -> bool {
                if (s.first && !mbar_wait(&bars->kv_full[s.ks], (s.it >> 1) & 1, ctl, 0x1302)) return false;
                return mbar_wait(&bars->q_full[s.st], s.qph, ctl, 0x1303);
            };
            // Shared-memory descriptors built once per layout; per MMA only an offset
            // in 16-byte units is added to the start-address field (14 bits: every
            // offset of this kernel stays below 256 KiB).
            const uint32_t sbase = smem_u32(smem);
            const uint64_t dK0 = make_sdesc(sbase, 16, 512, kSw64);       // K-major, 64-byte rows
            const uint64_t dMN0 = make_sdesc(sbase, 8192, 512, kSw64);    // MN-major, 64-byte rows
            const uint64_t dDS0 = make_sdesc(sbase, 16384, 1024, kSw128); // dS, MN-major, 128-byte rows
            auto u16 = [](uint32_t bytes) { return static_cast<uint64_t>(bytes >> 4); };
            // S^T_h = K' Q'_h^T and dP^T_h = V dO_h^T into buffer b
            auto issue_sdp = [&](const Step& s, int h, uint32_t b) {
                const uint64_t ko = u16(kKVOff + s.ks * 2 * kTileBytes), vo = ko + u16(kTileBytes);
                const uint64_t qo = u16(kQOff + s.st * kQStageBytes + 4096u * h), dof = qo + u16(kTileBytes);
                const uint32_t t_b = tmem + col_buf(b);
#pragma unroll
                for (int k = 0; k < kHeadDim / 16; ++k) umma_ss(t_b, dK0 + ko + 2 * k, dK0 + qo + 2 * k, id_s, k > 0);
#pragma unroll
                for (int k = 0; k < kHeadDim / 16; ++k)
                    umma_ss(t_b + 64, dK0 + vo + 2 * k, dK0 + dof + 2 * k, id_dp, k > 0);
                umma_commit(&bars->s_full[b]);
            };
            // dV += P^T_h dO_h, dK' += dS^T_h Q'_h (the item's first half-step starts them)
            auto issue_grads = [&](const Step& s, int h, uint32_t b) {
                const uint64_t qo = u16(kQOff + s.st * kQStageBytes + 4096u * h), dof = qo + u16(kTileBytes);
                const uint32_t t_p = tmem + col_pb(b);
                const uint32_t acc = (s.first && h == 0) ? 0u : 1u;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    umma_ts(tmem + kColDV, t_p + 8 * k, dMN0 + dof + 64 * k, id_dv, k > 0 ? 1u : acc);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    umma_ts(tmem + kColDK, t_p + 32 + 8 * k, dMN0 + qo + 64 * k, id_dk, k > 0 ? 1u : acc);
            };
            // dQ' = dS K' of a step into accumulator c
            auto issue_dq = [&](const Step& s, uint32_t c) {
                const uint64_t ko = u16(kKVOff + s.ks * 2 * kTileBytes);
                const uint64_t so = u16(kDSOff + c * kDSBytes);
#pragma unroll
                for (int k = 0; k < kTile / 16; ++k)
                    umma_ss(tmem + kColDQ + 32 * c, dDS0 + so + 128 * k, dMN0 + ko + 64 * k, id_dq, k > 0);
                umma_commit(&bars->dq_full[c]);
            };
            bool ok = true;
            Step cur = next_step();
            if (cur.valid) {
                ok = wait_inputs(cur);
                if (ok) {
                    tc_fence_after();
                    issue_sdp(cur, 0, 0);
                    issue_sdp(cur, 1, 1);
                }
            }
            uint32_t hc = 0, dkvph = 0;
            long long j = 0;  // steps done
            while (ok && cur.valid) {
                const Step nxt = next_step();
                bool nxt_ready = false;
                for (int h = 0; h < 2; ++h, ++hc) {
                    const uint32_t b = hc & 1u;
                    if (!mbar_wait(&bars->p_full[b], (hc >> 1) & 1u, ctl, 0x1304)) { ok = false; break; }
                    if (h == 0 && cur.first && cur.it > 0) {  // the epilogue has read the previous item's dV, dK'
                        if (!mbar_wait(&bars->dkv_free, dkvph, ctl, 0x1305)) { ok = false; break; }
                        dkvph ^= 1;
                    }
                    tc_fence_after();
                    issue_grads(cur, h, b);
                    if (h == 1) {
                        const uint32_t c = static_cast<uint32_t>(j & 1);
                        if (j >= 2 && !mbar_wait(&bars->dq_free[c], ((j >> 1) & 1) ^ 1, ctl, 0x1306)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        issue_dq(cur, c);
                        umma_commit(&bars->q_empty[cur.st]);
                        if (cur.last) {
                            umma_commit(&bars->dkv_full);
                            umma_commit(&bars->kv_empty[cur.ks]);
                        }
                        ++j;
                    }
                    // the half-step two ahead into the same S^T, dP^T buffer (the
                    // gradients read P^T, dS^T from their own columns)
                    if (nxt.valid) {
                        if (!nxt_ready) {
                            if (!wait_inputs(nxt)) { ok = false; break; }
                            nxt_ready = true;
                            tc_fence_after();
                        }
                        issue_sdp(nxt, h, b);
                    }
                }
                cur = nxt;
            }
            umma_commit(&bars->done);
            mbar_wait(&bars->done, 0, ctl, 0x13ff);
        }
        __syncwarp();
    } else if (warp < 8) {
        // ------------------------------------------------------------ P^T, dS^T (thread = key row)
        const int cw = warp >> 2;  // 32-column chunk of the 64-query half-step
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const float sl2 = g.scale_log2;
        uint32_t hc = 0, qc = 0;
        long long j = 0;
        bool ok = true;
        for (long long item = blockIdx.x; item < prm.items && ok; item += gridDim.x) {
            const Item I = item_of(g, item);
            const uint32_t keyseg = I.masked ? seg_at(d_tile_segs(g, I.u, I.win), r >> g.lBT) : 0u;
            for (int n = 0; n < I.nq && ok; ++n) {
                if (!q_active(g, I, n)) continue;
                const int st = qc % kQStages;
                ++qc;
                const float* lse2 = reinterpret_cast<const float*>(smem + kQOff + st * kQStageBytes + 2 * kTileBytes);
                const float* dvec = lse2 + kTile;
                uint8_t* ds = smem + kDSOff + (j & 1) * kDSBytes;
                // bit c: query columns [16 c, 16 c + 16) attend this key row
                // every 16-column group attends unless the window is cut by the mask
                const uint32_t a16 = I.masked ? d_allow16(g, keyseg, I.q0 + n, I.win) : 0xFFu;
                for (int h = 0; h < 2; ++h, ++hc) {
                    const uint32_t b = hc & 1u;
                    const int col0 = 64 * h + 32 * cw;  // this thread's 32 query columns
                    const uint32_t tc = tmem + lane_off + col_buf(b) + 32 * cw;  // S^T chunk; dP^T chunk at +64
                    const uint32_t tp = tmem + lane_off + col_pb(b) + 16 * cw;   // P^T chunk; dS^T chunk at +32
                    uint8_t* base = ds + h * 16384 + (r >> 3) * 1024 + (r & 7) * 128;
                    if (!__all_sync(0xFFFFFFFFu, mbar_wait(&bars->s_full[b], (hc >> 1) & 1u, ctl, 0x1401))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t grp2 = (a16 >> (col0 >> 4)) & 3u;
                    if (!__any_sync(0xFFFFFFFFu, grp2 != 0u)) {  // no key row of the warp attends these queries
                        const uint32_t z[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                        tmem_st16(tp, z);
                        tmem_st16(tp + 32, z);
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4)
                            *reinterpret_cast<uint4*>(base + (((4 * cw + q4) ^ (r & 7)) << 4)) = make_uint4(0, 0, 0, 0);
                    } else {
                        uint32_t sv[32], pv[32];
                        tmem_ld32(tc, sv);
                        tmem_ld32(tc + 64, pv);
                        tmem_wait_ld();
                        const bool ok0 = grp2 & 1u, ok1 = (grp2 >> 1) & 1u;
                        uint32_t wp[16], wd[16];
#pragma unroll
                        for (int e4 = 0; e4 < 8; ++e4) {
                            float4 L4 = *reinterpret_cast<const float4*>(lse2 + col0 + 4 * e4);
                            const float4 D4 = *reinterpret_cast<const float4*>(dvec + col0 + 4 * e4);
                            if (!(e4 < 4 ? ok0 : ok1)) L4 = make_float4(INFINITY, INFINITY, INFINITY, INFINITY);
                            const int e = 4 * e4;
                            float t0, t1, t2, t3;
                            ffma2(t0, t1, __uint_as_float(sv[e]), __uint_as_float(sv[e + 1]), sl2, sl2, -L4.x, -L4.y);
                            ffma2(t2, t3, __uint_as_float(sv[e + 2]), __uint_as_float(sv[e + 3]), sl2, sl2, -L4.z,
                                  -L4.w);
                            const float p0 = ex2_approx(t0), p1 = ex2_approx(t1), p2 = ex2_approx(t2),
                                        p3 = ex2_approx(t3);
                            float d0, d1, d2, d3;
                            fadd2(d0, d1, __uint_as_float(pv[e]), __uint_as_float(pv[e + 1]), -D4.x, -D4.y);
                            fadd2(d2, d3, __uint_as_float(pv[e + 2]), __uint_as_float(pv[e + 3]), -D4.z, -D4.w);
                            fmul2(d0, d1, d0, d1, p0, p1);
                            fmul2(d2, d3, d2, d3, p2, p3);
                            wp[2 * e4] = pack_bf16x2(p0, p1);
                            wp[2 * e4 + 1] = pack_bf16x2(p2, p3);
                            wd[2 * e4] = pack_f16x2(d0, d1);
                            wd[2 * e4 + 1] = pack_f16x2(d2, d3);
                        }
                        tmem_st16(tp, wp);
                        tmem_st16(tp + 32, wd);
                        // dS (queries along M, keys along K) as an MN-major operand of dQ'
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const int cc = 4 * cw + q4;
                            *reinterpret_cast<uint4*>(base + ((cc ^ (r & 7)) << 4)) =
                                make_uint4(wd[4 * q4], wd[4 * q4 + 1], wd[4 * q4 + 2], wd[4 * q4 + 3]);
                        }
                    }
                    tmem_wait_st();
                    fence_proxy_async_smem();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->p_full[b]);
                }
                ++j;
            }
        }
    } else {
        // ------------------------------------------------------------ dQ / dK / dV epilogue (warps 8-11)
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const bool leader = (quarter == 0 && lane == 0);
        float* dqst = reinterpret_cast<float*>(smem + kDQStOff);
        uint8_t* dkst = smem + kDKStOff;
        uint8_t* dvst = smem + kDVStOff;
        float2* tab = reinterpret_cast<float2*>(smem + kTabOff);
        uint32_t dkvph = 0;
        long long j = 0;
        int it = 0, tab_h = -1;
        bool ok = true;
        for (long long item = blockIdx.x; item < prm.items && ok; item += gridDim.x, ++it) {
            const Item I = item_of(g, item);
            // dQ' goes to the accumulator with its 2^e (the post kernel undoes it);
            // dK' and dV get 2^-e at the end of the item

            for (int n = 0; n < I.nq; ++n) {
                if (!q_active(g, I, n)) continue;
                const uint32_t c = static_cast<uint32_t>(j & 1);  // the step's dQ' accumulator
                if (!mbar_wait(&bars->dq_full[c], (j >> 1) & 1, ctl, 0x1501)) { ok = false; break; }
                tc_fence_after();
                uint32_t v[32];
                tmem_ld32(tmem + lane_off + kColDQ + 32 * c, v);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->dq_free[c]);
                float* buf = dqst + (j & 1) * kTile * kHeadDim;
                const float sc = prm.scale;
                if (leader) bulk_wait_read_but1();
                named_bar_sync(1, 128);
                // fp32 tile image, chunk c of row r at chunk position c ^ (r & 7)
                float4* rowp = reinterpret_cast<float4*>(buf + r * kHeadDim);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    rowp[c ^ (r & 7)] = make_float4(__uint_as_float(v[4 * c]) * sc, __uint_as_float(v[4 * c + 1]) * sc,
                                                    __uint_as_float(v[4 * c + 2]) * sc,
                                                    __uint_as_float(v[4 * c + 3]) * sc);
                }
                fence_proxy_async_smem();
                named_bar_sync(1, 128);
                if (leader) {
                    const size_t hv = static_cast<size_t>(I.h) * tiles + static_cast<size_t>(I.q0 + n);
                    bulk_reduce_add_f32(prm.ws + prm.L.dqacc + hv * kTile * kHeadDim * 4, buf, kTile * kHeadDim * 4);
                    bulk_commit();
                }
                ++j;
            }
            if (!ok) break;
            // item end: dV and dK' accumulators.  dk is un-rotated here, and the
            // key side of d theta taken with the item's rotated k' rows, which stay
            // in its K', V slot until every row has read them.
            // the window's gradient scaling 2^e undone
            const float down = exp2i(-__ldcg(reinterpret_cast<const int*>(prm.ws + prm.L.wexp) +
                                             static_cast<long long>(I.h) * g.tiles + I.u));
            if (!mbar_wait(&bars->dkv_full, dkvph, ctl, 0x1502)) break;
            dkvph ^= 1;
            tc_fence_after();
            uint32_t dvp[16];  // dv, bf16 pairs
            float dk[32];
            {
                const float sc = prm.scale * down;
                uint32_t vv[32], kk[32];
                tmem_ld32(tmem + lane_off + kColDV, vv);
                tmem_ld32(tmem + lane_off + kColDK, kk);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->dkv_free);
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    dvp[e] = pack_bf16x2(__uint_as_float(vv[2 * e]) * down, __uint_as_float(vv[2 * e + 1]) * down);
#pragma unroll
                for (int e = 0; e < 32; e += 2)
                    fmul2(dk[e], dk[e + 1], __uint_as_float(kk[e]), __uint_as_float(kk[e + 1]), sc, sc);
            }
            const int ks = it & 1;
            if (!mbar_wait(&bars->kv_full[ks], (it >> 1) & 1, ctl, 0x1503)) break;
            const Slot sl = slot_of(g, I.u, r);
            float part[16];
            {
                // k' (fp16) pairs of this row, read one pair at a time
                const uint8_t* krow = smem + kKVOff + ks * 2 * kTileBytes + r * kRowBytes;
                const int sw = (r >> 1) & 3;
#pragma unroll
                for (int ax = 0; ax < 2; ++ax) {
                    const float pos = sl.box.valid ? static_cast<float>(ax ? sl.i : sl.j) : 0.f;
#pragma unroll
                    for (int k = 0; k < 8; ++k) {  // the pair's cross product is the same in both frames
                        const int a = ax * 16 + 2 * k, b = a + 1;
                        const float2 kp = __half22float2(
                            *reinterpret_cast<const __half2*>(krow + (((a >> 3) ^ sw) << 4) + (a & 7) * 2));
                        part[ax * 8 + k] = pos * (dk[b] * kp.x - dk[a] * kp.y);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->kv_empty[ks]);
            if (I.h != tab_h) {  // every row is past its last use of the previous table
                build_table(tab, prm.theta + I.h * 16, g.M, r, 128);
                named_bar_sync(1, 128);
                tab_h = I.h;
            }
            rope32(dk, sl.i, sl.j, tab, true);
            if (leader) bulk_wait_read_all();
            named_bar_sync(1, 128);
            store_row_swz(dkst, r, dk);
            {
                uint8_t* row = dvst + r * kRowBytes;
                const int sw = (r >> 1) & 3;
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    *reinterpret_cast<uint4*>(row + ((c ^ sw) << 4)) =
                        make_uint4(dvp[4 * c], dvp[4 * c + 1], dvp[4 * c + 2], dvp[4 * c + 3]);
            }
            fence_proxy_async_smem();
            named_bar_sync(1, 128);
            if (leader) {
                tile_tma(g, &map_dv, dvst, nullptr, I.u, I.h, true);
                tile_tma(g, &map_dk, dkst, nullptr, I.u, I.h, true);
                bulk_commit();
            }
            // this warp's 16 key-side partials of the tile, group 4 + quarter
            // (the query side, from the post kernel, takes groups 0-3)
            float* out = prm.part + ((static_cast<long long>(I.h) * g.tiles + I.u) * 8 + 4 + quarter) * 16;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                float v = part[e];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == e) out[e] = v;
            }
        }
        if (leader) bulk_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------ 3. post
// dq of each token row (dQ' un-rotated) and the query side of d theta: per
// warp, 16 partials of the tile in groups 0-3 (the main kernel's epilogue
// writes the key side in groups 4-7).
__global__ void __launch_bounds__(128) post_kernel(const PostParams p) {
    __shared__ float2 tab[2 * 64 * 8];
    const Geo& g = p.g;
    const long long T = blockIdx.x / g.heads;  // heads of a tile in turn, as in prep
    const int h = static_cast<int>(blockIdx.x - T * g.heads);
    const long long ht = static_cast<long long>(h) * g.tiles + T;
    build_table(tab, p.theta + h * 16, g.M, threadIdx.x, blockDim.x);
    __syncthreads();
    const int r = threadIdx.x, lane = r & 31, warp = r >> 5;
    const Slot sl = slot_of(g, T, r);
    float part[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) part[e] = 0.f;
    if (sl.valid) {
        const long long tok = ((static_cast<long long>(sl.box.b) * g.H + sl.row) * g.W + sl.col) * g.heads + h;
        float dq[32], q[32];
        const float4* aq = reinterpret_cast<const float4*>(p.ws + p.L.dqacc + (ht * kTile + r) * kHeadDim * 4);
        // the window's gradient scaling 2^e, still in the accumulated dQ'
        const float down = exp2i(-reinterpret_cast<const int*>(p.ws + p.L.wexp)[ht]);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float4 a = aq[c ^ (r & 7)];  // swizzled fp32 tile image
            dq[4 * c] = a.x * down; dq[4 * c + 1] = a.y * down; dq[4 * c + 2] = a.z * down; dq[4 * c + 3] = a.w * down;
        }
        rope32(dq, sl.i, sl.j, tab, true);
        load_row_bf16(p.q + tok * 4, q);
#pragma unroll
        for (int ax = 0; ax < 2; ++ax) {
            const float pos = static_cast<float>(ax ? sl.i : sl.j);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int a = ax * 16 + 2 * kk, b = a + 1;
                part[ax * 8 + kk] = pos * (dq[b] * q[a] - dq[a] * q[b]);
            }
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) p.dq[tok * 4 + c] = pack_chunk(dq, c);
    }
    float* out = reinterpret_cast<float*>(const_cast<uint8_t*>(p.ws) + p.L.part) + (ht * 8 + warp) * 16;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        float v = part[e];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == e) out[e] = v;
    }
}

// ------------------------------------------------------------------ 4. reduce
// One launch, grid (kSplit, heads), in a fixed order (deterministic d theta):
//   level 1: block b of head h sums its contiguous share of the head's
//            [per_head][16] partials into scratch[h][b][16];
//   level 2: the head's last block to finish (a per-head counter, zeroed by
//            the kernel before this one) sums the kSplit level-1 sums.
constexpr int kSplit = 64;

// Rows [per_head b / nb, per_head (b + 1) / nb) of head h's [per_head][16]
// partials: 16 groups of strided rows, then the 16 group sums, into out[h][b].
__device__ __forceinline__ void sum_rows(const float* part, long long per_head, int h, int b, int nb, float* out,
                                         float (&acc)[16][17]) {
    const long long lo = per_head * b / nb, hi = per_head * (b + 1) / nb;
    const int comp = threadIdx.x & 15, grp = threadIdx.x >> 4;
    float s = 0.f;
    for (long long T = lo + grp; T < hi; T += 16) s += __ldcg(part + (static_cast<long long>(h) * per_head + T) * 16 + comp);
    acc[grp][comp] = s;
    __syncthreads();
    if (threadIdx.x < 16) {
        float t = 0.f;
        for (int i = 0; i < 16; ++i) t += acc[i][threadIdx.x];
        out[(static_cast<long long>(h) * nb + b) * 16 + threadIdx.x] = t;
    }
}

__global__ void __launch_bounds__(256) dtheta_kernel(const float* part, long long per_head, float* scratch,
                                                     unsigned int* cnt, float* out) {
    __shared__ float acc[16][17];
    __shared__ bool last;
    const int h = blockIdx.y, b = blockIdx.x, nb = gridDim.x;
    sum_rows(part, per_head, h, b, nb, scratch, acc);
    if (threadIdx.x < 16) __threadfence();  // this block's sums visible before it is counted
    __syncthreads();
    if (threadIdx.x == 0) last = atomicAdd(cnt + h, 1u) == static_cast<unsigned int>(nb - 1);
    __syncthreads();
    if (!last) return;
    __threadfence();
    sum_rows(scratch, nb, h, 0, 1, out, acc);
}

// part: [heads][per_head][16]; dtheta: [heads][16]; scratch: heads * kSplit * 16 floats; cnt: heads
// counters that are zero when the launch starts
cudaError_t launch_dtheta(const float* part, long long per_head, int heads, float* scratch, unsigned int* cnt,
                          float* dtheta, cudaStream_t stream) {
    dtheta_kernel<<<dim3(kSplit, heads), 256, 0, stream>>>(part, per_head, scratch, cnt, dtheta);
    return cudaGetLastError();
}

}  // namespace bwdk

size_t bwd_workspace_bytes(const Geo& g) { return bwdk::ws_layout(g).total; }

void bwd_image_offsets(const Geo& g, size_t* qimg, size_t* kimg) {
    const bwdk::WsLayout L = bwdk::ws_layout(g);
    *qimg = L.qimg;
    *kimg = L.kimg;
}

cudaError_t launch_rope_images(const Geo& g, const void* q, const void* k, const float* theta, uint8_t* ws,
                               cudaStream_t stream) {
    using namespace bwdk;
    const long long ht = static_cast<long long>(g.heads) * g.tiles;
    PrepParams pp{g, static_cast<const uint4*>(q), static_cast<const uint4*>(k), nullptr, nullptr, nullptr,
                  nullptr, theta, ws, ws_layout(g), kPrepImages};
    prep_kernel<<<static_cast<unsigned>(ht), 128, 0, stream>>>(pp);
    return cudaGetLastError();
}

long long bwd_items(const Geo& g) { return bwd_item_count(g); }


cudaError_t launch_bwd(const Geo& g, const BwdPtrs& p, const BwdMaps& maps, unsigned int* status,
                       unsigned long long limit_ns, int num_sms, cudaStream_t stream, cudaEvent_t const* events,
                       bool images_ready) {
    using namespace bwdk;
    const WsLayout L = ws_layout(g);
    const long long ht = static_cast<long long>(g.heads) * g.tiles;
    const float scale = static_cast<float>(1.0 / 5.656854249492380195);  // 1/sqrt(32)
    cudaError_t e = cudaSuccess;
    auto mark = [&](int i) {
        if (events && e == cudaSuccess) e = cudaEventRecord(events[i], stream);
    };
    if (g.N < kTile) {
        // windows inside one tile: the whole backward of a tile in one kernel
        float* part = reinterpret_cast<float*>(p.ws + L.part);
        mark(0);
        mark(1);
        e = launch_small_bwd(g, p, part, reinterpret_cast<unsigned int*>(p.ws + L.cnt), status, limit_ns, num_sms,
                             stream);
        if (e != cudaSuccess) return e;
        mark(2);
        mark(3);
        if ((e = launch_dtheta(part, g.tiles * 4, g.heads, reinterpret_cast<float*>(p.ws + L.part2),
                               reinterpret_cast<unsigned int*>(p.ws + L.cnt), p.dtheta,
                               stream)) != cudaSuccess)
            return e;
        mark(4);
        return e;
    }
    static SmemOptIn optin;
    if ((e = optin.ensure(reinterpret_cast<const void*>(main_kernel), kSmemBytes)) != cudaSuccess) return e;
    mark(0);
    PrepParams pp{g,
                  static_cast<const uint4*>(p.q),
                  static_cast<const uint4*>(p.k),
                  static_cast<const uint4*>(p.v),
                  static_cast<const uint4*>(p.o),
                  static_cast<const uint4*>(p.dout),
                  p.lse,
                  p.theta,
                  p.ws,
                  L,
                  images_ready ? kPrepReuse : kPrepFull};
    prep_kernel<<<static_cast<unsigned>(ht), 128, 0, stream>>>(pp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    scale_kernel<<<static_cast<unsigned>(g.heads * g.wins), 128, 0, stream>>>(g, p.ws, L);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    mark(1);

    MainParams mp;
    mp.g = g;
    mp.ws = p.ws;
    mp.L = L;
    mp.status = status;
    mp.limit_ns = limit_ns;
    mp.items = bwd_items(g);
    mp.scale = scale;
    mp.theta = p.theta;
    mp.part = reinterpret_cast<float*>(p.ws + L.part);
    const long long grid = mp.items < num_sms ? mp.items : num_sms;
    main_kernel<<<static_cast<unsigned>(grid), kThreads, kSmemBytes, stream>>>(maps.v, maps.dv, maps.dout, maps.dk, mp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    mark(2);

    PostParams qp{g, static_cast<const uint4*>(p.q), p.theta, static_cast<uint4*>(p.dq), p.ws, L, scale};
    post_kernel<<<static_cast<unsigned>(ht), 128, 0, stream>>>(qp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    mark(3);
    if ((e = launch_dtheta(reinterpret_cast<const float*>(p.ws + L.part), g.tiles * 8, g.heads,
                           reinterpret_cast<float*>(p.ws + L.part2), reinterpret_cast<unsigned int*>(p.ws + L.cnt),
                           p.dtheta, stream)) != cudaSuccess)
        return e;
    mark(4);
    return e;
}

}  // namespace fswin
