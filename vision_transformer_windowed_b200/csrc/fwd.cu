// Forward kernel: fused shifted-window attention with window-local 2D RoPE.
//
// Persistent, one CTA per SM, holding two independent workers (w = 0, 1).  A
// work item is one 128-row query tile and the key/value tiles of its group;
// the workers of a CTA take alternate items.  Each worker owns:
//   warps 4w .. 4w+3  softmax (thread = query row = TMEM lane); the same
//                     threads also apply the RoPE rotation to their Q row and,
//                     one tile ahead, to their row of each K tile in shared
//                     memory (bf16 in, fp16 out)
//   warp 8 + w        TMA producer (window boxes at shifted addresses)
//   warp 10 + w       tcgen05 MMA issuer: S = Q'K'^T and O_tile = P V in TMEM
// plus its own Q slots, K/V ring, output staging tile, RoPE table and 256 TMEM
// columns.  The workers share nothing but the SM, so neither ever waits for
// the other.
//
// The online softmax keeps O in registers and folds in each P V tile product,
// rescaling only when the running maximum grows by more than 2^8 (exact: the
// final normalisation uses the same maximum as the sum).
#include <cuda.h>
#include <cuda_runtime.h>

#include "dgeo.cuh"
#include "geometry.cuh"
#include "kernels.cuh"
#include "ptx.cuh"
#include "schedule.cuh"
#include "tile_io.cuh"

namespace fswin {

namespace fwdk {

constexpr int kThreads = 384;  // 12 warps: 3 per SM sub-partition, up to 168 registers each
constexpr int kStages = 4;     // K/V ring depth per worker
constexpr int kWarpTma = 8, kWarpMma = 10;

// shared-memory layout per worker (offsets from a 1024-byte aligned base)
constexpr int kQBytes = 2 * kTileBytes;               // 2 Q slots
constexpr int kKVBytes = kStages * 2 * kTileBytes;    // stages x (K, V)
constexpr int kTabBytes = 2 * 8 * 64 * 8;             // [2 axes][8 pairs][64 positions] float2
constexpr int kWorkerBytes = kQBytes + kKVBytes + kTileBytes + kTabBytes;
constexpr int kBarOff = 2 * kWorkerBytes;
constexpr int kSmemBytes = kBarOff + 2048 + 1024;
__device__ __forceinline__ int q_off(int w) { return w * kWorkerBytes; }
__device__ __forceinline__ int kv_off(int w) { return w * kWorkerBytes + kQBytes; }
__device__ __forceinline__ int ost_off(int w) { return w * kWorkerBytes + kQBytes + kKVBytes; }
__device__ __forceinline__ int tab_off(int w) { return w * kWorkerBytes + kQBytes + kKVBytes + kTileBytes; }

// TMEM columns per worker: two S buffers of 128 columns, used by alternate
// tiles.  A tile's P (bf16) is written over the first 64 columns of its S
// buffer as the softmax consumes them, and the tile's P V product goes to
// columns 64-95 of the same buffer (consumed before P V is issued), so the next
// tile's S = Q K^T, in the other buffer, runs while this tile's softmax does.
constexpr uint32_t kTmemCols = 512;
__device__ __forceinline__ uint32_t col_s(int w, uint32_t b) { return w * 256 + b * 128; }
constexpr uint32_t kColP = 0, kColO = 64;  // within an S buffer

struct WorkerBars {
    uint64_t q_full[2], q_ready[2], q_empty[2];
    uint64_t kv_full[kStages], kv_ready[kStages], kv_empty[kStages];
    uint64_t s_full[2], s_empty[2], p_full, o_full, done;  // s_empty[b]: buffer b's P V product read
    uint64_t grp;  // the worker's four softmax warps (a bounded group barrier)
};
struct Bars {
    WorkerBars w[2];
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Bars) <= 2048, "barrier block overflows its shared-memory slot");

struct Params {
    Geo g;
    const float* theta;  // [heads][2][8]
    float* lse;          // [B,H,W,heads], or null (inference: not written)
    // null, or the rotated fp16 q', k' tile images [heads][tiles][128 rows]
    // (64-byte swizzle): Q', K' are then bulk copies of them, not rotated here
    const uint8_t *qimg, *kimg;
    unsigned int* status;
    unsigned long long limit_ns;
    long long items;
};

// Rotates token row r of a swizzled (64-byte swizzle) tile in place: bf16 in,
// fp16 out (the rotated operands of S = Q'K'^T are held in fp16, whose 11-bit
// significand keeps their rounding well below the bf16 rounding of the inputs).
// Channel pairs 0-7 turn by the column position pj, pairs 8-15 by the row
// position pi.  The table is [axis][pair][position], so that lanes holding
// neighbouring tokens read neighbouring table words (no bank conflicts).
__device__ __forceinline__ void rope_row(uint8_t* __restrict__ tile, int r, int pi, int pj,
                                         const float2* __restrict__ tab) {
    uint8_t* row = tile + r * kRowBytes;
    const int sw = (r >> 1) & 3;
    uint4 v[4];
    float2 t[16];  // (cos, sin) of the 16 channel pairs
#pragma unroll
    for (int c = 0; c < 4; ++c) v[c] = *reinterpret_cast<const uint4*>(row + ((c ^ sw) << 4));
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        t[k] = tab[k * 64 + pj];
        t[8 + k] = tab[(8 + k) * 64 + pi];
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint32_t w[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 cs = t[4 * c + e];
            const float a = bf16lo_to_f32(w[e]), b = bf16hi_to_f32(w[e]);
            w[e] = pack_f16x2(a * cs.x - b * cs.y, a * cs.y + b * cs.x);
        }
        v[c] = make_uint4(w[0], w[1], w[2], w[3]);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4*>(row + ((c ^ sw) << 4)) = v[c];
}

// Rotates this thread's row of one tile (unless the tile arrived rotated) and
// signals the MMA issuer (one arrival per warp): the tile's generic-proxy
// writes are fenced for the tensor core.
__device__ __forceinline__ void rotate_and_signal(uint8_t* tile, int r, long long tile_idx, const Geo& g,
                                                  const float2* tab, uint64_t* bar, int lane, bool rotate) {
    if (rotate) {
        int pi, pj;
        tile_row_pos(g, tile_idx, r, &pi, &pj);
        rope_row(tile, r, pi, pj, tab);
        fence_proxy_async_smem();
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(bar);
}

__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
               const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_o,
               const __grid_constant__ Params prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars* bars = reinterpret_cast<Bars*>(smem + kBarOff);
    const Geo& g = prm.g;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    FS_TRACE_INIT();
    if (tid == 0) {
        for (int w = 0; w < 2; ++w) {
            WorkerBars& b = bars->w[w];
            for (int i = 0; i < 2; ++i) {
                mbar_init(&b.q_full[i], 1);
                mbar_init(&b.q_ready[i], 4);
                mbar_init(&b.q_empty[i], 1);
            }
            for (int i = 0; i < kStages; ++i) {
                mbar_init(&b.kv_full[i], 1);
                mbar_init(&b.kv_ready[i], 4);
                mbar_init(&b.kv_empty[i], 1);
            }
            for (int i = 0; i < 2; ++i) {
                mbar_init(&b.s_full[i], 1);
                mbar_init(&b.s_empty[i], 4);
            }
            mbar_init(&b.p_full, 4);
            mbar_init(&b.o_full, 1);
            mbar_init(&b.done, 1);
            mbar_init(&b.grp, 4);
        }
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
    // worker of this warp, and its items: 2 * (blockIdx.x + k * gridDim.x) + w
    const int wk = warp < 8 ? (warp >> 2) : (warp & 1);
    WorkerBars& B = bars->w[wk];
    const long long item0 = 2ll * blockIdx.x + wk, istep = 2ll * gridDim.x;

    if (warp == kWarpTma || warp == kWarpTma + 1) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&map_q);
            prefetch_tmap(&map_k);
            prefetch_tmap(&map_v);
            int it = 0;
            uint32_t kvc = 0;
            bool ok = true;
            for (long long item = item0; item < prm.items && ok; item += istep, ++it) {
                const FwdItem I = d_fwd_item(g, item);
                const int qi = it & 1;
                if (!mbar_wait(&B.q_empty[qi], ((it >> 1) & 1) ^ 1, ctl, 0x101)) break;
                mbar_arrive_expect_tx(&B.q_full[qi], kTileBytes);
                if (prm.qimg)
                    bulk_load(smem + q_off(wk) + qi * kTileBytes,
                              prm.qimg + (static_cast<size_t>(I.h) * g.tiles + static_cast<size_t>(I.X)) * kTileBytes,
                              kTileBytes, &B.q_full[qi]);
                else
                    tile_tma(g, &map_q, smem + q_off(wk) + qi * kTileBytes, &B.q_full[qi], I.X, I.h, false);
                for (int u = 0; u < I.nkv; ++u) {
                    if (!((I.act >> u) & 1u)) continue;
                    const int st = kvc % kStages;
                    const uint32_t ph = (kvc / kStages) & 1;
                    ++kvc;
                    if (!mbar_wait(&B.kv_empty[st], ph ^ 1, ctl, 0x102)) { ok = false; break; }
                    uint8_t* ks = smem + kv_off(wk) + st * 2 * kTileBytes;
                    mbar_arrive_expect_tx(&B.kv_full[st], 2 * kTileBytes);
                    if (prm.kimg)
                        bulk_load(ks,
                                  prm.kimg + (static_cast<size_t>(I.h) * g.tiles + static_cast<size_t>(I.kv0 + u)) *
                                                 kTileBytes,
                                  kTileBytes, &B.kv_full[st]);
                    else
                        tile_tma(g, &map_k, ks, &B.kv_full[st], I.kv0 + u, I.h, false);
                    tile_tma(g, &map_v, ks + kTileBytes, &B.kv_full[st], I.kv0 + u, I.h, false);
                }
            }
        }
    } else if (warp == kWarpMma || warp == kWarpMma + 1) {
        // ------------------------------------------------------------ MMA issue
        if (lane == 0) {
            const uint32_t idesc_qk = make_idesc(kTile, kTile, false, false, true);  // fp16 Q', K'
            const uint32_t idesc_pv = make_idesc_bf16(kTile, kHeadDim, false, true);
            // Shared-memory descriptors built once; per MMA only an offset (in
            // 16-byte units) is added to the start-address field.
            const uint64_t dq0 = make_sdesc(smem_u32(smem + q_off(wk)), 16, 512, kSw64);
            const uint64_t dk0 = make_sdesc(smem_u32(smem + kv_off(wk)), 16, 512, kSw64);
            const uint64_t dv0 = make_sdesc(smem_u32(smem + kv_off(wk) + kTileBytes), 8192, 512, kSw64);
            constexpr uint32_t kQStep = kTileBytes >> 4, kKVStep = (2 * kTileBytes) >> 4;
            int it = 0;
            uint32_t kvc = 0, pph = 0, tc = 0;  // tc: tiles of this worker so far (S buffer tc & 1)
            bool ok = true;
            auto issue_pv = [&](int st, uint32_t b) {
                const uint64_t dv = dv0 + static_cast<uint64_t>(st) * kKVStep;
                const uint32_t t_b = tmem + col_s(wk, b);
#pragma unroll
                for (int k = 0; k < kTile / 16; ++k)
                    umma_ts(t_b + kColO, t_b + kColP + 8 * k, dv + 64 * k, idesc_pv, k > 0);
                umma_commit(&B.o_full);
                umma_commit(&B.kv_empty[st]);
            };
            for (long long item = item0; item < prm.items && ok; item += istep, ++it) {
                const FwdItem I = d_fwd_item(g, item);
                const int qi = it & 1;
                if (!mbar_wait(&B.q_ready[qi], (it >> 1) & 1, ctl, 0x301)) break;
                const uint64_t dq = dq0 + static_cast<uint64_t>(qi) * kQStep;
                int pend = -1;
                for (int u = 0; u < I.nkv && ok; ++u) {
                    if (!((I.act >> u) & 1u)) continue;
                    const int st = kvc % kStages;
                    const uint32_t ph = (kvc / kStages) & 1;
                    ++kvc;
                    if (!mbar_wait(&B.kv_ready[st], ph, ctl, 0x302)) { ok = false; break; }
                    // S buffer b is free once the softmax has read the P V product of
                    // the tile two back (which also means that tile's P V is done)
                    const uint32_t b = tc & 1u;
                    if (tc >= 2 && !mbar_wait(&B.s_empty[b], ((tc >> 1) & 1u) ^ 1u, ctl, 0x303)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t t_s = tmem + col_s(wk, b);
                    const uint64_t dk = dk0 + static_cast<uint64_t>(st) * kKVStep;
                    umma_ss(t_s, dq, dk, idesc_qk, 0u);
                    umma_ss(t_s, dq + 2, dk + 2, idesc_qk, 1u);  // second 16-channel step: +32 bytes
                    umma_commit(&B.s_full[b]);
                    // then P V of the previous tile once its P is in TMEM
                    if (pend >= 0) {
                        if (!mbar_wait(&B.p_full, pph, ctl, 0x304)) { ok = false; break; }
                        pph ^= 1;
                        tc_fence_after();
                        issue_pv(pend, b ^ 1u);
                    }
                    pend = st;
                    ++tc;
                }
                if (ok && pend >= 0) {
                    if (!mbar_wait(&B.p_full, pph, ctl, 0x306)) break;
                    pph ^= 1;
                    tc_fence_after();
                    issue_pv(pend, (tc - 1) & 1u);
                }
                umma_commit(&B.q_empty[qi]);
            }
            umma_commit(&B.done);
            mbar_wait(&B.done, 0, ctl, 0x3ff);
        }
        __syncwarp();
    } else if (warp < 8) {
        // ------------------------------------------------------------ softmax + RoPE (warps 0-7)
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t t_row = tmem + lane_off;  // this warp's TMEM lanes
        uint32_t tcs = 0;                         // tiles of this worker so far (S buffer tcs & 1)
        uint8_t* ost = smem + ost_off(wk);
        float2* tab = reinterpret_cast<float2*>(smem + tab_off(wk));
        const bool leader = (quarter == 0 && lane == 0);
        const bool rotate = prm.qimg == nullptr;  // Q', K' arrive rotated from the images otherwise
        const float sl2 = g.scale_log2;
        uint32_t oph = 0, gph = 0, kvc_rot = 0;
        int tab_head = -1;
        bool ok = true;
        // Waits are made warp-uniform: a lane that gave up takes its warp out
        // with it, so that no warp-collective TMEM access runs on a partial warp.
        auto wwait = [&](uint64_t* bar, uint32_t ph, unsigned int where) -> bool {
            return __all_sync(0xFFFFFFFFu, mbar_wait(bar, ph, ctl, where));
        };
        // Barrier of the worker's 128 softmax threads on an mbarrier (one arrival
        // per warp), so that it too gives up after the wait limit.
        auto group_sync = [&](unsigned int where) -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(&B.grp);
            const bool done = wwait(&B.grp, gph, where);
            gph ^= 1;
            return done;
        };
        // The current item, this thread's segment byte in it, and the next of
        // its key tiles still to rotate.
        FwdItem I{};
        uint32_t myseg = 0;
        int unext = -1;
        auto rotate_next = [&]() -> bool {
            if (unext < 0) return true;
            const int st = kvc_rot % kStages;
            const uint32_t ph = (kvc_rot / kStages) & 1;
            ++kvc_rot;
            if (!wwait(&B.kv_full[st], ph, 0x402)) return false;
            rotate_and_signal(smem + kv_off(wk) + st * 2 * kTileBytes, r, I.kv0 + unext, g, tab, &B.kv_ready[st],
                              lane, rotate);
            const uint32_t rest = unext + 1 < 32 ? (I.act >> (unext + 1)) : 0u;
            unext = rest ? unext + __ffs(rest) : -1;
            return true;
        };
        // Set-up of the jt-th item of this worker: RoPE table (when the head
        // changes), then this thread's Q row and its row of the first K tile, so
        // that the item's first S = Q K^T can start.
        auto start_item = [&](long long item, int jt) -> bool {
            I = d_fwd_item(g, item);
            if (rotate && I.h != tab_head) {
                if (!group_sync(0x406)) return false;  // rotations with the old table done
                tab_head = I.h;
                const float* th = prm.theta + I.h * 16;
                for (int e = r; e < 16 * g.M; e += 128) {
                    const int ap = e / g.M, pos = e - ap * g.M;  // ap = axis * 8 + pair
                    float sn, cs;
                    sincosf(static_cast<float>(pos) * th[ap], &sn, &cs);
                    tab[ap * 64 + pos] = make_float2(cs, sn);
                }
                if (!group_sync(0x407)) return false;
            }
            myseg = I.masked ? seg_at(d_tile_segs(g, I.X, I.win), r >> g.lBT) : 0u;
            unext = __ffs(I.act) - 1;
            const int qi = jt & 1;
            if (!wwait(&B.q_full[qi], (jt >> 1) & 1, 0x401)) return false;
            rotate_and_signal(smem + q_off(wk) + qi * kTileBytes, r, I.X, g, tab, &B.q_ready[qi], lane, rotate);
            return rotate_next();
        };

        if (item0 < prm.items) ok = start_item(item0, 0);
        int it = 0;
        for (long long item = item0; item < prm.items && ok; item += istep, ++it) {
            float o[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = 0.f;
            float m = -INFINITY, l = 0.f;
            bool first = true;
            for (int u = 0; u < I.nkv; ++u) {
                if (!((I.act >> u) & 1u)) continue;
                // rotate the following K tile while this tile's S is computed
                if (!rotate_next()) { ok = false; break; }
                // every 16-column group attends unless the window is cut by the mask
                const uint32_t a16 = I.masked ? d_allow16(g, myseg, I.kv0 + u, I.win) : 0xFFu;
                const bool full = a16 == 0xFFu;
                const uint32_t b = tcs & 1u;
                const uint32_t t_s = t_row + col_s(wk, b);
                if (!wwait(&B.s_full[b], (tcs >> 1) & 1u, 0x403)) { ok = false; break; }
                tc_fence_after();
                if (!first) {  // the previous tile's P V product, in the other S buffer
                    if (!wwait(&B.o_full, oph, 0x404)) { ok = false; break; }
                    oph ^= 1;
                    tc_fence_after();
                    uint32_t v[32];
                    tmem_ld32(t_row + col_s(wk, b ^ 1u) + kColO, v);
                    tmem_wait_ld();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&B.s_empty[b ^ 1u]);
#pragma unroll
                    for (int e = 0; e < 32; e += 2)
                        fadd2(o[e], o[e + 1], o[e], o[e + 1], __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
                } else {
                    // the item's first tile: its row maximum in a pass of its own
                    float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {  // rolled: keeps live ranges (registers) short
                        uint32_t v[32];
                        tmem_ld32(t_s + 32 * c, v);
                        tmem_wait_ld();
                        if (!full) {
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                if (!((a16 >> (2 * c + (e >> 4))) & 1u)) v[e] = __float_as_uint(-INFINITY);
                        }
#pragma unroll
                        for (int e = 0; e < 32; e += 2)
                            mx4[(e >> 1) & 3] =
                                fmax3(mx4[(e >> 1) & 3], __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
                    }
                    m = fmaxf(fmax3(mx4[0], mx4[1], mx4[2]), mx4[3]) * sl2;  // O and l are zero
                }
                // Probabilities, row sum, bf16 P into TMEM.  A masked 16-column group
                // gets the addend -inf: exp2(-inf) = 0 for free.  After an item's first
                // tile the running maximum m is known, so one pass suffices: each
                // chunk's maximum is checked first, and only when it exceeds m by more
                // than 2^64 (or m is still -inf) are m, l, O and the tile's P chunks
                // already written rescaled.  (P up to 2^64 stays far inside the range of
                // bf16 and of the fp32 sums; the result is the same softmax.)
                float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t v[32];
                    tmem_ld32(t_s + 32 * c, v);
                    tmem_wait_ld();
                    const bool ok0 = (a16 >> (2 * c)) & 1u, ok1 = (a16 >> (2 * c + 1)) & 1u;
                    if (!first) {
                        float c4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                        if (ok0) {
#pragma unroll
                            for (int e = 0; e < 16; e += 2)
                                c4[(e >> 1) & 1] = fmax3(c4[(e >> 1) & 1], __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
                        }
                        if (ok1) {
#pragma unroll
                            for (int e = 16; e < 32; e += 2)
                                c4[2 + ((e >> 1) & 1)] =
                                    fmax3(c4[2 + ((e >> 1) & 1)], __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
                        }
                        const float cm = fmaxf(fmaxf(c4[0], c4[1]), fmaxf(c4[2], c4[3])) * sl2;
                        const bool grow = cm > m + 64.f;
                        if (__any_sync(0xFFFFFFFFu, grow)) {
                            const float alpha = grow ? ex2_approx(m - cm) : 1.f;
                            if (grow) m = cm;
#pragma unroll
                            for (int e = 0; e < 32; e += 2) fmul2(o[e], o[e + 1], o[e], o[e + 1], alpha, alpha);
                            l *= alpha;
#pragma unroll
                            for (int e = 0; e < 4; ++e) l4[e] *= alpha;
                            if (c > 0) tmem_wait_st();
#pragma unroll 1
                            for (int k = 0; k < c; ++k) {  // this tile's P chunks already in TMEM
                                uint32_t pw[16];
                                tmem_ld16(t_s + kColP + 16 * k, pw);
                                tmem_wait_ld();
#pragma unroll
                                for (int e = 0; e < 16; ++e)
                                    pw[e] = pack_bf16x2(bf16lo_to_f32(pw[e]) * alpha, bf16hi_to_f32(pw[e]) * alpha);
                                tmem_st16(t_s + kColP + 16 * k, pw);
                            }
                        }
                    }
                    const float mu = (m == -INFINITY) ? 0.f : m;
                    const float add0 = ok0 ? -mu : -INFINITY;
                    const float add1 = ok1 ? -mu : -INFINITY;
                    uint32_t w[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float ad = e < 8 ? add0 : add1;
                        float t0, t1;
                        ffma2(t0, t1, __uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]), sl2, sl2, ad, ad);
                        const float p0 = ex2_approx(t0), p1 = ex2_approx(t1);
                        const int a = (e & 1) * 2;
                        fadd2(l4[a], l4[a + 1], l4[a], l4[a + 1], p0, p1);
                        w[e] = pack_bf16x2(p0, p1);
                    }
                    tmem_st16(t_s + kColP + 16 * c, w);  // over columns of S already read
                }
                l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&B.p_full);
                first = false;
                ++tcs;
            }
            if (!ok) break;
            const long long X = I.X;
            const int h = I.h;
            const Win wq = I.win;
            // the next item's Q row and first K row before this item's epilogue:
            // its first S = Q K^T then runs during the epilogue
            const long long next = item + istep;
            if (next < prm.items && !start_item(next, it + 1)) break;
            if (!wwait(&B.o_full, oph, 0x405)) break;
            oph ^= 1;
            tc_fence_after();
            {
                const uint32_t bl = (tcs - 1) & 1u;  // the item's last tile
                uint32_t v[32];
                tmem_ld32(t_row + col_s(wk, bl) + kColO, v);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&B.s_empty[bl]);
#pragma unroll
                for (int e = 0; e < 32; e += 2)
                    fadd2(o[e], o[e + 1], o[e], o[e + 1], __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
            }
            const float inv = 1.f / l;
            // epilogue: O row into the staging tile (64-byte swizzle), then TMA stores
            if (leader) bulk_wait_read_all();
            if (!group_sync(0x408)) break;
            {
                uint8_t* row = ost + r * kRowBytes;
                const int sw = (r >> 1) & 3;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint4 w;
                    w.x = pack_bf16x2(o[8 * c + 0] * inv, o[8 * c + 1] * inv);
                    w.y = pack_bf16x2(o[8 * c + 2] * inv, o[8 * c + 3] * inv);
                    w.z = pack_bf16x2(o[8 * c + 4] * inv, o[8 * c + 5] * inv);
                    w.w = pack_bf16x2(o[8 * c + 6] * inv, o[8 * c + 7] * inv);
                    *reinterpret_cast<uint4*>(row + ((c ^ sw) << 4)) = w;
                }
            }
            fence_proxy_async_smem();
            if (!group_sync(0x409)) break;
            if (leader) {
                tile_tma(g, &map_o, ost, nullptr, X, h, true);
                bulk_commit();
            }
            // log-sum-exp of this row, at the row's token of the original grid
            Win w = wq;
            if (!g.tpw) {
                const int widx = r >> (g.lnbw + g.lBT);  // window of the row inside the tile
                if (widx) w = win_of(g, wq.gw + widx);
            }
            if (w.valid && prm.lse != nullptr) {  // no lse: inference
                int pi, pj;
                tile_row_pos(g, X, r, &pi, &pj);
                int row = w.wr * g.M + pi + g.s, col = w.wc * g.M + pj + g.s;
                if (row >= g.Hp) row -= g.Hp;
                if (col >= g.Wp) col -= g.Wp;
                if (row < g.H && col < g.W) {  // not a padded position
                    const float lse2 = m + lg2_approx(l);
                    const long long tok = ((static_cast<long long>(w.b) * g.H + row) * g.W + col) * g.heads + h;
                    prm.lse[tok] = lse2 * 0.69314718055994530942f;
                }
            }
        }
        if (leader) bulk_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace fwdk

long long fwd_items(const Geo& g) { return fwd_item_count(g); }

cudaError_t launch_fwd(const Geo& g, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                       const CUtensorMap& mo, const void* q, const void* k, const void* v, void* o,
                       const float* theta, float* lse, unsigned int* status,
                       unsigned long long limit_ns, int num_sms, cudaStream_t stream, cudaEvent_t const* events,
                       uint8_t* train_ws) {
    fwdk::Params prm;
    prm.g = g;
    prm.theta = theta;
    prm.lse = lse;
    prm.qimg = prm.kimg = nullptr;
    prm.status = status;
    prm.limit_ns = limit_ns;
    prm.items = fwd_items(g);
    if (prm.items == 0) return cudaSuccess;
    if (g.N < kTile) {  // windows inside one tile
        if (events) {
            cudaError_t e = cudaEventRecord(events[0], stream);
            if (e != cudaSuccess) return e;
        }
        cudaError_t e = launch_small_fwd(g, q, k, v, theta, o, lse, status, limit_ns, num_sms, stream);
        if (e == cudaSuccess && events) e = cudaEventRecord(events[1], stream);
        return e;
    }
    static SmemOptIn optin;
    if (cudaError_t e = optin.ensure(reinterpret_cast<const void*>(fwdk::fwd_kernel), fwdk::kSmemBytes))
        return e;
    const long long pairs = (prm.items + 1) / 2;  // each CTA runs two workers
    const long long grid = pairs < num_sms ? pairs : num_sms;
    if (events) {
        cudaError_t e = cudaEventRecord(events[0], stream);
        if (e != cudaSuccess) return e;
    }
    if (train_ws) {  // rotated q', k' images first, once per row, into the backward's workspace
        if (cudaError_t e = launch_rope_images(g, q, k, theta, train_ws, stream)) return e;
        size_t qo = 0, ko = 0;
        bwd_image_offsets(g, &qo, &ko);
        prm.qimg = train_ws + qo;
        prm.kimg = train_ws + ko;
    }
    fwdk::fwd_kernel<<<static_cast<unsigned>(grid), fwdk::kThreads, fwdk::kSmemBytes, stream>>>(mq, mk, mv, mo, prm);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess && events) e = cudaEventRecord(events[1], stream);
    return e;
}

}  // namespace fswin
