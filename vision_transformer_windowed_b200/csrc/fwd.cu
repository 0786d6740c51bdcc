// Forward kernel: fused shifted-window attention with window-local 2D RoPE.
//
// Persistent, warp-specialised, one CTA per SM.  A work item is a pair of
// 128-row query tiles (A and B) that share one stream of key/value tiles:
//   warps 0-3  softmax for tile A (thread = query row = TMEM lane)
//   warps 4-7  softmax for tile B
//   warp 8     RoPE: rotate Q and K tiles in shared memory as they land
//   warp 9     TMA producer (window boxes at shifted addresses, no gather copy)
//   warps 10-11 tcgen05 MMA issuers, one per query tile (they never wait on each
//              other): S = Q'K'^T and O_tile = P V into TMEM
// The online softmax keeps O in registers and folds in each P V tile product,
// rescaling only when the running maximum grows by more than 2^8 (exact: the
// final normalisation uses the same maximum as the sum).
#include <cuda.h>
#include <cuda_runtime.h>

#include "geometry.cuh"
#include "kernels.cuh"
#include "ptx.cuh"
#include "schedule.cuh"
#include "tile_io.cuh"
#include "dgeo.cuh"

namespace fswin {

namespace fwdk {

// 12 warps: 3 per SM sub-partition, so each thread may hold up to 168 registers.
constexpr int kThreads = 384;
constexpr int kStages = 6;
constexpr int kWarpRot = 8, kRotWarps = 1, kWarpTma = 9, kWarpMma = 10;  // MMA: warps 10 (tile A), 11 (tile B)

// shared-memory layout (offsets from a 1024-byte aligned base)
constexpr int kQOff = 0;                                   // 2 slots x 2 tiles
constexpr int kKVOff = kQOff + 2 * 2 * kTileBytes;         // stages x (K, V)
constexpr int kOStOff = kKVOff + kStages * 2 * kTileBytes; // 2 output staging tiles
constexpr int kTabOff = kOStOff + 2 * kTileBytes;          // 2 x [2][64][8] float2
constexpr int kBarOff = kTabOff + 2 * 2 * 64 * 8 * 8;
constexpr int kSmemBytes = kBarOff + 1024 + 1024;

// TMEM columns, per query tile T: S [128 cols], P (bf16) [64], O tile [32]
constexpr uint32_t kTmemCols = 512;
__device__ __forceinline__ uint32_t col_s(int T) { return T * 256; }
__device__ __forceinline__ uint32_t col_p(int T) { return T * 256 + 128; }
__device__ __forceinline__ uint32_t col_o(int T) { return T * 256 + 192; }

struct Bars {
    uint64_t q_full[2], q_ready[2], q_empty[2];
    uint64_t kv_full[kStages], kv_ready[kStages], kv_empty[kStages];
    uint64_t s_full[2], s_free[2], p_full[2], o_full[2];
    uint64_t done;
    uint32_t tmem_base;
    int abort_flag;
};

struct Params {
    Geo g;
    const float* theta;  // [heads][2][8]
    float* lse;          // [B,H,W,heads]
    unsigned int* status;
    unsigned long long limit_ns;
    long long items;
};

// Rotate token row r of a swizzled (64-byte swizzle) tile in place: bf16 in,
// fp16 out (the rotated operands of S = Q'K'^T are held in fp16, whose 11-bit
// significand keeps their rounding well below the bf16 rounding of the inputs).
// All loads first, then the arithmetic, then all stores: the row and the table
// are both in shared memory, so interleaving would serialise every chunk.
__device__ __noinline__ void rope_row(uint8_t* __restrict__ tile, int r, int pi, int pj,
                                      const float2* __restrict__ tab) {
    uint8_t* row = tile + r * kRowBytes;
    const int sw = (r >> 1) & 3;
    uint4 v[4];
    float4 t[8];  // (cos, sin) of the 16 channel pairs
#pragma unroll
    for (int c = 0; c < 4; ++c) v[c] = *reinterpret_cast<const uint4*>(row + ((c ^ sw) << 4));
    const float4* tx = reinterpret_cast<const float4*>(tab + pj * 8);
    const float4* ty = reinterpret_cast<const float4*>(tab + (64 + pi) * 8);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        t[q] = tx[q];
        t[4 + q] = ty[q];
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint32_t w[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int pr = 4 * c + e;  // channel pair 0..15 (0-7: x axis, 8-15: y axis)
            const float4 tt = t[pr >> 1];
            const float cs = (pr & 1) ? tt.z : tt.x, sn = (pr & 1) ? tt.w : tt.y;
            const float a = bf16lo_to_f32(w[e]), b = bf16hi_to_f32(w[e]);
            w[e] = pack_f16x2(a * cs - b * sn, a * sn + b * cs);
        }
        v[c] = make_uint4(w[0], w[1], w[2], w[3]);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4*>(row + ((c ^ sw) << 4)) = v[c];
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
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->q_full[i], 1);
            mbar_init(&bars->q_ready[i], kRotWarps);
            mbar_init(&bars->q_empty[i], 2);  // one commit per MMA-issuing thread
            mbar_init(&bars->s_full[i], 1);
            mbar_init(&bars->p_full[i], 4);
            mbar_init(&bars->s_free[i], 4);
            mbar_init(&bars->o_full[i], 1);
        }
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&bars->kv_full[i], 1);
            mbar_init(&bars->kv_ready[i], kRotWarps);
            mbar_init(&bars->kv_empty[i], 2);  // one arrival per MMA-issuing thread
        }
        mbar_init(&bars->done, 2);
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

    if (warp == kWarpTma) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&map_q);
            prefetch_tmap(&map_k);
            prefetch_tmap(&map_v);
            int it = 0;
            uint32_t kvc = 0;
            bool ok = true;
            for (long long item = blockIdx.x; item < prm.items && ok; item += gridDim.x, ++it) {
                const FwdItem I = d_fwd_item(g, item);
                const int qi = it & 1;
                if (!mbar_wait(&bars->q_empty[qi], ((it >> 1) & 1) ^ 1, ctl, 0x101)) break;
                uint8_t* qs = smem + kQOff + qi * 2 * kTileBytes;
                mbar_arrive_expect_tx(&bars->q_full[qi], (I.tB >= 0 ? 2 : 1) * kTileBytes);
                tile_tma(g, &map_q, qs, &bars->q_full[qi], I.tA, I.h, false);
                if (I.tB >= 0) tile_tma(g, &map_q, qs + kTileBytes, &bars->q_full[qi], I.tB, I.h, false);
                const uint32_t used = I.act[0] | I.act[1];
                for (int u = 0; u < I.nkv; ++u) {
                    if (!((used >> u) & 1u)) continue;
                    const int st = kvc % kStages;
                    const uint32_t ph = (kvc / kStages) & 1;
                    ++kvc;
                    if (!mbar_wait(&bars->kv_empty[st], ph ^ 1, ctl, 0x102)) { ok = false; break; }
                    uint8_t* ks = smem + kKVOff + st * 2 * kTileBytes;
                    mbar_arrive_expect_tx(&bars->kv_full[st], 2 * kTileBytes);
                    tile_tma(g, &map_k, ks, &bars->kv_full[st], I.kv0 + u, I.h, false);
                    tile_tma(g, &map_v, ks + kTileBytes, &bars->kv_full[st], I.kv0 + u, I.h, false);
                }
            }
        }
    } else if (warp >= kWarpRot && warp < kWarpRot + kRotWarps) {
        // ------------------------------------------------------------ RoPE
        const int r0 = tid - kWarpRot * 32;  // rows r0, r0 + 32, ... of every tile
        constexpr int kRotThreads = kRotWarps * 32;
        int it = 0;
        uint32_t kvc = 0;
        bool ok = true;
        int tab_head = -1, tab_buf = 1;
        for (long long item = blockIdx.x; item < prm.items && ok; item += gridDim.x, ++it) {
            const FwdItem I = d_fwd_item(g, item);
            // cos/sin table of the item's head, rebuilt only when the head changes
            // (double-buffered; the barrier orders it against the previous rotations)
            if (I.h != tab_head) {
                tab_buf ^= 1;
                tab_head = I.h;
                float2* tw = reinterpret_cast<float2*>(smem + kTabOff) + tab_buf * (2 * 64 * 8);
                const float* th = prm.theta + I.h * 16;
                for (int e = r0; e < 2 * g.M * 8; e += kRotThreads) {
                    const int ax = e / (g.M * 8), rem = e - ax * g.M * 8, pos = rem >> 3, k = rem & 7;
                    float sn, cs;
                    sincosf(static_cast<float>(pos) * th[ax * 8 + k], &sn, &cs);
                    tw[(ax * 64 + pos) * 8 + k] = make_float2(cs, sn);
                }
                named_bar_sync(1, kRotThreads);
            }
            const float2* tab = reinterpret_cast<const float2*>(smem + kTabOff) + tab_buf * (2 * 64 * 8);
            const int qi = it & 1;
            if (!mbar_wait(&bars->q_full[qi], (it >> 1) & 1, ctl, 0x201)) break;
            uint8_t* qs = smem + kQOff + qi * 2 * kTileBytes;
#pragma unroll 1
            for (int h2 = 0; h2 < kTile / kRotThreads; ++h2) {
                const int r = r0 + h2 * kRotThreads;
                int pi, pj;
                tile_row_pos(g, I.tA, r, &pi, &pj);
                rope_row(qs, r, pi, pj, tab);
                if (I.tB >= 0) {
                    tile_row_pos(g, I.tB, r, &pi, &pj);
                    rope_row(qs + kTileBytes, r, pi, pj, tab);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->q_ready[qi]);
            const uint32_t used = I.act[0] | I.act[1];
            for (int u = 0; u < I.nkv; ++u) {
                if (!((used >> u) & 1u)) continue;
                const int st = kvc % kStages;
                const uint32_t ph = (kvc / kStages) & 1;
                ++kvc;
                if (!mbar_wait(&bars->kv_full[st], ph, ctl, 0x202)) { ok = false; break; }
#pragma unroll 1
                for (int h2 = 0; h2 < kTile / kRotThreads; ++h2) {
                    const int r = r0 + h2 * kRotThreads;
                    int pi, pj;
                    tile_row_pos(g, I.kv0 + u, r, &pi, &pj);
                    rope_row(smem + kKVOff + st * 2 * kTileBytes, r, pi, pj, tab);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->kv_ready[st]);
            }
        }
    } else if (warp == kWarpMma || warp == kWarpMma + 1) {
        // ------------------------------------------------------------ MMA issue, one thread per query tile
        if (lane == 0) {
            const int T = warp - kWarpMma;
            const uint32_t idesc_qk = make_idesc(kTile, kTile, false, false, true);  // fp16 Q', K'
            const uint32_t idesc_pv = make_idesc_bf16(kTile, kHeadDim, false, true);
            // Shared-memory descriptors built once; per MMA only an offset (in 16-byte
            // units) is added to the start-address field.
            const uint64_t dq0 = make_sdesc(smem_u32(smem + kQOff + T * kTileBytes), 16, 512, kSw64);
            const uint64_t dk0 = make_sdesc(smem_u32(smem + kKVOff), 16, 512, kSw64);
            const uint64_t dv0 = make_sdesc(smem_u32(smem + kKVOff + kTileBytes), 8192, 512, kSw64);
            constexpr uint32_t kStep = (2 * kTileBytes) >> 4;  // next Q slot / next K,V stage
            const uint32_t t_s = tmem + col_s(T), t_p = tmem + col_p(T), t_o = tmem + col_o(T);
            int it = 0;
            uint32_t kvc = 0, pph = 0, sfph = 0;
            bool ok = true;
            auto issue_pv = [&](int st) {
                const uint64_t dv = dv0 + static_cast<uint64_t>(st) * kStep;
#pragma unroll
                for (int k = 0; k < kTile / 16; ++k) umma_ts(t_o, t_p + 8 * k, dv + 64 * k, idesc_pv, k > 0);
                umma_commit(&bars->o_full[T]);
                umma_commit(&bars->kv_empty[st]);
            };
            for (long long item = blockIdx.x; item < prm.items && ok; item += gridDim.x, ++it) {
                const FwdItem I = d_fwd_item(g, item);
                const int qi = it & 1;
                if (!mbar_wait(&bars->q_ready[qi], (it >> 1) & 1, ctl, 0x301)) break;
                const uint64_t dq = dq0 + static_cast<uint64_t>(qi) * kStep;
                const uint32_t mine = I.act[T], used = I.act[0] | I.act[1];
                int pend = -1;
                for (int u = 0; u < I.nkv && ok; ++u) {
                    if (!((used >> u) & 1u)) continue;
                    const int st = kvc % kStages;
                    const uint32_t ph = (kvc / kStages) & 1;
                    ++kvc;
                    if (!mbar_wait(&bars->kv_ready[st], ph, ctl, 0x302)) { ok = false; break; }
                    if (!((mine >> u) & 1u)) {  // only the other query tile reads this stage
                        mbar_arrive(&bars->kv_empty[st]);
                        continue;
                    }
                    tc_fence_after();
                    // the next S = Q K^T as soon as the softmax has read the previous S,
                    // then P V of the previous tile once its P is in TMEM
                    if (pend >= 0) {
                        if (!mbar_wait(&bars->s_free[T], sfph, ctl, 0x307 + T)) { ok = false; break; }
                        sfph ^= 1;
                        tc_fence_after();
                    }
                    const uint64_t dk = dk0 + static_cast<uint64_t>(st) * kStep;
                    umma_ss(t_s, dq, dk, idesc_qk, 0u);
                    umma_ss(t_s, dq + 2, dk + 2, idesc_qk, 1u);  // second 16-channel step: +32 bytes
                    umma_commit(&bars->s_full[T]);
                    if (pend >= 0) {
                        if (!mbar_wait(&bars->p_full[T], pph, ctl, 0x303 + T)) { ok = false; break; }
                        pph ^= 1;
                        tc_fence_after();
                        issue_pv(pend);
                    }
                    pend = st;
                }
                if (ok && pend >= 0) {
                    if (!mbar_wait(&bars->s_free[T], sfph, ctl, 0x309 + T)) break;
                    sfph ^= 1;
                    if (!mbar_wait(&bars->p_full[T], pph, ctl, 0x305 + T)) break;
                    pph ^= 1;
                    tc_fence_after();
                    issue_pv(pend);
                }
                umma_commit(&bars->q_empty[qi]);
            }
            umma_commit(&bars->done);
            mbar_wait(&bars->done, 0, ctl, 0x3ff);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax (warps 0-7)
        const int T = warp >> 2;
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t t_s = tmem + lane_off + col_s(T), t_p = tmem + lane_off + col_p(T),
                       t_o = tmem + lane_off + col_o(T);
        uint8_t* ost = smem + kOStOff + T * kTileBytes;
        const bool leader = (quarter == 0 && lane == 0);
        const float sl2 = g.scale_log2;
        uint32_t sph = 0, oph = 0;
        bool ok = true;
        for (long long item = blockIdx.x; item < prm.items && ok; item += gridDim.x) {
            const FwdItem I = d_fwd_item(g, item);
            if (T == 1 && I.tB < 0) continue;
            const long long X = T ? I.tB : I.tA;
            const Win wq = I.paired ? d_tile_win(g, X) : I.win;
            const uint32_t myseg = seg_at(d_tile_segs(g, X, wq), r >> g.lBT);
            const uint32_t myact = T ? I.act[1] : I.act[0];
            float o[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = 0.f;
            float m = -INFINITY, l = 0.f;
            bool first = true;
            for (int u = 0; u < I.nkv; ++u) {
                if (!((myact >> u) & 1u)) continue;
                const uint32_t a16 = d_allow16(g, myseg, I.kv0 + u, wq);
                const bool full = a16 == 0xFFu;
                if (!mbar_wait(&bars->s_full[T], sph, ctl, 0x401 + T)) { ok = false; break; }
                sph ^= 1;
                tc_fence_after();
                // pass 1: row maximum of the attended raw scores
                float mx8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) mx8[e] = -INFINITY;
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {  // rolled: keeps live ranges (registers) short
                    uint32_t v[32];
                    tmem_ld32(t_s + 32 * c, v);
                    tmem_wait_ld();
                    if (full) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) mx8[e & 7] = fmaxf(mx8[e & 7], __uint_as_float(v[e]));
                    } else {
                        const bool ok0 = (a16 >> (2 * c)) & 1u, ok1 = (a16 >> (2 * c + 1)) & 1u;
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const float x = (e < 16 ? ok0 : ok1) ? __uint_as_float(v[e]) : -INFINITY;
                            mx8[e & 7] = fmaxf(mx8[e & 7], x);
                        }
                    }
                }
                const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                       fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
                const float m_tile = mx * sl2;
                if (!first) {
                    if (!mbar_wait(&bars->o_full[T], oph, ctl, 0x403 + T)) { ok = false; break; }
                    oph ^= 1;
                    tc_fence_after();
                    uint32_t v[32];
                    tmem_ld32(t_o, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; e += 2)
                        fadd2(o[e], o[e + 1], o[e], o[e + 1], __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
                }
                if (m_tile > m + 8.f) {
                    const float alpha = ex2_approx(m - m_tile);
#pragma unroll
                    for (int e = 0; e < 32; e += 2) fmul2(o[e], o[e + 1], o[e], o[e + 1], alpha, alpha);
                    l *= alpha;
                    m = m_tile;
                }
                const float mu = (m == -INFINITY) ? 0.f : m;
                // pass 2: probabilities, row sum, bf16 P into TMEM
                // A masked 16-column group gets the addend -inf: its scores map to
                // exp2(-inf) = 0 with no extra instruction.
                float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t v[32];
                    tmem_ld32(t_s + 32 * c, v);
                    tmem_wait_ld();
                    if (c == 3) {  // S fully read: the next S = Q K^T may overwrite it
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&bars->s_free[T]);
                    }
                    const float add0 = ((a16 >> (2 * c)) & 1u) ? -mu : -INFINITY;
                    const float add1 = ((a16 >> (2 * c + 1)) & 1u) ? -mu : -INFINITY;
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
                    tmem_st16(t_p + 16 * c, w);
                }
                l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->p_full[T]);
                first = false;
            }
            if (!ok) break;
            if (!mbar_wait(&bars->o_full[T], oph, ctl, 0x405 + T)) break;
            oph ^= 1;
            tc_fence_after();
            {
                uint32_t v[32];
                tmem_ld32(t_o, v);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; e += 2)
                        fadd2(o[e], o[e + 1], o[e], o[e + 1], __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
            }
            const float inv = 1.f / l;
            // epilogue: O row into the staging tile (64-byte swizzle), then TMA stores
            if (leader) bulk_wait_read_all();
            named_bar_sync(2 + T, 128);
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
            named_bar_sync(2 + T, 128);
            if (leader) {
                tile_tma(g, &map_o, ost, nullptr, X, I.h, true);
                bulk_commit();
            }
            const Slot me = d_slot_of(g, X, r);
            if (me.box.valid) {
                const float lse2 = m + lg2_approx(l);
                const long long tok =
                    ((static_cast<long long>(me.box.b) * g.H + me.row) * g.W + me.col) * g.heads + I.h;
                prm.lse[tok] = lse2 * 0.69314718055994530942f;
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
                       const CUtensorMap& mo, const float* theta, float* lse, unsigned int* status,
                       unsigned long long limit_ns, int num_sms, cudaStream_t stream, cudaEvent_t const* events) {
    fwdk::Params prm;
    prm.g = g;
    prm.theta = theta;
    prm.lse = lse;
    prm.status = status;
    prm.limit_ns = limit_ns;
    prm.items = fwd_items(g);
    if (prm.items == 0) return cudaSuccess;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(fwdk::fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             fwdk::kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    const long long grid = prm.items < num_sms ? prm.items : num_sms;
    if (events) {
        cudaError_t e = cudaEventRecord(events[0], stream);
        if (e != cudaSuccess) return e;
    }
    fwdk::fwd_kernel<<<static_cast<unsigned>(grid), fwdk::kThreads, fwdk::kSmemBytes, stream>>>(mq, mk, mv, mo, prm);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess && events) e = cudaEventRecord(events[1], stream);
    return e;
}

}  // namespace fswin
