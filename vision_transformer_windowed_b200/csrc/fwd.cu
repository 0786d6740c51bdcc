// Forward kernel: fused shifted-window attention with window-local 2D RoPE.
//
// Persistent, warp-specialised, one CTA per SM.  A work item is a pair of
// 128-row query tiles (A and B) that share one stream of key/value tiles:
//   warps 0-3  softmax for tile A (thread = query row = TMEM lane)
//   warps 4-7  softmax for tile B
//   warps 8-11 RoPE: rotate Q and K tiles in shared memory as they land
//   warp 12    TMA producer (window boxes at shifted addresses, no gather copy)
//   warp 13    tcgen05 MMA issuer: S = Q'K'^T and O_tile = P V into TMEM
// The online softmax keeps O in registers and folds in each P V tile product,
// rescaling only when the running maximum grows by more than 2^8 (exact: the
// final normalisation uses the same maximum as the sum).
#include <cuda.h>
#include <cuda_runtime.h>

#include "geometry.cuh"
#include "kernels.cuh"
#include "ptx.cuh"
#include "schedule.cuh"

namespace fswin {

namespace fwdk {

constexpr int kThreads = 448;
constexpr int kStages = 6;
constexpr int kWarpRot = 8, kWarpTma = 12, kWarpMma = 13;

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
    uint64_t s_full[2], p_full[2], o_full[2];
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

using Item = FwdItem;
__device__ __forceinline__ Item item_of(const Geo& g, long long it) { return fwd_item(g, it); }
__device__ __forceinline__ bool active(const Geo& g, const Item& I, int T, int u) { return fwd_active(g, I, T, u); }

__device__ __forceinline__ void load_tile_boxes(const Geo& g, const CUtensorMap* map, uint8_t* dst, uint64_t* bar,
                                                long long tile, int h) {
    for (int i = 0; i < g.bpt; ++i) {
        const Box bx = box_of(g, tile * g.bpt + i);
        tma_load_5d(dst + i * g.BT * kRowBytes, map, bar, 0, h, bx.col0, bx.row0, bx.b);
    }
}

// Rotate token row r of a swizzled (64-byte swizzle) tile in place: bf16 in,
// fp16 out (the rotated operands of S = Q'K'^T are held in fp16, whose 11-bit
// significand keeps their rounding well below the bf16 rounding of the inputs).
__device__ __forceinline__ void rope_row(uint8_t* tile, int r, int pi, int pj, const float2* tab) {
    uint8_t* row = tile + r * kRowBytes;
    const int sw = (r >> 1) & 3;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint4* p = reinterpret_cast<uint4*>(row + ((c ^ sw) << 4));
        uint4 v = *p;
        const int ax = c >> 1;
        const float2* t = tab + (ax * 64 + (ax ? pi : pj)) * 8 + (c & 1) * 4;
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float a = bf16lo_to_f32(w[e]), b = bf16hi_to_f32(w[e]);
            const float2 cs = t[e];
            w[e] = pack_f16x2(a * cs.x - b * cs.y, a * cs.y + b * cs.x);
        }
        *p = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
               const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_o,
               const Params prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars* bars = reinterpret_cast<Bars*>(smem + kBarOff);
    const Geo& g = prm.g;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->q_full[i], 1);
            mbar_init(&bars->q_ready[i], 4);
            mbar_init(&bars->q_empty[i], 1);
            mbar_init(&bars->s_full[i], 1);
            mbar_init(&bars->p_full[i], 4);
            mbar_init(&bars->o_full[i], 1);
        }
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&bars->kv_full[i], 1);
            mbar_init(&bars->kv_ready[i], 4);
            mbar_init(&bars->kv_empty[i], 1);
        }
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

    if (warp == kWarpTma) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&map_q);
            prefetch_tmap(&map_k);
            prefetch_tmap(&map_v);
            int it = 0;
            uint32_t kvc = 0;
            for (long long item = blockIdx.x; item < prm.items; item += gridDim.x, ++it) {
                const Item I = item_of(g, item);
                const int qi = it & 1;
                if (!mbar_wait(&bars->q_empty[qi], ((it >> 1) & 1) ^ 1, ctl, 0x101)) break;
                uint8_t* qs = smem + kQOff + qi * 2 * kTileBytes;
                mbar_arrive_expect_tx(&bars->q_full[qi], (I.tB >= 0 ? 2 : 1) * kTileBytes);
                load_tile_boxes(g, &map_q, qs, &bars->q_full[qi], I.tA, I.h);
                if (I.tB >= 0) load_tile_boxes(g, &map_q, qs + kTileBytes, &bars->q_full[qi], I.tB, I.h);
                bool ok = true;
                for (int u = 0; u < I.nkv && ok; ++u) {
                    if (!active(g, I, 0, u) && !active(g, I, 1, u)) continue;
                    const int st = kvc % kStages;
                    const uint32_t ph = (kvc / kStages) & 1;
                    ++kvc;
                    if (!mbar_wait(&bars->kv_empty[st], ph ^ 1, ctl, 0x102)) { ok = false; break; }
                    uint8_t* ks = smem + kKVOff + st * 2 * kTileBytes;
                    mbar_arrive_expect_tx(&bars->kv_full[st], 2 * kTileBytes);
                    load_tile_boxes(g, &map_k, ks, &bars->kv_full[st], I.kv0 + u, I.h);
                    load_tile_boxes(g, &map_v, ks + kTileBytes, &bars->kv_full[st], I.kv0 + u, I.h);
                }
                if (!ok) break;
            }
        }
    } else if (warp >= kWarpRot && warp < kWarpRot + 4) {
        // ------------------------------------------------------------ RoPE
        const int r = tid - kWarpRot * 32;
        int it = 0;
        uint32_t kvc = 0;
        bool ok = true;
        for (long long item = blockIdx.x; item < prm.items && ok; item += gridDim.x, ++it) {
            const Item I = item_of(g, item);
            float2* tab = reinterpret_cast<float2*>(smem + kTabOff) + (it & 1) * (2 * 64 * 8);
            const float* th = prm.theta + I.h * 16;
            for (int e = r; e < 2 * g.M * 8; e += 128) {
                const int ax = e / (g.M * 8), rem = e - ax * g.M * 8, pos = rem >> 3, k = rem & 7;
                float sn, cs;
                sincosf(static_cast<float>(pos) * th[ax * 8 + k], &sn, &cs);
                tab[(ax * 64 + pos) * 8 + k] = make_float2(cs, sn);
            }
            named_bar_sync(1, 128);
            const int qi = it & 1;
            if (!mbar_wait(&bars->q_full[qi], (it >> 1) & 1, ctl, 0x201)) break;
            uint8_t* qs = smem + kQOff + qi * 2 * kTileBytes;
            {
                const Slot sa = slot_of(g, I.tA, r);
                rope_row(qs, r, sa.i, sa.j, tab);
                if (I.tB >= 0) {
                    const Slot sb = slot_of(g, I.tB, r);
                    rope_row(qs + kTileBytes, r, sb.i, sb.j, tab);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->q_ready[qi]);
            for (int u = 0; u < I.nkv; ++u) {
                if (!active(g, I, 0, u) && !active(g, I, 1, u)) continue;
                const int st = kvc % kStages;
                const uint32_t ph = (kvc / kStages) & 1;
                ++kvc;
                if (!mbar_wait(&bars->kv_full[st], ph, ctl, 0x202)) { ok = false; break; }
                const Slot sk = slot_of(g, I.kv0 + u, r);
                rope_row(smem + kKVOff + st * 2 * kTileBytes, r, sk.i, sk.j, tab);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->kv_ready[st]);
            }
        }
    } else if (warp == kWarpMma) {
        // ------------------------------------------------------------ MMA issue
        if (lane == 0) {
            const uint32_t idesc_qk = make_idesc(kTile, kTile, false, false, true);  // fp16 Q', K'
            const uint32_t idesc_pv = make_idesc_bf16(kTile, kHeadDim, false, true);
            int it = 0;
            uint32_t kvc = 0;
            uint32_t pph[2] = {0, 0};
            bool ok = true;
            auto issue_pv = [&](int T, int st) {
                const uint32_t vaddr = smem_u32(smem + kKVOff + st * 2 * kTileBytes + kTileBytes);
#pragma unroll
                for (int k = 0; k < kTile / 16; ++k)
                    umma_ts(tmem + col_o(T), tmem + col_p(T) + 8 * k, make_sdesc(vaddr + 1024 * k, 8192, 512, kSw64),
                            idesc_pv, k > 0);
                umma_commit(&bars->o_full[T]);
            };
            for (long long item = blockIdx.x; item < prm.items && ok; item += gridDim.x, ++it) {
                const Item I = item_of(g, item);
                const int qi = it & 1;
                if (!mbar_wait(&bars->q_ready[qi], (it >> 1) & 1, ctl, 0x301)) break;
                tc_fence_after();
                const uint32_t qaddr = smem_u32(smem + kQOff + qi * 2 * kTileBytes);
                int pend[2] = {-1, -1};
                int readers[kStages];
                for (int u = 0; u < I.nkv && ok; ++u) {
                    const bool aA = active(g, I, 0, u), aB = active(g, I, 1, u);
                    if (!aA && !aB) continue;
                    const int st = kvc % kStages;
                    const uint32_t ph = (kvc / kStages) & 1;
                    ++kvc;
                    if (!mbar_wait(&bars->kv_ready[st], ph, ctl, 0x302)) { ok = false; break; }
                    tc_fence_after();
                    readers[st] = (aA ? 1 : 0) + (aB ? 1 : 0);
                    const uint32_t kaddr = smem_u32(smem + kKVOff + st * 2 * kTileBytes);
                    for (int T = 0; T < 2; ++T) {
                        if (!(T ? aB : aA)) continue;
                        if (pend[T] >= 0) {
                            if (!mbar_wait(&bars->p_full[T], pph[T], ctl, 0x303 + T)) { ok = false; break; }
                            pph[T] ^= 1;
                            tc_fence_after();
                            issue_pv(T, pend[T]);
                            if (--readers[pend[T]] == 0) umma_commit(&bars->kv_empty[pend[T]]);
                        }
#pragma unroll
                        for (int k = 0; k < kHeadDim / 16; ++k)
                            umma_ss(tmem + col_s(T), make_sdesc(qaddr + T * kTileBytes + 32 * k, 16, 512, kSw64),
                                    make_sdesc(kaddr + 32 * k, 16, 512, kSw64), idesc_qk, k > 0);
                        umma_commit(&bars->s_full[T]);
                        pend[T] = st;
                    }
                }
                for (int T = 0; T < 2 && ok; ++T) {
                    if (pend[T] < 0) continue;
                    if (!mbar_wait(&bars->p_full[T], pph[T], ctl, 0x305 + T)) { ok = false; break; }
                    pph[T] ^= 1;
                    tc_fence_after();
                    issue_pv(T, pend[T]);
                    if (--readers[pend[T]] == 0) umma_commit(&bars->kv_empty[pend[T]]);
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
            const Item I = item_of(g, item);
            if (T == 1 && I.tB < 0) continue;
            const long long X = T ? I.tB : I.tA;
            const Slot me = slot_of(g, X, r);
            const long long myseg = seg_of(me.box);
            float o[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = 0.f;
            float m = -INFINITY, l = 0.f;
            bool first = true;
            for (int u = 0; u < I.nkv; ++u) {
                if (!active(g, I, T, u)) continue;
                const uint32_t allow = allow_mask(g, myseg, I.kv0 + u);
                const bool full = allow == ((1u << g.bpt) - 1u);
                if (!mbar_wait(&bars->s_full[T], sph, ctl, 0x401 + T)) { ok = false; break; }
                sph ^= 1;
                tc_fence_after();
                // pass 1: row maximum of the raw scores
                float mx8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) mx8[e] = -INFINITY;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t v[32];
                    tmem_ld32(t_s + 32 * c, v);
                    tmem_wait_ld();
                    if (full) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) mx8[e & 7] = fmaxf(mx8[e & 7], __uint_as_float(v[e]));
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const int kb = (32 * c + e) / g.BT;
                            if ((allow >> kb) & 1u) mx8[e & 7] = fmaxf(mx8[e & 7], __uint_as_float(v[e]));
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
                    for (int e = 0; e < 32; ++e) o[e] += __uint_as_float(v[e]);
                }
                if (m_tile > m + 8.f) {
                    const float alpha = ex2_approx(m - m_tile);
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] *= alpha;
                    l *= alpha;
                    m = m_tile;
                }
                const float mu = (m == -INFINITY) ? 0.f : m;
                // pass 2: probabilities, row sum, bf16 P into TMEM
                float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t v[32];
                    tmem_ld32(t_s + 32 * c, v);
                    tmem_wait_ld();
                    float p[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) p[e] = ex2_approx(fmaf(__uint_as_float(v[e]), sl2, -mu));
                    if (!full) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const int kb = (32 * c + e) / g.BT;
                            if (!((allow >> kb) & 1u)) p[e] = 0.f;
                        }
                    }
                    uint32_t w[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        l4[e & 3] += p[2 * e] + p[2 * e + 1];
                        w[e] = pack_bf16x2(p[2 * e], p[2 * e + 1]);
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
                for (int e = 0; e < 32; ++e) o[e] += __uint_as_float(v[e]);
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
                for (int i = 0; i < g.bpt; ++i) {
                    const Box bx = box_of(g, X * g.bpt + i);
                    if (bx.valid) tma_store_5d(&map_o, ost + i * g.BT * kRowBytes, 0, I.h, bx.col0, bx.row0, bx.b);
                }
                bulk_commit();
            }
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
