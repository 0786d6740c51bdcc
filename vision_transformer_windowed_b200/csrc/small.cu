// Kernels for windows of fewer than 128 tokens (M = 4, 8): a 128-slot tile
// then holds whole windows (several of them), so a work item is one (tile,
// head) and all of its attention stays inside the tile.
//
// At these sizes a window box of a shifted grid is as small as 4 x 4 tokens,
// too small for TMA box copies to keep up, so threads move token rows
// themselves (the forward's row warps, the backward's mover warp): coalesced
// 16-byte cp.async copies (8 whole 64-byte rows per warp instruction) issued
// one work item ahead, and coalesced 16-byte stores of the results.  Work items are (tile, head) with
// heads innermost while every head's RoPE table fits in shared memory, so the
// heads of a token, which are adjacent in memory, are read close together.
#include <cuda.h>
#include <cuda_runtime.h>

#include "dgeo.cuh"
#include "geometry.cuh"
#include "kernels.cuh"
#include "ptx.cuh"
#include "rows.cuh"

namespace fswin {

namespace smallk {

constexpr int kTabHeads = 4;            // resident cos/sin tables
constexpr int kTabPerHead = 2 * 8 * 8;  // [axis][pair][position < 8] float2

// Item -> (tile, head): heads innermost when all tables are resident.
__device__ __forceinline__ void small_item(const Geo& g, bool head_minor, long long it, long long* X, int* h) {
    const uint32_t i32 = static_cast<uint32_t>(it);
    if (head_minor) {
        const uint32_t x = fdiv(g.fd_heads, i32);
        *X = x;
        *h = static_cast<int>(i32 - x * static_cast<uint32_t>(g.heads));
    } else {
        const uint32_t hh = fdiv(g.fd_tiles, i32);
        *h = static_cast<int>(hh);
        *X = it - static_cast<long long>(hh) * g.tiles;
    }
}

// ------------------------------------------------------------------ backward
// Windows of fewer than 128 tokens (M = 4, 8) lie whole inside one 128-slot
// tile, so every gradient of a tile's tokens comes from that tile alone.  One
// persistent kernel then does the whole backward of a tile on chip, with no
// workspace round trip: only 4 x 16 d theta partials per tile leave it.
//   warps 0-3: thread = slot row.  D, lse and the RoPE of its q and k rows;
//              the row of P^T and dS^T of its key; the epilogue of its token
//              (dq, dk un-rotated, dv, the d theta terms), staged over the
//              slot's q, k, v rows.  Thread 0 also issues the MMAs:
//              S^T = K' Q'^T, dP^T = V dO^T right after the barrier that ends
//              the rotation, then dV = P^T dO, dK' = dS^T Q', dQ' = dS K' once
//              every warp has written P^T, dS^T and dS.
//   warp 4:    mover: the q, k, v, dO rows of each item (and its o rows) with
//              16-byte async copies one item ahead, completing on mbarriers (a
//              window box of a shifted grid is as small as 4 x 4 tokens, too
//              small for TMA box copies to keep up), and the stores of the
//              staged dq, dk, dv rows.
// Two CTAs share an SM (256 TMEM columns each).  Work items are (tile, head),
// heads innermost when their RoPE tables fit, so the heads of a token, which
// are adjacent in memory, are read close together in time.
namespace bwd {

constexpr int kThreads = 160;
constexpr int kWarpMover = 4;
constexpr int kSlotBytes = 4 * kTileBytes;        // q, k, v, dO tiles of one item
constexpr int kSlotOff = 0;                        // 2 slots
constexpr int kOOff = 2 * kSlotBytes;              // o tile
constexpr int kDSOff = kOOff + kTileBytes;         // dS (queries along M), MN-major 128-byte swizzle
constexpr int kVecOff = kDSOff + 4 * kTileBytes;   // lse2[128], D[128]
constexpr int kTabOff = kVecOff + 2 * kTile * 4;
constexpr int kBarOff = kTabOff + kTabHeads * kTabPerHead * 8;
constexpr int kSmemBytes = kBarOff + 256 + 1024;   // + alignment of the base
constexpr uint32_t kTmemCols = 256;
// TMEM columns: S^T [0,128), dP^T [128,256); P^T (bf16) over S^T [0,64), dS^T
// (fp16) over dP^T [128,192); the products over columns already consumed.
constexpr uint32_t kColS = 0, kColDP = 128, kColP = 0, kColDS = 128;
constexpr uint32_t kColDV = 64, kColDQ = 96, kColDK = 192;

struct Bars {
    uint64_t s_full, p_ready, mma2_done, grp, done;
    uint64_t slot_full[2], o_full, o_free, staged;  // row copies and stores (mover warp)
    float2 nrm[2][4];  // per item parity, per row warp: max |dO row|^2, max |v row|^2 (gradient scaling)
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Bars) <= 256, "barrier block overflows its slot");

struct Params {
    Geo g;
    const uint8_t *q, *k, *v, *o, *dout;  // bf16 [B, H, W, heads, 32]
    uint8_t *dq, *dk, *dv;
    const float *lse, *theta;
    float* part;  // [heads][tiles][16]
    unsigned int* dtheta_cnt;  // zeroed here for the d theta reduction launched next
    unsigned int* status;
    unsigned long long limit_ns;
    long long items;
    float scale;
    bool head_minor;
};

__global__ void __launch_bounds__(kThreads, 2) small_kernel(const __grid_constant__ Params prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars* bars = reinterpret_cast<Bars*>(smem + kBarOff);
    const Geo& g = prm.g;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (blockIdx.x == 0)  // the d theta reduction's counters, for its launch after this one
        for (int i = tid; i < g.heads; i += kThreads) prm.dtheta_cnt[i] = 0u;
    if (tid == 0) {
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->p_ready, 4);
        mbar_init(&bars->mma2_done, 1);
        mbar_init(&bars->grp, 4);
        mbar_init(&bars->done, 1);
        mbar_init(&bars->slot_full[0], 32);  // one cp.async arrival per mover lane
        mbar_init(&bars->slot_full[1], 32);
        mbar_init(&bars->o_full, 32);
        mbar_init(&bars->o_free, 4);
        mbar_init(&bars->staged, 4);
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
    // this CTA's items: blockIdx.x + j * gridDim.x, j < n
    // this CTA's items: a contiguous run, so that consecutive items are the
    // heads of one tile (heads innermost) and share the tile's geometry
    const long long per = (prm.items + gridDim.x - 1) / gridDim.x;
    const long long first = static_cast<long long>(blockIdx.x) * per;
    const long long n = prm.items > first ? (prm.items - first < per ? prm.items - first : per) : 0;
    auto item_at = [&](long long j) { return first + j; };

    if (warp == kWarpMover) {
        // ------------------------------------------------------------ row copies and result stores
        // Lane l moves 16-byte chunk l % 4 of row 8 i + l / 4 of each group of 32
        // rows: every instruction moves 8 whole 64-byte rows.  Copies arrive on an
        // mbarrier when they land (one arrival per lane); padding rows are zero
        // filled on load and skipped on store.
        bool ok = true;
        auto mwait = [&](uint64_t* bar, uint32_t ph, unsigned int where) -> bool {
            return __all_sync(0xFFFFFFFFu, mbar_wait(bar, ph, ctl, where));
        };
        // token (head 0) of rows lane + 32 q of the last tile seen
        long long mv_X = -1, mv_tok0[4] = {0, 0, 0, 0};
        bool mv_valid[4] = {false, false, false, false};
        auto geo4 = [&](long long j, int* h) {
            long long X;
            small_item(g, prm.head_minor, item_at(j), &X, h);
            if (X == mv_X) return;
            mv_X = X;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                int pi, pj;
                mv_valid[q] = slot_token(g, X, lane + 32 * q, 0, &pi, &pj, &mv_tok0[q]);
            }
        };
        // load (into the tiles) or store (from them) the rows of item j
        auto move = [&](long long j, const uint8_t* const* gsrc, uint8_t* const* gdst, uint8_t* const* tiles, int nt,
                        bool load) {
            int h;
            geo4(j, &h);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int sl_lane = 8 * i + (lane >> 2), c = lane & 3;
                    const long long tok = __shfl_sync(0xFFFFFFFFu, mv_tok0[q] + h, sl_lane);
                    const bool valid = __shfl_sync(0xFFFFFFFFu, mv_valid[q] ? 1 : 0, sl_lane) != 0;
                    const int row = 32 * q + sl_lane;
                    const uint32_t off = row * kRowBytes + ((c ^ ((row >> 1) & 3)) << 4);
                    const long long go = tok * kRowBytes + 16 * c;
                    for (int x = 0; x < nt; ++x) {
                        if (load)
                            cp_async16(smem_u32(tiles[x] + off), valid ? gsrc[x] + go : gsrc[x], valid ? 16u : 0u);
                        else if (valid)
                            *reinterpret_cast<uint4*>(gdst[x] + go) = *reinterpret_cast<const uint4*>(tiles[x] + off);
                    }
                }
            }
        };
        const uint8_t* qkvd[4] = {prm.q, prm.k, prm.v, prm.dout};
        const uint8_t* osrc[1] = {prm.o};
        uint8_t* grads[3] = {prm.dq, prm.dk, prm.dv};
        uint8_t* otile[1] = {smem + kOOff};
        auto slot_tiles = [&](long long j, uint8_t** t) {
            uint8_t* sl = smem + kSlotOff + (j & 1) * kSlotBytes;
            for (int x = 0; x < 4; ++x) t[x] = sl + x * kTileBytes;
        };
        uint8_t* st[4];
        if (n > 0) {
            slot_tiles(0, st);
            move(0, qkvd, nullptr, st, 4, true);
            cp_async_mbar_arrive(&bars->slot_full[0]);
            move(0, osrc, nullptr, otile, 1, true);
            cp_async_mbar_arrive(&bars->o_full);
        }
        if (n > 1) {
            slot_tiles(1, st);
            move(1, qkvd, nullptr, st, 4, true);
            cp_async_mbar_arrive(&bars->slot_full[1]);
        }
        for (long long j = 0; j < n && ok; ++j) {
            const uint32_t ph = static_cast<uint32_t>(j & 1);
            if (j + 1 < n) {  // the next item's o rows once the rows have read this item's
                if (!mwait(&bars->o_free, ph, 0x2401)) break;
                move(j + 1, osrc, nullptr, otile, 1, true);
                cp_async_mbar_arrive(&bars->o_full);
            }
            if (!mwait(&bars->staged, ph, 0x2402)) break;  // dq, dk, dv staged over the slot's q, k, v
            slot_tiles(j, st);
            move(j, nullptr, grads, st, 3, false);
            __syncwarp();  // every lane has read the staged rows: the slot takes item j+2's rows
            if (j + 2 < n) {
                move(j + 2, qkvd, nullptr, st, 4, true);
                cp_async_mbar_arrive(&bars->slot_full[j & 1]);
            }
        }
        cp_async_wait<0>();
    } else {
        // ------------------------------------------------------------ rows (warps 0-3)
        // thread 0 also issues the MMAs: S^T, dP^T once every row is rotated,
        // the gradients once every warp has written P^T, dS^T and dS
        const uint32_t id_s = make_idesc(kTile, kTile, false, false, true);     // fp16 K', Q'
        const uint32_t id_dp = make_idesc(kTile, kTile, false, false, false);   // bf16 V, dO
        const uint32_t id_dv = make_idesc(kTile, kHeadDim, false, true, false); // P^T (TMEM) x dO
        const uint32_t id_dk = make_idesc(kTile, kHeadDim, false, true, true);  // dS^T (TMEM) x Q'
        const uint32_t id_dq = make_idesc(kTile, kHeadDim, true, true, true);   // dS (smem) x K'
        const uint32_t sbase = smem_u32(smem);
        const uint64_t dK0 = make_sdesc(sbase, 16, 512, kSw64);        // K-major, 64-byte rows
        const uint64_t dMN0 = make_sdesc(sbase, 8192, 512, kSw64);     // MN-major, 64-byte rows
        const uint64_t dDS = make_sdesc(sbase + kDSOff, 16384, 1024, kSw128);
        const int r = tid;
        const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        const float sl2 = g.scale_log2;
        float* lse2v = reinterpret_cast<float*>(smem + kVecOff);
        float* dvec = lse2v + kTile;
        float2* tabs = reinterpret_cast<float2*>(smem + kTabOff);
        uint8_t* ds = smem + kDSOff;
        uint32_t gph = 0;
        bool ok = true;
        // Waits are warp-uniform, so that no warp-collective TMEM access runs on
        // a partial warp; the group barrier is an mbarrier with a bounded wait.
        auto wwait = [&](uint64_t* bar, uint32_t ph, unsigned int where) -> bool {
            return __all_sync(0xFFFFFFFFu, mbar_wait(bar, ph, ctl, where));
        };
        auto group_sync = [&](unsigned int where) -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->grp);
            const bool passed = wwait(&bars->grp, gph, where);
            gph ^= 1;
            return passed;
        };
        // This row's token in item j (invalid for padding windows), and the
        // item's 16-column masks for this row.
        struct RowTok {
            long long X, tok;
            int h, pi, pj;
            bool valid;
        };
        // geometry of this row in the last tile seen (shared by the tile's heads)
        long long geo_X = -1, geo_tok0 = 0;
        int geo_pi = 0, geo_pj = 0;
        bool geo_valid = false;
        uint32_t geo_a16 = 0;
        auto geo_for = [&](long long X) {
            if (X == geo_X) return;
            geo_X = X;
            geo_valid = slot_token(g, X, r, 0, &geo_pi, &geo_pj, &geo_tok0);  // token of head 0
            const uint64_t segs = d_tile_segs(g, X, d_tile_win(g, X));
            geo_a16 = allow16(g, seg_at(segs, r >> g.lBT), segs);  // bit c: columns [16c, 16c+16)
        };
        auto row_tok = [&](long long j) {
            RowTok t;
            small_item(g, prm.head_minor, item_at(j), &t.X, &t.h);
            geo_for(t.X);
            t.valid = geo_valid;
            t.tok = geo_tok0 + t.h;  // heads are innermost in the token layout
            t.pi = geo_pi;
            t.pj = geo_pj;
            return t;
        };
        auto row_mask = [&](const RowTok& t) {
            geo_for(t.X);
            return geo_a16;
        };
        RowTok cur = n > 0 ? row_tok(0) : RowTok{};
        int tab_head = -1;
        if (prm.head_minor) {  // every head's table, once
            for (int hh = 0; hh < g.heads; ++hh)
                build_small_table(tabs + hh * kTabPerHead, prm.theta + hh * 16, g.M, r, kTile);
            ok = group_sync(0x2301);
        }
        float lse_cur = (n > 0 && cur.valid) ? __ldg(prm.lse + cur.tok) : 0.f;
        uint32_t a16 = n > 0 ? row_mask(cur) : 0u;
        for (long long j = 0; j < n && ok; ++j) {
            const uint32_t ph = static_cast<uint32_t>(j & 1);
            const float2* tab = tabs;
            if (prm.head_minor) {
                tab = tabs + cur.h * kTabPerHead;
            } else if (cur.h != tab_head) {
                if (!group_sync(0x2302)) break;  // no row still rotates with the old table
                build_small_table(tabs, prm.theta + cur.h * 16, g.M, r, kTile);
                if (!group_sync(0x2303)) break;
                tab_head = cur.h;
            }
            uint8_t* sl = smem + kSlotOff + (j & 1) * kSlotBytes;
            if (!wwait(&bars->slot_full[j & 1], static_cast<uint32_t>((j >> 1) & 1), 0x2304) ||
                !wwait(&bars->o_full, ph, 0x2305))
                break;
            // D = dO . O of this row's token, and the squared norms of its dO and
            // v rows (the bound of the gradient scaling below); then the next
            // item's o rows
            float D = 0.f;
            {
                float a[32], b[32];
                load_row_swz(smem + kOOff, r, a, false);
                load_row_swz(sl + 3 * kTileBytes, r, b, false);
                float d4[4] = {0.f, 0.f, 0.f, 0.f};  // four independent partial sums
                float n4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    ffma2(d4[0], d4[1], a[e], a[e + 1], b[e], b[e + 1], d4[0], d4[1]);
                    ffma2(d4[2], d4[3], a[e + 2], a[e + 3], b[e + 2], b[e + 3], d4[2], d4[3]);
                    ffma2(n4[0], n4[1], b[e], b[e + 1], b[e], b[e + 1], n4[0], n4[1]);
                    ffma2(n4[2], n4[3], b[e + 2], b[e + 3], b[e + 2], b[e + 3], n4[2], n4[3]);
                }
                D = (d4[0] + d4[1]) + (d4[2] + d4[3]);
                const float ndo = warp_max_nonneg((n4[0] + n4[1]) + (n4[2] + n4[3]));
                const float nv = warp_max_nonneg(row_norm2(sl + 2 * kTileBytes, r));
                if (lane == 0) bars->nrm[ph][warp] = make_float2(ndo, nv);
            }
            __syncwarp();  // every lane has read its o row: the mover may load the next item's
            if (lane == 0) mbar_arrive(&bars->o_free);
            const RowTok nxt = j + 1 < n ? row_tok(j + 1) : RowTok{};
            dvec[r] = D;
            // RoPE of this row's q and k, bf16 in, fp16 out, in place
            {
                float x[32];
                load_row_swz(sl, r, x, false);
                rope32_small(x, cur.pi, cur.pj, tab, false);
                store_row_swz(sl, r, x, true);
                load_row_swz(sl + kTileBytes, r, x, false);
                rope32_small(x, cur.pi, cur.pj, tab, false);
                store_row_swz(sl + kTileBytes, r, x, true);
            }
            fence_proxy_async_smem();
            if (!group_sync(0x2306)) break;  // every row rotated; the previous item's products read by every warp
            if (r == 0) {
                tc_fence_after();
                const uint64_t qo = static_cast<uint64_t>((kSlotOff + (j & 1) * kSlotBytes) >> 4);
                const uint64_t ko = qo + (kTileBytes >> 4), vo = qo + (2 * kTileBytes >> 4), dof = qo + (3 * kTileBytes >> 4);
#pragma unroll
                for (int k = 0; k < kHeadDim / 16; ++k) umma_ss(tmem + kColS, dK0 + ko + 2 * k, dK0 + qo + 2 * k, id_s, k > 0);
#pragma unroll
                for (int k = 0; k < kHeadDim / 16; ++k)
                    umma_ss(tmem + kColDP, dK0 + vo + 2 * k, dK0 + dof + 2 * k, id_dp, k > 0);
                umma_commit(&bars->s_full);
            }
            // the tile's gradient scaling 2^e (GradScale in rows.cuh): lse2 - e makes the
            // probabilities 2^e P; every row's shifted lse2 is in place after the barrier,
            // which passes while the tensor core computes S^T and dP^T
            const int gexp = grad_scale_exp4(bars->nrm[ph]);
            lse2v[r] = cur.valid ? lse_cur * 1.4426950408889634f - static_cast<float>(gexp)
                                 : INFINITY;  // padding: no probability
            if (!group_sync(0x2309)) break;
            const float lse_nxt = (j + 1 < n && nxt.valid) ? __ldg(prm.lse + nxt.tok) : 0.f;
            // row of P^T and dS^T of this key, 32 query columns at a time
            if (!wwait(&bars->s_full, ph, 0x2307)) break;
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint8_t* base = ds + (c >> 1) * 16384 + (r >> 3) * 1024 + (r & 7) * 128;
                if (!__any_sync(0xFFFFFFFFu, ((a16 >> (2 * c)) & 3u) != 0u)) {  // P, dS = 0 for the whole warp
                    const uint32_t z[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                    tmem_st16(trow + kColP + 16 * c, z);
                    tmem_st16(trow + kColDS + 16 * c, z);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        *reinterpret_cast<uint4*>(base + (((4 * (c & 1) + q4) ^ (r & 7)) << 4)) = make_uint4(0, 0, 0, 0);
                    continue;
                }
                uint32_t sv[32], pv[32];
                tmem_ld32(trow + kColS + 32 * c, sv);
                tmem_ld32(trow + kColDP + 32 * c, pv);
                tmem_wait_ld();
                const bool ok0 = (a16 >> (2 * c)) & 1u, ok1 = (a16 >> (2 * c + 1)) & 1u;
                uint32_t wp[16], wd[16];
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4) {
                    float4 L4 = *reinterpret_cast<const float4*>(lse2v + 32 * c + 4 * e4);
                    const float4 D4 = *reinterpret_cast<const float4*>(dvec + 32 * c + 4 * e4);
                    if (!(e4 < 4 ? ok0 : ok1)) L4 = make_float4(INFINITY, INFINITY, INFINITY, INFINITY);
                    const int e = 4 * e4;
                    float t0, t1, t2, t3;
                    ffma2(t0, t1, __uint_as_float(sv[e]), __uint_as_float(sv[e + 1]), sl2, sl2, -L4.x, -L4.y);
                    ffma2(t2, t3, __uint_as_float(sv[e + 2]), __uint_as_float(sv[e + 3]), sl2, sl2, -L4.z, -L4.w);
                    const float p0 = ex2_approx(t0), p1 = ex2_approx(t1), p2 = ex2_approx(t2), p3 = ex2_approx(t3);
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
                // over columns of S^T and dP^T already read
                tmem_st16(trow + kColP + 16 * c, wp);
                tmem_st16(trow + kColDS + 16 * c, wd);
                // dS (queries along M, keys along K) as an MN-major operand
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const int cc = 4 * (c & 1) + q4;
                    *reinterpret_cast<uint4*>(base + ((cc ^ (r & 7)) << 4)) =
                        make_uint4(wd[4 * q4], wd[4 * q4 + 1], wd[4 * q4 + 2], wd[4 * q4 + 3]);
                }
            }
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->p_ready);
            if (r == 0 && mbar_wait(&bars->p_ready, ph, ctl, 0x2203)) {  // every warp's P^T, dS^T and dS written
                tc_fence_after();
                const uint64_t qo = static_cast<uint64_t>((kSlotOff + (j & 1) * kSlotBytes) >> 4);
                const uint64_t ko = qo + (kTileBytes >> 4), dof = qo + (3 * kTileBytes >> 4);
#pragma unroll
                for (int k = 0; k < kTile / 16; ++k)
                    umma_ts(tmem + kColDV, tmem + kColP + 8 * k, dMN0 + dof + 64 * k, id_dv, k > 0);
#pragma unroll
                for (int k = 0; k < kTile / 16; ++k)
                    umma_ts(tmem + kColDK, tmem + kColDS + 8 * k, dMN0 + qo + 64 * k, id_dk, k > 0);
#pragma unroll
                for (int k = 0; k < kTile / 16; ++k)
                    umma_ss(tmem + kColDQ, dDS + 128 * k, dMN0 + ko + 64 * k, id_dq, k > 0);
                umma_commit(&bars->mma2_done);
            }
            // the next item's masks while the MMAs run
            const uint32_t a16_nxt = j + 1 < n ? row_mask(nxt) : 0u;
            // epilogue of this row's token: dq, dk (un-rotated), dv, d theta terms
            if (!wwait(&bars->mma2_done, ph, 0x2308)) break;
            tc_fence_after();
            float part[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) part[e] = 0.f;
#pragma unroll 1
            for (int which = 0; which < 2; ++which) {  // 0: q side, 1: k side
                uint32_t t[32];
                tmem_ld32(trow + (which ? kColDK : kColDQ), t);
                tmem_wait_ld();
                float dx[32], x[32];
                // softmax scale, and the 2^e scaling undone (the exponent again from the
                // item's norms, which stay in place until item j + 2)
                const float sc = prm.scale * exp2i(-grad_scale_exp4(bars->nrm[ph]));
#pragma unroll
                for (int e = 0; e < 32; e += 2)
                    fmul2(dx[e], dx[e + 1], __uint_as_float(t[e]), __uint_as_float(t[e + 1]), sc, sc);
                uint8_t* tile = sl + which * kTileBytes;
                load_row_swz(tile, r, x, true);  // rotated q' or k' (fp16)
                // d theta: the pair's cross product is the same before and after the rotation
#pragma unroll
                for (int ax = 0; ax < 2; ++ax) {
                    const float pos = static_cast<float>(ax ? cur.pi : cur.pj);
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int a = ax * 16 + 2 * k, b = a + 1;
                        part[ax * 8 + k] = fmaf(pos, dx[b] * x[a] - dx[a] * x[b], part[ax * 8 + k]);
                    }
                }
                rope32_small(dx, cur.pi, cur.pj, tab, true);
                store_row_swz(tile, r, dx);  // dq or dk (bf16), staged over q' or k'
            }
            {
                uint32_t t[32];
                tmem_ld32(trow + kColDV, t);
                tmem_wait_ld();
                tc_fence_before();  // ordered before the next item's MMAs by its group barrier
                __syncwarp();
                float x[32];
                const float down = exp2i(-grad_scale_exp4(bars->nrm[ph]));
#pragma unroll
                for (int e = 0; e < 32; ++e) x[e] = __uint_as_float(t[e]) * down;
                store_row_swz(sl + 2 * kTileBytes, r, x);  // dv, staged over v
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->staged);  // the mover stores them
            // this warp's 16 d theta partials of the tile (summed in a fixed order
            // later): a butterfly that halves the values at each step, so that
            // lane pair (2c, 2c+1) ends with the warp sum of component c
            if (!cur.valid) {
#pragma unroll
                for (int e = 0; e < 16; ++e) part[e] = 0.f;
            }
#pragma unroll
            for (int half = 8, bit = 16; half >= 1; half >>= 1, bit >>= 1) {
                const bool upper = (lane & bit) != 0;
#pragma unroll
                for (int e = 0; e < half; ++e) {
                    const float send = upper ? part[e] : part[e + half];
                    const float keep = upper ? part[e + half] : part[e];
                    part[e] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, bit);
                }
            }
            part[0] += __shfl_xor_sync(0xFFFFFFFFu, part[0], 1);
            // component held by this lane: bits 4..1 of the lane, most significant first
            const int comp = ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1);
            if ((lane & 1) == 0)
                prm.part[((static_cast<long long>(cur.h) * g.tiles + cur.X) * 4 + warp) * 16 + comp] = part[0];
            cur = nxt;
            lse_cur = lse_nxt;
            a16 = a16_nxt;
        }
        if (r == 0) {  // every MMA issued here has completed before the columns are freed
            umma_commit(&bars->done);
            mbar_wait(&bars->done, 0, ctl, 0x22ff);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace bwd

// ------------------------------------------------------------------ forward
// One tile is the whole key set of its queries, so the softmax of a row is
// exact in one go (maximum, then probabilities and their sum) with no running
// rescale.  TMEM: S [0,128), P (bf16) over S [0,64), O over S [64,96): 128
// columns, so up to four CTAs share an SM.
//   warps 0-3: thread = slot row: copies, RoPE of its q and k rows, the
//              softmax of its query, the epilogue (O / l, log-sum-exp);
//              thread 0 also issues S = Q'K'^T right after the barrier that
//              ends the rotation, and O = P V once every warp has written P
//              (no separate MMA warp: each hand-off to one cost a wake-up)
namespace fwd {

constexpr int kThreads = 128;
constexpr int kSlotBytes = 3 * kTileBytes;  // q, k, v tiles of one item
constexpr int kSlotOff = 0;                  // 2 slots
constexpr int kTabOff = 2 * kSlotBytes;
constexpr int kBarOff = kTabOff + kTabHeads * kTabPerHead * 8;
constexpr int kSmemBytes = kBarOff + 256 + 1024;  // + alignment of the base
constexpr uint32_t kTmemCols = 128;
constexpr uint32_t kColS = 0, kColP = 0, kColO = 64;

struct Bars {
    uint64_t s_full, p_ready, o_full, grp, done;
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Bars) <= 256, "barrier block overflows its slot");

struct Params {
    Geo g;
    const uint8_t *q, *k, *v;  // bf16 [B, H, W, heads, 32]
    uint8_t* o;
    const float* theta;
    float* lse;  // [B, H, W, heads]
    unsigned int* status;
    unsigned long long limit_ns;
    long long items;
    bool head_minor;
};

__global__ void __launch_bounds__(kThreads, 4) fwd_kernel(const __grid_constant__ Params prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars* bars = reinterpret_cast<Bars*>(smem + kBarOff);
    const Geo& g = prm.g;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->p_ready, 4);
        mbar_init(&bars->o_full, 1);
        mbar_init(&bars->grp, 4);
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
    // this CTA's items: a contiguous run, so that consecutive items are the
    // heads of one tile (heads innermost) and share the tile's geometry
    const long long per = (prm.items + gridDim.x - 1) / gridDim.x;
    const long long first = static_cast<long long>(blockIdx.x) * per;
    const long long n = prm.items > first ? (prm.items - first < per ? prm.items - first : per) : 0;
    auto item_at = [&](long long j) { return first + j; };

    {
        // thread 0 also issues the MMAs (S = Q'K'^T once the four warps have
        // rotated their rows, O = P V once they have written P)
        const uint32_t id_s = make_idesc(kTile, kTile, false, false, true);     // fp16 Q', K'
        const uint32_t id_pv = make_idesc_bf16(kTile, kHeadDim, false, true);  // P (TMEM) x V
        const uint32_t sbase = smem_u32(smem);
        const uint64_t dK0 = make_sdesc(sbase, 16, 512, kSw64);     // K-major, 64-byte rows
        const uint64_t dMN0 = make_sdesc(sbase, 8192, 512, kSw64);  // MN-major, 64-byte rows
        // ------------------------------------------------------------ rows (warps 0-3)
        const int r = tid;
        const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        const float sl2 = g.scale_log2;
        float2* tabs = reinterpret_cast<float2*>(smem + kTabOff);
        uint32_t gph = 0;
        bool ok = true;
        auto wwait = [&](uint64_t* bar, uint32_t ph, unsigned int where) -> bool {
            return __all_sync(0xFFFFFFFFu, mbar_wait(bar, ph, ctl, where));
        };
        auto group_sync = [&](unsigned int where) -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->grp);
            const bool passed = wwait(&bars->grp, gph, where);
            gph ^= 1;
            return passed;
        };
        struct RowTok {
            long long X, tok;
            int h, pi, pj;
            bool valid;
        };
        // geometry of this row in the last tile seen (shared by the tile's heads)
        long long geo_X = -1, geo_tok0 = 0;
        int geo_pi = 0, geo_pj = 0;
        bool geo_valid = false;
        uint32_t geo_a16 = 0;
        auto geo_for = [&](long long X) {
            if (X == geo_X) return;
            geo_X = X;
            geo_valid = slot_token(g, X, r, 0, &geo_pi, &geo_pj, &geo_tok0);  // token of head 0
            const uint64_t segs = d_tile_segs(g, X, d_tile_win(g, X));
            geo_a16 = allow16(g, seg_at(segs, r >> g.lBT), segs);  // bit c: columns [16c, 16c+16)
        };
        auto row_tok = [&](long long j) {
            RowTok t;
            small_item(g, prm.head_minor, item_at(j), &t.X, &t.h);
            geo_for(t.X);
            t.valid = geo_valid;
            t.tok = geo_tok0 + t.h;  // heads are innermost in the token layout
            t.pi = geo_pi;
            t.pj = geo_pj;
            return t;
        };
        auto row_mask = [&](const RowTok& t) {
            geo_for(t.X);
            return geo_a16;
        };
        // coalesced copies of the warp's 32 rows of q, k, v (8 rows per instruction)
        auto copy_slot = [&](long long j, const RowTok& t) {
            uint8_t* sl = smem + kSlotOff + (j & 1) * kSlotBytes;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int sl_lane = 8 * i + (lane >> 2), c = lane & 3;
                const long long tok = __shfl_sync(0xFFFFFFFFu, t.tok, sl_lane);
                const bool valid = __shfl_sync(0xFFFFFFFFu, t.valid ? 1 : 0, sl_lane) != 0;
                const int row = warp * 32 + sl_lane;
                const uint32_t off = row * kRowBytes + ((c ^ ((row >> 1) & 3)) << 4);
                const long long go = tok * kRowBytes + 16 * c;
                cp_async16(smem_u32(sl + off), valid ? prm.q + go : prm.q, valid ? 16u : 0u);
                cp_async16(smem_u32(sl + kTileBytes + off), valid ? prm.k + go : prm.k, valid ? 16u : 0u);
                cp_async16(smem_u32(sl + 2 * kTileBytes + off), valid ? prm.v + go : prm.v, valid ? 16u : 0u);
            }
        };
        // commit groups: at the start of item j only item j+1's copies may be in flight
        RowTok cur = n > 0 ? row_tok(0) : RowTok{};
        if (n > 0) copy_slot(0, cur);
        cp_async_commit();
        if (n > 1) copy_slot(1, row_tok(1));
        cp_async_commit();
        int tab_head = -1;
        if (prm.head_minor) {  // every head's table, once
            for (int hh = 0; hh < g.heads; ++hh)
                build_small_table(tabs + hh * kTabPerHead, prm.theta + hh * 16, g.M, r, kTile);
            ok = group_sync(0x3301);
        }
        uint32_t a16 = n > 0 ? row_mask(cur) : 0u;
        for (long long j = 0; j < n && ok; ++j) {
            const uint32_t ph = static_cast<uint32_t>(j & 1);
            const float2* tab = tabs;
            if (prm.head_minor) {
                tab = tabs + cur.h * kTabPerHead;
            } else if (cur.h != tab_head) {
                if (!group_sync(0x3302)) break;  // no row still rotates with the old table
                build_small_table(tabs, prm.theta + cur.h * 16, g.M, r, kTile);
                if (!group_sync(0x3303)) break;
                tab_head = cur.h;
            }
            uint8_t* sl = smem + kSlotOff + (j & 1) * kSlotBytes;
            cp_async_wait<1>();
            __syncwarp();  // rows copied by other lanes of the warp
            // RoPE of this row's q and k, bf16 in, fp16 out, in place
            {
                float x[32];
                load_row_swz(sl, r, x, false);
                rope32_small(x, cur.pi, cur.pj, tab, false);
                store_row_swz(sl, r, x, true);
                load_row_swz(sl + kTileBytes, r, x, false);
                rope32_small(x, cur.pi, cur.pj, tab, false);
                store_row_swz(sl + kTileBytes, r, x, true);
            }
            fence_proxy_async_smem();
            if (!group_sync(0x3304)) break;  // every row rotated; the previous item's O read by every warp
            if (r == 0) {
                tc_fence_after();
                const uint64_t qo = static_cast<uint64_t>((kSlotOff + (j & 1) * kSlotBytes) >> 4);
                const uint64_t ko = qo + (kTileBytes >> 4);
#pragma unroll
                for (int k = 0; k < kHeadDim / 16; ++k) umma_ss(tmem + kColS, dK0 + qo + 2 * k, dK0 + ko + 2 * k, id_s, k > 0);
                umma_commit(&bars->s_full);
            }
            const RowTok nxt = j + 1 < n ? row_tok(j + 1) : RowTok{};
            // softmax of this query row: the maximum, then probabilities and their sum
            if (!wwait(&bars->s_full, ph, 0x3305)) break;
            tc_fence_after();
            float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                const uint32_t grp2 = (a16 >> (2 * c)) & 3u;  // this row's 16-column groups of the chunk
                if (!__any_sync(0xFFFFFFFFu, grp2 != 0u)) continue;  // no row of the warp attends them
                uint32_t v[32];
                tmem_ld32(trow + kColS + 32 * c, v);
                tmem_wait_ld();
                if (grp2 != 3u) {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (!((grp2 >> (e >> 4)) & 1u)) v[e] = __float_as_uint(-INFINITY);
                }
#pragma unroll
                for (int e = 0; e < 32; e += 2)
                    mx4[(e >> 1) & 3] = fmax3(mx4[(e >> 1) & 3], __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
            }
            const float m = fmaxf(fmax3(mx4[0], mx4[1], mx4[2]), mx4[3]) * sl2;  // a row always attends itself
            float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                if (!__any_sync(0xFFFFFFFFu, ((a16 >> (2 * c)) & 3u) != 0u)) {  // P = 0 for the whole warp
                    const uint32_t z[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                    tmem_st16(trow + kColP + 16 * c, z);
                    continue;
                }
                uint32_t v[32];
                tmem_ld32(trow + kColS + 32 * c, v);
                tmem_wait_ld();
                const float add0 = ((a16 >> (2 * c)) & 1u) ? -m : -INFINITY;
                const float add1 = ((a16 >> (2 * c + 1)) & 1u) ? -m : -INFINITY;
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
                tmem_st16(trow + kColP + 16 * c, w);  // over columns of S already read
            }
            const float l = (l4[0] + l4[1]) + (l4[2] + l4[3]);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->p_ready);
            if (r == 0 && mbar_wait(&bars->p_ready, ph, ctl, 0x3203)) {  // every warp's P written
                tc_fence_after();
                const uint64_t vo = static_cast<uint64_t>((kSlotOff + (j & 1) * kSlotBytes + 2 * kTileBytes) >> 4);
#pragma unroll
                for (int k = 0; k < kTile / 16; ++k) umma_ts(tmem + kColO, tmem + kColP + 8 * k, dMN0 + vo + 64 * k, id_pv, k > 0);
                umma_commit(&bars->o_full);
            }
            const uint32_t a16_nxt = j + 1 < n ? row_mask(nxt) : 0u;
            // epilogue: O / l into the staging rows (over q'), log-sum-exp
            if (!wwait(&bars->o_full, ph, 0x3306)) break;
            tc_fence_after();
            {
                uint32_t t[32];
                tmem_ld32(trow + kColO, t);
                tmem_wait_ld();
                tc_fence_before();  // ordered before the next item's S by its group barrier
                __syncwarp();
                const float inv = 1.f / l;
                float x[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) x[e] = __uint_as_float(t[e]) * inv;
                store_row_swz(sl, r, x);
            }
            if (cur.valid && prm.lse != nullptr)  // no lse: inference
                prm.lse[cur.tok] = (m + lg2_approx(l)) * 0.69314718055994530942f;
            __syncwarp();
            // coalesced stores of the warp's 32 rows of O (8 rows per instruction)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int sl_lane = 8 * i + (lane >> 2), c = lane & 3;
                const long long tok = __shfl_sync(0xFFFFFFFFu, cur.tok, sl_lane);
                const bool valid = __shfl_sync(0xFFFFFFFFu, cur.valid ? 1 : 0, sl_lane) != 0;
                const int row = warp * 32 + sl_lane;
                const uint32_t off = row * kRowBytes + ((c ^ ((row >> 1) & 3)) << 4);
                if (valid)
                    *reinterpret_cast<uint4*>(prm.o + tok * kRowBytes + 16 * c) = *reinterpret_cast<const uint4*>(sl + off);
            }
            __syncwarp();  // the staged rows are read: the slot takes item j+2's rows
            if (j + 2 < n) copy_slot(j + 2, row_tok(j + 2));
            cp_async_commit();
            cur = nxt;
            a16 = a16_nxt;
        }
        cp_async_wait<0>();
        if (r == 0) {  // every MMA issued here has completed before the columns are freed
            umma_commit(&bars->done);
            mbar_wait(&bars->done, 0, ctl, 0x32ff);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace fwd

}  // namespace smallk

cudaError_t launch_small_bwd(const Geo& g, const BwdPtrs& p, float* part, unsigned int* dtheta_cnt,
                             unsigned int* status, unsigned long long limit_ns, int num_sms, cudaStream_t stream) {
    using namespace smallk;
    static SmemOptIn optin;
    if (cudaError_t e = optin.ensure(reinterpret_cast<const void*>(bwd::small_kernel), bwd::kSmemBytes)) return e;
    bwd::Params sp;
    sp.g = g;
    sp.q = static_cast<const uint8_t*>(p.q);
    sp.k = static_cast<const uint8_t*>(p.k);
    sp.v = static_cast<const uint8_t*>(p.v);
    sp.o = static_cast<const uint8_t*>(p.o);
    sp.dout = static_cast<const uint8_t*>(p.dout);
    sp.dq = static_cast<uint8_t*>(p.dq);
    sp.dk = static_cast<uint8_t*>(p.dk);
    sp.dv = static_cast<uint8_t*>(p.dv);
    sp.lse = p.lse;
    sp.theta = p.theta;
    sp.part = part;
    sp.dtheta_cnt = dtheta_cnt;
    sp.status = status;
    sp.limit_ns = limit_ns;
    sp.items = static_cast<long long>(g.heads) * g.tiles;
    sp.scale = static_cast<float>(1.0 / 5.656854249492380195);  // 1/sqrt(32)
    sp.head_minor = g.heads <= kTabHeads;
    const long long grid = sp.items < 2ll * num_sms ? sp.items : 2ll * num_sms;  // two CTAs per SM
    bwd::small_kernel<<<static_cast<unsigned>(grid), bwd::kThreads, bwd::kSmemBytes, stream>>>(sp);
    return cudaGetLastError();
}

cudaError_t launch_small_fwd(const Geo& g, const void* q, const void* k, const void* v, const float* theta, void* o,
                             float* lse, unsigned int* status, unsigned long long limit_ns, int num_sms,
                             cudaStream_t stream) {
    using namespace smallk;
    static SmemOptIn optin;
    if (cudaError_t e = optin.ensure(reinterpret_cast<const void*>(fwd::fwd_kernel), fwd::kSmemBytes)) return e;
    fwd::Params fp;
    fp.g = g;
    fp.q = static_cast<const uint8_t*>(q);
    fp.k = static_cast<const uint8_t*>(k);
    fp.v = static_cast<const uint8_t*>(v);
    fp.o = static_cast<uint8_t*>(o);
    fp.theta = theta;
    fp.lse = lse;
    fp.status = status;
    fp.limit_ns = limit_ns;
    fp.items = static_cast<long long>(g.heads) * g.tiles;
    fp.head_minor = g.heads <= kTabHeads;
    const long long grid = fp.items < 4ll * num_sms ? fp.items : 4ll * num_sms;  // four CTAs per SM
    fwd::fwd_kernel<<<static_cast<unsigned>(grid), fwd::kThreads, fwd::kSmemBytes, stream>>>(fp);
    return cudaGetLastError();
}

}  // namespace fswin
