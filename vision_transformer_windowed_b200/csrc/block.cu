// Forward of the whole window-attention block of a Swin layer (inference) for
// windows of fewer than 128 tokens (M = 4, 8) and at most three heads:
//   qkv = x W_qkv^T + b_qkv, o_h = windowed RoPE attention of head h,
//   y = o W_o^T + b_o
// (the attention module of a FlashSwin block, thelatestinai.com 2610.04664,
// Figure 1B).  One persistent kernel: a work item is one 128-slot tile with
// all of its heads, so x is read and y written once per token, and q, k, v
// and o never leave the chip.  A CTA runs two items at a time (pipelines
// p = 0, 1: alternate items of its run), each with its own 256 TMEM columns,
// x buffer, head tiles, o tiles and barriers:
//   warps 4p .. 4p+3 (rows of pipeline p): thread = slot row = TMEM lane.
//       Per head: the biases and the RoPE of its q, k row (TMEM -> fp16 q',
//       k' and bf16 v tiles), the softmax of its query row, O / l into the
//       head's o tile; per item y + b_o into the staging tiles (the o tiles,
//       once read).  Row 0 of the pipeline also issues its MMAs, each as
//       soon as the rows' barrier before it passes: per head
//       q|k|v = x [W_q,h; W_k,h; W_v,h]^T (N = 96; the next head's right after
//       this head's S, so that it runs during the softmax), S = Q'K'^T,
//       O_h = P V; per item Y = sum_h O_h W_o[:, 32h:32h+32]^T.
//   warp 8 + p (mover of pipeline p): x rows in (16-byte cp.async) as soon as
//       the pipeline's x buffer is free, y rows out as soon as they are staged.
// The weights and biases stay in shared memory for the whole launch.
#include <cuda.h>
#include <cuda_runtime.h>

#include "dgeo.cuh"
#include "geometry.cuh"
#include "kernels.cuh"
#include "ptx.cuh"
#include "rows.cuh"

namespace fswin {

namespace blockk {

constexpr int kMaxHeads = 3;
constexpr int kPipes = 2;
constexpr int kThreads = 320;
constexpr int kWarpMover = 8;  // movers: warps 8 and 9
constexpr int kQkvRows = 3 * kHeadDim;  // q, k, v rows of one head in a W_qkv chunk tile

// Shared memory (offsets from a 1024-byte aligned base).  A weight "chunk" is
// the 32 input channels [32c, 32c + 32) of every output row, 64-byte rows,
// 64-byte swizzle (the K-major operand layout of the MMAs); the W_qkv chunk
// rows are ordered head by head, q, k, v rows of a head together.
constexpr int kWqkvChunk = kMaxHeads * kQkvRows * kRowBytes;  // 18 KB
constexpr int kWqkvOff = 0;
constexpr int kWoChunk = kMaxHeads * kHeadDim * kRowBytes;    // 6 KB
constexpr int kWoOff = kWqkvOff + kMaxHeads * kWqkvChunk;
// per pipeline: the x chunks of its item, a head's q' (fp16), k' (fp16), v
// (bf16) tiles, the heads' o tiles (then the y staging)
constexpr int kXBytes = kMaxHeads * kTileBytes;
constexpr int kPipeBytes = kXBytes + 3 * kTileBytes + kMaxHeads * kTileBytes;
constexpr int kPipeOff = kWoOff + kMaxHeads * kWoChunk;
constexpr int kPX = 0, kPHead = kXBytes, kPO = kXBytes + 3 * kTileBytes;
constexpr int kBiasOff = kPipeOff + kPipes * kPipeBytes;      // b_qkv [3C], b_o [C] (fp32)
constexpr int kTabPerHead = 2 * 8 * 8;                        // [axis][pair][position < 8] float2
constexpr int kTabOff = kBiasOff + 4 * kMaxHeads * kHeadDim * 4;
constexpr int kBarOff = kTabOff + kMaxHeads * kTabPerHead * 8;
constexpr int kSmemBytes = kBarOff + 512 + 1024;  // + alignment of the base
static_assert(kPipeOff % 1024 == 0 && kPipeBytes % 1024 == 0, "tile alignment");
static_assert(kWoOff % 1024 == 0 && kWqkvChunk % 1024 == 0 && kWoChunk % 512 == 0, "weight tile alignment");
static_assert(kSmemBytes <= 232448, "more shared memory than a CTA may have");

// TMEM columns of pipeline p, from 256 p: q|k|v of a head [0, 96) (then Y
// [0, C)), O_h [96, 128), S [128, 256) with P (bf16) over its consumed columns.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColQKV = 0, kColY = 0, kColO = 96, kColS = 128;

struct PipeBars {
    uint64_t x_full, x_free;                     // per item: x landed (32 mover lanes); last q|k|v MMAs done
    uint64_t qkv_full, s_full, p_ready, o_full;  // per head
    uint64_t o_ready, y_full, y_free, staged, y_done;      // per item
    uint64_t grp;                                          // the pipeline's four row warps
};
struct Bars {
    PipeBars pp[kPipes];
    uint64_t done;
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Bars) <= 512, "barrier block overflows its slot");

struct Params {
    Geo g;
    const uint8_t* x;  // bf16 [B, H, W, C]
    const uint8_t *w_qkv, *w_o;  // bf16 [3C, C], [C, C]
    const float *b_qkv, *b_o, *theta;
    uint8_t* y;  // bf16 [B, H, W, C]
    unsigned int* status;
    unsigned long long limit_ns;
    long long items;  // tiles
};

__global__ void __launch_bounds__(kThreads, 1) block_kernel(const __grid_constant__ Params prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars* bars = reinterpret_cast<Bars*>(smem + kBarOff);
    const Geo& g = prm.g;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int heads = g.heads, C = heads * kHeadDim;
    float* bias = reinterpret_cast<float*>(smem + kBiasOff);  // b_qkv [3C], then b_o at [3 * 96]
    float2* tabs = reinterpret_cast<float2*>(smem + kTabOff);

    if (tid == 0) {
        for (int p = 0; p < kPipes; ++p) {
            PipeBars& B = bars->pp[p];
            mbar_init(&B.x_full, 32);  // one arrival per mover lane, once its copies have landed
            mbar_init(&B.x_free, 1);
            mbar_init(&B.qkv_full, 1);
            mbar_init(&B.s_full, 1);
            mbar_init(&B.p_ready, 4);
            mbar_init(&B.o_full, 1);
            mbar_init(&B.o_ready, 4);
            mbar_init(&B.y_full, 1);
            mbar_init(&B.y_free, 4);
            mbar_init(&B.staged, 4);
            mbar_init(&B.y_done, 1);
            mbar_init(&B.grp, 4);
        }
        mbar_init(&bars->done, kPipes);  // each pipeline's MMA-issuing thread
        bars->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&bars->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    // weights (64-byte swizzled chunk tiles), biases and RoPE tables, once
    for (int i = tid; i < heads * 3 * C * 4; i += kThreads) {
        const int q16 = i & 3, rest = i >> 2;
        const int n = rest % (3 * C), c = rest / (3 * C);  // tile row n: head n / 96, then q, k, v rows
        const int hh = n / kQkvRows, part = (n % kQkvRows) / kHeadDim, e = n % kHeadDim;
        const size_t src = static_cast<size_t>(part * C + hh * kHeadDim + e) * C + 32 * c + 8 * q16;
        *reinterpret_cast<uint4*>(smem + kWqkvOff + c * kWqkvChunk + n * kRowBytes + ((q16 ^ ((n >> 1) & 3)) << 4)) =
            *reinterpret_cast<const uint4*>(prm.w_qkv + 2 * src);
    }
    for (int i = tid; i < heads * C * 4; i += kThreads) {
        const int q16 = i & 3, rest = i >> 2;
        const int n = rest % C, c = rest / C;
        const size_t src = static_cast<size_t>(n) * C + 32 * c + 8 * q16;
        *reinterpret_cast<uint4*>(smem + kWoOff + c * kWoChunk + n * kRowBytes + ((q16 ^ ((n >> 1) & 3)) << 4)) =
            *reinterpret_cast<const uint4*>(prm.w_o + 2 * src);
    }
    for (int i = tid; i < 3 * C; i += kThreads) bias[i] = prm.b_qkv[i];
    for (int i = tid; i < C; i += kThreads) bias[3 * kMaxHeads * kHeadDim + i] = prm.b_o[i];
    for (int hh = 0; hh < heads; ++hh) build_small_table(tabs + hh * kTabPerHead, prm.theta + hh * 16, g.M, tid, kThreads);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const Ctl ctl{prm.status, &bars->abort_flag, prm.limit_ns};
    // this CTA's items (tiles): a contiguous run; pipeline p takes its items p, p + 2, ...
    const long long per = (prm.items + gridDim.x - 1) / gridDim.x;
    const long long first = static_cast<long long>(blockIdx.x) * per;
    const long long n = prm.items > first ? (prm.items - first < per ? prm.items - first : per) : 0;
    auto pipe_base = [&](int p) { return smem + kPipeOff + p * kPipeBytes; };
    if (warp >= kWarpMover) {
        // ------------------------------------------------------------ x rows in, y rows out (pipeline p)
        // Lane l moves 16-byte chunk l % 4 of row 8 i + l / 4 of each group of 32
        // rows: every instruction moves 8 whole 64-byte rows of one chunk tile.
        const int p = warp - kWarpMover;
        PipeBars& B = bars->pp[p];
        uint8_t* pb = pipe_base(p);
        auto mwait = [&](uint64_t* bar, uint32_t ph, unsigned int where) -> bool {
            return __all_sync(0xFFFFFFFFu, mbar_wait(bar, ph, ctl, where));
        };
        long long mv_X = -1, mv_t[4] = {0, 0, 0, 0};  // token (B, H, W index) of rows lane + 32 q
        bool mv_valid[4] = {false, false, false, false};
        auto geo = [&](long long X) {
            if (X == mv_X) return;
            mv_X = X;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                int pi, pj;
                long long tok0;
                mv_valid[q] = slot_token(g, X, lane + 32 * q, 0, &pi, &pj, &tok0);
                mv_t[q] = tok0 / heads;
            }
        };
        // x rows of item j into the pipeline's x buffer; each lane waits for its
        // own copies and fences them for the tensor core (the async proxy)
        // before it arrives
        auto load = [&](long long j) {
            geo(first + j);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int sl_lane = 8 * i + (lane >> 2), cp = lane & 3;
                    const long long t = __shfl_sync(0xFFFFFFFFu, mv_t[q], sl_lane);
                    const bool valid = __shfl_sync(0xFFFFFFFFu, mv_valid[q] ? 1 : 0, sl_lane) != 0;
                    const int row = 32 * q + sl_lane;
                    const uint32_t off = row * kRowBytes + ((cp ^ ((row >> 1) & 3)) << 4);
                    const long long go = t * C * 2 + 16 * cp;
                    for (int c = 0; c < heads; ++c)
                        cp_async16(smem_u32(pb + kPX + c * kTileBytes + off), valid ? prm.x + go + 64 * c : prm.x,
                                   valid ? 16u : 0u);
                }
            }
            cp_async_commit();
            cp_async_wait<0>();
            fence_proxy_async_smem();
            mbar_arrive(&B.x_full);
        };
        // y rows of item j from the staging tiles: per group of 32 rows, all
        // shared loads first, then the global stores
        auto store = [&](long long j) {
            geo(first + j);
            const uint32_t s0 = smem_u32(pb + kPO);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint4 v[4][kMaxHeads];
                long long go[4];
                bool valid[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int sl_lane = 8 * i + (lane >> 2), cp = lane & 3;
                    go[i] = __shfl_sync(0xFFFFFFFFu, mv_t[q], sl_lane) * C * 2 + 16 * cp;
                    valid[i] = __shfl_sync(0xFFFFFFFFu, mv_valid[q] ? 1 : 0, sl_lane) != 0;
                    const int row = 32 * q + sl_lane;
                    const uint32_t off = row * kRowBytes + ((cp ^ ((row >> 1) & 3)) << 4);
#pragma unroll
                    for (int c = 0; c < kMaxHeads; ++c)
                        if (c < heads) v[i][c] = ld_shared_v4(s0 + c * kTileBytes + off);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    if (valid[i]) {
#pragma unroll
                        for (int c = 0; c < kMaxHeads; ++c)
                            if (c < heads) st_global_v4(prm.y + go[i] + 64 * c, v[i][c]);
                    }
            }
        };
        const long long count = p < n ? (n - p + 1) / 2 : 0;  // the pipeline's items: p, p + 2, ...
        if (count > 0) load(p);
        for (long long jj = 0; jj < count; ++jj) {
            if (jj + 1 < count) {  // the next item's x once this item's q|k|v MMAs are done with the buffer
                if (!mwait(&B.x_free, static_cast<uint32_t>(jj & 1), 0x5401)) break;
                load(p + 2 * (jj + 1));
            }
            if (!mwait(&B.staged, static_cast<uint32_t>(jj & 1), 0x5402)) break;
            store(p + 2 * jj);
            __syncwarp();  // every lane has read the staged rows
            if (lane == 0) mbar_arrive(&B.y_done);
        }
        cp_async_wait<0>();
    } else {
        // ------------------------------------------------------------ rows (warps 0-7)
        const int p = warp >> 2, wq = warp & 3;
        const int r = wq * 32 + lane;
        PipeBars& B = bars->pp[p];
        uint8_t* pb = pipe_base(p);
        const uint32_t trow = tmem + 256 * p + (static_cast<uint32_t>(wq * 32) << 16);
        const float sl2 = g.scale_log2;
        uint8_t* qt = pb + kPHead;
        uint8_t* kt = qt + kTileBytes;
        uint8_t* vt = qt + 2 * kTileBytes;
        uint32_t gph = 0, hc = 0;
        bool ok = true;
        // thread 0 of the pipeline issues its MMAs: per head q|k|v (the next
        // head's right after this head's S), S = Q'K'^T once every row is
        // rotated, O_h = P V once every warp has written P; per item Y
        const bool issuer = r == 0;
        const uint32_t id_qkv = make_idesc(kTile, kQkvRows, false, false, false);  // bf16 x, W_qkv
        const uint32_t id_s = make_idesc(kTile, kTile, false, false, true);         // fp16 Q', K'
        const uint32_t id_pv = make_idesc(kTile, kHeadDim, false, true, false);     // P (TMEM) x V, bf16
        const uint32_t id_y = make_idesc(kTile, C, false, false, false);            // bf16 O, W_o
        const uint32_t sbase = smem_u32(smem);
        const uint64_t dK0 = make_sdesc(sbase, 16, 512, kSw64);     // K-major, 64-byte rows
        const uint64_t dMN0 = make_sdesc(sbase, 8192, 512, kSw64);  // MN-major, 64-byte rows
        auto u16 = [](int bytes) { return static_cast<uint64_t>(bytes >> 4); };
        const uint32_t tb = tmem + 256 * p;
        const int pbo = kPipeOff + p * kPipeBytes;
        // q|k|v of head h: x (its chunk tiles) times the head's 96 W_qkv rows
        auto issue_qkv = [&](int h) {
            for (int c = 0; c < heads; ++c)
#pragma unroll
                for (int ks = 0; ks < 2; ++ks)
                    umma_ss(tb + kColQKV, dK0 + u16(pbo + kPX + c * kTileBytes) + 2 * ks,
                            dK0 + u16(kWqkvOff + c * kWqkvChunk + h * kQkvRows * kRowBytes) + 2 * ks, id_qkv,
                            (c | ks) != 0);
            umma_commit(&B.qkv_full);
            // the last head's q|k|v is the last MMA that reads the item's x:
            // the mover may refill the buffer once it completes
            if (h == heads - 1) umma_commit(&B.x_free);
        };
        auto wwait = [&](uint64_t* bar, uint32_t ph, unsigned int where) -> bool {
            return __all_sync(0xFFFFFFFFu, mbar_wait(bar, ph, ctl, where));
        };
        auto group_sync = [&](unsigned int where) -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(&B.grp);
            const bool passed = wwait(&B.grp, gph, where);
            gph ^= 1;
            return passed;
        };
        for (long long jj = 0; p + 2 * jj < n && ok; ++jj) {
            const long long X = first + p + 2 * jj;
            int pi, pj;
            long long tok0;
            slot_token(g, X, r, 0, &pi, &pj, &tok0);
            const uint64_t segs = d_tile_segs(g, X, d_tile_win(g, X));
            const uint32_t a16 = allow16(g, seg_at(segs, r >> g.lBT), segs);  // bit c: columns [16c, 16c+16)
            if (issuer) {  // the item's x landed; every row has read the previous Y
                if (!mbar_wait(&B.x_full, static_cast<uint32_t>(jj & 1), ctl, 0x5201) ||
                    (jj > 0 && !mbar_wait(&B.y_free, static_cast<uint32_t>((jj - 1) & 1), ctl, 0x5202))) {
                    ok = false;
                } else {
                    tc_fence_after();
                    issue_qkv(0);
                }
            }
            for (int h = 0; h < heads && ok; ++h, ++hc) {
                const uint32_t ph = hc & 1u;
                const float2* tab = tabs + h * kTabPerHead;
                // q, k, v of this row and head: + biases, RoPE of q and k, into the head's tiles
                if (!wwait(&B.qkv_full, ph, 0x5301)) { ok = false; break; }
                tc_fence_after();
#pragma unroll 1
                for (int part = 0; part < 3; ++part) {
                    uint32_t t[32];
                    tmem_ld32(trow + kColQKV + 32 * part, t);
                    tmem_wait_ld();
                    const float* b = bias + part * C + h * kHeadDim;
                    float x[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) x[e] = __uint_as_float(t[e]) + b[e];
                    if (part < 2) rope32_small(x, pi, pj, tab, false);
                    store_row_swz(part == 0 ? qt : (part == 1 ? kt : vt), r, x, part < 2);  // q', k' fp16; v bf16
                }
                tc_fence_before();
                fence_proxy_async_smem();
                if (!group_sync(0x5302)) { ok = false; break; }  // every row's q', k', v written, its q|k|v read
                if (issuer) {
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < kHeadDim / 16; ++ks)
                        umma_ss(tb + kColS, dK0 + u16(pbo + kPHead) + 2 * ks,
                                dK0 + u16(pbo + kPHead + kTileBytes) + 2 * ks, id_s, ks > 0);
                    umma_commit(&B.s_full);
                    if (h + 1 < heads) issue_qkv(h + 1);  // during this head's softmax
                }
                // softmax of this query row: the maximum, then probabilities and their sum
                if (!wwait(&B.s_full, ph, 0x5303)) { ok = false; break; }
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
                        tmem_st16(trow + kColS + 16 * c, z);
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
                    tmem_st16(trow + kColS + 16 * c, w);  // P over columns of S already read
                }
                const float l = (l4[0] + l4[1]) + (l4[2] + l4[3]);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&B.p_ready);
                if (issuer && mbar_wait(&B.p_ready, ph, ctl, 0x5203)) {  // every warp's P written
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < kTile / 16; ++k)
                        umma_ts(tb + kColO, tb + kColS + 8 * k, dMN0 + u16(pbo + kPHead + 2 * kTileBytes) + 64 * k,
                                id_pv, k > 0);
                    umma_commit(&B.o_full);
                }
                // O_h / l into the head's o tile
                if (!wwait(&B.o_full, ph, 0x5304)) { ok = false; break; }
                tc_fence_after();
                uint32_t t[32];
                tmem_ld32(trow + kColO, t);
                tmem_wait_ld();
                tc_fence_before();
                // the pipeline's previous y rows, staged over the o tiles, are stored
                if (h == 0 && jj > 0 && !wwait(&B.y_done, static_cast<uint32_t>((jj - 1) & 1), 0x5305)) {
                    ok = false;
                    break;
                }
                const float inv = 1.f / l;
                float x[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) x[e] = __uint_as_float(t[e]) * inv;
                store_row_swz(pb + kPO + h * kTileBytes, r, x);
            }
            if (!ok) break;
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&B.o_ready);
            if (issuer && mbar_wait(&B.o_ready, static_cast<uint32_t>(jj & 1), ctl, 0x5204)) {  // every o tile written
                tc_fence_after();
                for (int h = 0; h < heads; ++h)
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks)
                        umma_ss(tb + kColY, dK0 + u16(pbo + kPO + h * kTileBytes) + 2 * ks,
                                dK0 + u16(kWoOff + h * kWoChunk) + 2 * ks, id_y, (h | ks) != 0);
                umma_commit(&B.y_full);
            }
            // y = Y + b_o into the staging tiles (the o tiles, read by the finished Y MMAs)
            if (!wwait(&B.y_full, static_cast<uint32_t>(jj & 1), 0x5306)) break;
            tc_fence_after();
            for (int c = 0; c < heads; ++c) {
                uint32_t t[32];
                tmem_ld32(trow + kColY + 32 * c, t);
                tmem_wait_ld();
                const float* b = bias + 3 * kMaxHeads * kHeadDim + 32 * c;
                float x[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) x[e] = __uint_as_float(t[e]) + b[e];
                store_row_swz(pb + kPO + c * kTileBytes, r, x);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&B.y_free);
                mbar_arrive(&B.staged);  // the mover stores them
            }
        }
        if (issuer) {  // every MMA issued here has completed before the columns are freed
            umma_commit(&bars->done);
            mbar_wait(&bars->done, 0, ctl, 0x52ff);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace blockk

cudaError_t launch_block_fwd(const Geo& g, const BlockPtrs& p, unsigned int* status, unsigned long long limit_ns,
                             int num_sms, cudaStream_t stream) {
    using namespace blockk;
    static SmemOptIn optin;
    if (cudaError_t e = optin.ensure(reinterpret_cast<const void*>(block_kernel), kSmemBytes)) return e;
    Params prm;
    prm.g = g;
    prm.x = static_cast<const uint8_t*>(p.x);
    prm.w_qkv = static_cast<const uint8_t*>(p.w_qkv);
    prm.w_o = static_cast<const uint8_t*>(p.w_o);
    prm.b_qkv = p.b_qkv;
    prm.b_o = p.b_o;
    prm.theta = p.theta;
    prm.y = static_cast<uint8_t*>(p.y);
    prm.status = status;
    prm.limit_ns = limit_ns;
    prm.items = g.tiles;
    const long long grid = prm.items < num_sms ? prm.items : num_sms;
    if (grid <= 0) return cudaSuccess;
    block_kernel<<<static_cast<unsigned>(grid), kThreads, kSmemBytes, stream>>>(prm);
    return cudaGetLastError();
}

}  // namespace fswin
