// Windowed attention with a low-rank additive bias: heads of d = 32 channels,
// every window size, optional window-local RoPE.
//
// The bias of head h is U_h W_h^T over window-local positions t = i M + j (the
// factors are fp32 [M*M][16], shared by every window of the batch).  It joins the
// score product as 16 more contraction channels: a query tile's second half tile
// holds sqrt(d) U_t (fp16) and a key tile's holds W_u, so one K = 48 product
// gives q'.k' + sqrt(d) U_t.W_u, which the softmax scale 1/sqrt(d) turns into
// scale q'.k' + U_t.W_u.  The second half tiles are laid out like any 32-channel
// tile (64-byte rows, 64-byte swizzle) with channels 16..31 zero, so the
// gradient products dQ~ = dS K~ and dK~ = dS^T Q~ also carry, in their second
// halves, the window's shares sum_u dS_tu W_u of dU_t and sum_t dS_tu U_t of dW_u.
// A fixed-order two-level sum over the windows of the batch turns the shares
// into dU and dW.
//
// Kernels (plain one-tile pipelines: one CTA of row warps walks its work items,
// four in the forward, eight in the backward's main kernel; thread 0 issues the
// MMAs):
//   forward:  item = (query tile, head); the key tiles of its group in turn,
//             online softmax with O in registers;
//   backward: prep (per tile and head: the largest |dO row| and |v row| for the
//             gradient scaling, zeroed accumulator rows), main (item = (key tile,
//             head); the query tiles of its group in turn: S^T, dP^T, P'^T and
//             dS'^T, dV and dK~ accumulated in TMEM, dQ~ added with 16-byte fp32
//             vector reductions into the query rows' accumulator rows; at the
//             item's end dk, dv, the key side of d theta and the dW shares),
//             post (dq and the query side of d theta), the fixed-order d theta
//             sum of the other backward kernels, and the dU / dW sum.
// Accumulator row of a (head, tile, slot), 64 fp32: [0, 32) dQ', [32, 48) the
// slot's dU share, [48, 64) its dW share.
#include <cuda.h>
#include <cuda_runtime.h>

#include "dgeo.cuh"
#include "geometry.cuh"
#include "kernels.cuh"
#include "ptx.cuh"
#include "rows.cuh"
#include "schedule.cuh"

namespace fswin {

namespace lrbk {

constexpr int kPairs = 8;                       // RoPE pairs per axis (d = 32)
constexpr int kTabBytes = 2 * kPairs * 64 * 8;  // [axis][pair][position < 64] float2
constexpr float kSqrtD = 5.656854249492380195f; // sqrt(32): the query factor's pre-scale
constexpr int kWinChunk = 16;                   // windows per first-level dU / dW sum

// cos/sin of pos * theta[h][axis][k], pos < M, as [axis * 8 + k][64 positions].
__device__ __forceinline__ void build_table(float2* tab, const float* theta_h, int M, int t, int nt) {
    for (int e = t; e < 2 * kPairs * M; e += nt) {
        const int ak = e / M, pos = e - ak * M;
        float sn, cs;
        sincosf(static_cast<float>(pos) * theta_h[ak], &sn, &cs);
        tab[ak * 64 + pos] = make_float2(cs, sn);
    }
}

// Rotates (inv: un-rotates) a 32-channel row: pairs of channels 0..15 by the
// column position j, pairs of channels 16..31 by the row position i.
__device__ __forceinline__ void rope_row(float (&x)[32], int i, int j, const float2* tab, bool inv) {
#pragma unroll
    for (int ax = 0; ax < 2; ++ax) {
        const int pos = ax ? i : j;
#pragma unroll
        for (int k = 0; k < kPairs; ++k) {
            const float2 cs = tab[(ax * kPairs + k) * 64 + pos];
            const float sn = inv ? -cs.y : cs.y;
            const float a = x[ax * 16 + 2 * k], b = x[ax * 16 + 2 * k + 1];
            x[ax * 16 + 2 * k] = a * cs.x - b * sn;
            x[ax * 16 + 2 * k + 1] = a * sn + b * cs.x;
        }
    }
}

// cp.async copies of the warp's 32 rows of a [.., 32] bf16 tensor into a tile:
// lane l moves 16-byte chunk l % 4 of rows l / 4 + 8 i, so each instruction
// moves eight whole 64-byte rows.  tok / valid: this lane's own row.
__device__ __forceinline__ void copy_rows(uint8_t* tile, const uint8_t* src, long long tok, bool valid, int warp,
                                          int lane) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int rl = (lane >> 2) + 8 * i, c = lane & 3;
        const long long tk = __shfl_sync(0xFFFFFFFFu, tok, rl);
        const bool vd = __shfl_sync(0xFFFFFFFFu, valid ? 1 : 0, rl) != 0;
        const int row = warp * 32 + rl;
        uint8_t* dst = tile + row * kRowBytes + ((c ^ ((row >> 1) & 3)) << 4);
        cp_async16(smem_u32(dst), vd ? src + tk * kRowBytes + 16 * c : src, vd ? 16u : 0u);
    }
}

// Coalesced 16-byte stores of the warp's 32 staged rows (valid ones only).
__device__ __forceinline__ void store_rows(uint8_t* dst, const uint8_t* tile, long long tok, bool valid, int warp,
                                           int lane) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int rl = (lane >> 2) + 8 * i, c = lane & 3;
        const long long tk = __shfl_sync(0xFFFFFFFFu, tok, rl);
        const bool vd = __shfl_sync(0xFFFFFFFFu, valid ? 1 : 0, rl) != 0;
        const int row = warp * 32 + rl;
        const uint8_t* s = tile + row * kRowBytes + ((c ^ ((row >> 1) & 3)) << 4);
        if (vd) *reinterpret_cast<uint4*>(dst + tk * kRowBytes + 16 * c) = *reinterpret_cast<const uint4*>(s);
    }
}

// A factor row's 16 fp32 values, loaded into registers (no wait here).
__device__ __forceinline__ void load_factor(float4 (&f)[4], const float* src) {
    const float4* p = reinterpret_cast<const float4*>(src);
#pragma unroll
    for (int c = 0; c < 4; ++c) f[c] = __ldg(p + c);
}

// Row r of a factor half tile: mul * f as fp16 in channels 0..15, zeros in 16..31.
__device__ __forceinline__ void put_factor(uint8_t* tile, int r, const float4 (&f)[4], float mul) {
    float x[32];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        x[4 * c] = f[c].x * mul;
        x[4 * c + 1] = f[c].y * mul;
        x[4 * c + 2] = f[c].z * mul;
        x[4 * c + 3] = f[c].w * mul;
    }
#pragma unroll
    for (int e = 16; e < 32; ++e) x[e] = 0.f;
    store_row_swz(tile, r, x, true);
}

// Row r of a staged bf16 q or k tile to fp16, rotated when a table is given.
__device__ __forceinline__ void prep_row(uint8_t* tile, int r, int i, int j, const float2* tab) {
    float x[32];
    load_row_swz(tile, r, x, false);
    if (tab) rope_row(x, i, j, tab, false);
    store_row_swz(tile, r, x, true);
}

__device__ __forceinline__ void load_row32(const uint8_t* base, long long tok, float (&a)[32]) {
    const uint4* p = reinterpret_cast<const uint4*>(base + tok * kRowBytes);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint4 v = p[c];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            a[8 * c + 2 * e] = bf16lo_to_f32(w[e]);
            a[8 * c + 2 * e + 1] = bf16hi_to_f32(w[e]);
        }
    }
}

// ------------------------------------------------------------------ forward
namespace fwd {

constexpr int kThreads = 128;
constexpr int kKVBufs = 3;                        // key buffers: staged, in the score product, in P V
constexpr int kQOff = 0;                          // Q~ half tiles: q' and sqrt(d) U (then the staged O)
constexpr int kKVOff = kQOff + 2 * kTileBytes;    // key buffers: K~ half tiles (k', W), V tile
constexpr int kKVBytes = 3 * kTileBytes;
constexpr int kTabOff = kKVOff + kKVBufs * kKVBytes;
constexpr int kBarOff = kTabOff + kTabBytes;
constexpr int kSmemBytes = kBarOff + 256 + 1024;  // + alignment of the base
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kSBuf = 128;                   // two S buffers, at columns 0 and 128
constexpr uint32_t kColP = 0, kColO = 64;         // within an S buffer: bf16 P, then the tile's P V

struct Bars {
    uint64_t s_full, o_full, grp, done;
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Bars) <= 256, "barrier block overflows its slot");

struct Params {
    Geo g;
    const uint8_t *q, *k, *v;  // bf16 [B, H, W, heads, 32]
    uint8_t* o;
    const float* theta;        // [heads][2][8], or null: no rotation
    const float *u, *w;        // [heads][M*M][16]
    float* lse;                // [B, H, W, heads] or null
    unsigned int* status;
    unsigned long long limit_ns;
    long long items;
};

// The loop over an item's key tiles keeps one product in flight behind the
// softmax: tile u's P V goes to the spare columns of u's S buffer, and the next
// tile's S goes to the other buffer.  Thread 0 issues both in order, so when the
// softmax sees tile u+1's S complete, tile u's P V is complete too (a commit
// covers every earlier product of its thread) and is added to the O registers
// then; only an item's last P V has a barrier of its own.  The key buffers
// rotate over three: while tile u's S is computed, tile u+1's rows are copied
// into the buffer of tile u-2, whose P V completed before tile u-1's softmax.
__global__ void __launch_bounds__(kThreads, 2) fwd_kernel(const __grid_constant__ Params prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars* bars = reinterpret_cast<Bars*>(smem + kBarOff);
    const Geo& g = prm.g;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, r = tid;

    if (tid == 0) {
        mbar_init(&bars->s_full, 1);
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
    const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const Ctl ctl{prm.status, &bars->abort_flag, prm.limit_ns};
    const uint32_t id_s = make_idesc(kTile, kTile, false, false, true);    // fp16 Q~, K~
    const uint32_t id_pv = make_idesc_bf16(kTile, kHeadDim, false, true);  // P (TMEM) x V
    const uint32_t sbase = smem_u32(smem);
    const uint64_t dK0 = make_sdesc(sbase, 16, 512, kSw64);     // K-major, 64-byte rows
    const uint64_t dMN0 = make_sdesc(sbase, 8192, 512, kSw64);  // MN-major, 64-byte rows
    const float sl2 = g.scale_log2;
    float2* tab = reinterpret_cast<float2*>(smem + kTabOff);
    const float2* rtab = prm.theta ? tab : nullptr;
    uint8_t* q0 = smem + kQOff;
    uint8_t* q1 = q0 + kTileBytes;
    uint32_t gph = 0, sph = 0, oph = 0, tcs = 0;  // tcs: tiles whose S was issued; S buffer tcs & 1
    int tab_head = -1;
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

    for (long long it = blockIdx.x; it < prm.items && ok; it += gridDim.x) {
        const FwdItem I = d_fwd_item(g, it);
        if (rtab && I.h != tab_head) {
            if (!group_sync(0x6301)) break;  // no row still rotates with the old table
            build_table(tab, prm.theta + I.h * 2 * kPairs, g.M, r, kThreads);
            if (!group_sync(0x6302)) break;
            tab_head = I.h;
        }
        const float* uh = prm.u + static_cast<long long>(I.h) * g.N * 16;
        const float* wh = prm.w + static_cast<long long>(I.h) * g.N * 16;
        // this thread's query row, its token and its segment byte
        int pi, pj;
        long long qtok;
        const bool qvalid = slot_token(g, I.X, r, I.h, &pi, &pj, &qtok);
        const uint32_t myseg = I.masked ? seg_at(d_tile_segs(g, I.X, I.win), r >> g.lBT) : 0u;
        if (!group_sync(0x6303)) break;  // the previous item's staged O rows are stored
        // A key tile's K, V rows (copies) and key factor row (loads into
        // registers, written to the tile when the tile is prepared).
        auto kv_stage = [&](int u, int b, int& ki, int& kj, float4 (&f)[4]) {
            long long ktok;
            const bool kvalid = slot_token(g, I.kv0 + u, r, I.h, &ki, &kj, &ktok);
            uint8_t* kb = smem + kKVOff + b * kKVBytes;
            copy_rows(kb, prm.k, ktok, kvalid, warp, lane);
            copy_rows(kb + 2 * kTileBytes, prm.v, ktok, kvalid, warp, lane);
            cp_async_commit();
            load_factor(f, wh + (ki * g.M + kj) * 16);
        };
        auto next_kv = [&](int u) {
            while (u < I.nkv && !((I.act >> u) & 1u)) ++u;
            return u;
        };
        copy_rows(q0, prm.q, qtok, qvalid, warp, lane);
        cp_async_commit();
        float4 fq[4], fk[4];
        load_factor(fq, uh + (pi * g.M + pj) * 16);
        int u = next_kv(0), b = 0, ki = 0, kj = 0;
        if (u < I.nkv) kv_stage(u, 0, ki, kj, fk);
        put_factor(q1, r, fq, kSqrtD);
        cp_async_wait<0>();
        __syncwarp();
        prep_row(q0, r, pi, pj, rtab);
        float o[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = 0.f;
        float m = -INFINITY, l = 0.f;
        bool first = true;
        while (u < I.nkv && ok) {
            const long long kt = I.kv0 + u;
            const int un = next_kv(u + 1);
            const int koff = kKVOff + b * kKVBytes;
            const uint32_t sb = (tcs & 1u) * kSBuf;
            cp_async_wait<0>();
            __syncwarp();
            prep_row(smem + koff, r, ki, kj, rtab);
            put_factor(smem + koff + kTileBytes, r, fk, 1.f);
            fence_proxy_async_smem();
            if (!group_sync(0x6304)) { ok = false; break; }  // every Q~ and K~ row staged, P V rows read
            if (r == 0) {
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < kHeadDim / 16; ++k)  // q'.k'
                    umma_ss(tmem + sb, dK0 + (kQOff >> 4) + 2 * k, dK0 + (koff >> 4) + 2 * k, id_s, k > 0);
                // sqrt(d) U.W: the 16 factor channels only
                umma_ss(tmem + sb, dK0 + ((kQOff + kTileBytes) >> 4), dK0 + ((koff + kTileBytes) >> 4), id_s, 1u);
                umma_commit(&bars->s_full);
            }
            int nki = 0, nkj = 0;
            const int nb = b == kKVBufs - 1 ? 0 : b + 1;
            if (un < I.nkv) kv_stage(un, nb, nki, nkj, fk);
            const uint32_t a16 = I.masked ? d_allow16(g, myseg, kt, I.win) : 0xFFu;
            if (!wwait(&bars->s_full, sph, 0x6305)) { ok = false; break; }
            sph ^= 1;
            tc_fence_after();
            const uint32_t t_s = trow + sb;
            if (!first) {  // the previous tile's P V, complete with this S
                uint32_t v[32];
                tmem_ld32(trow + (sb ^ kSBuf) + kColO, v);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; e += 2)
                    fadd2(o[e], o[e + 1], o[e], o[e + 1], __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
            } else {
                // the item's first tile: its row maximum in a pass of its own
                float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t v[32];
                    tmem_ld32(t_s + 32 * c, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (!((a16 >> (2 * c + (e >> 4))) & 1u)) v[e] = __float_as_uint(-INFINITY);
#pragma unroll
                    for (int e = 0; e < 32; e += 2)
                        mx4[(e >> 1) & 3] = fmax3(mx4[(e >> 1) & 3], __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
                }
                m = fmaxf(fmax3(mx4[0], mx4[1], mx4[2]), mx4[3]) * sl2;  // O and l are zero
            }
            // Probabilities, row sum and bf16 P in one pass.  After the first tile
            // each chunk's maximum is checked against the running maximum m; only
            // when it exceeds m by more than 64 (in log2 units), or m is still
            // -inf, are m, l, O and the chunks of P already written rescaled.  P
            // up to 2^64 stays far inside the range of bf16 and of the fp32 sums,
            // and the softmax is the same.
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
            if (!group_sync(0x6306)) { ok = false; break; }  // every row's P written
            if (r == 0) {
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < kTile / 16; ++k)
                    umma_ts(tmem + sb + kColO, tmem + sb + kColP + 8 * k, dMN0 + ((koff + 2 * kTileBytes) >> 4) + 64 * k,
                            id_pv, k > 0);
                if (un >= I.nkv) umma_commit(&bars->o_full);  // the item's last product
            }
            first = false;
            ++tcs;
            u = un;
            b = nb;
            ki = nki;
            kj = nkj;
        }
        if (!ok) break;
        if (!first) {  // the last tile's P V
            if (!wwait(&bars->o_full, oph, 0x6307)) break;
            oph ^= 1;
            tc_fence_after();
            uint32_t v[32];
            tmem_ld32(trow + ((tcs - 1u) & 1u) * kSBuf + kColO, v);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; e += 2)
                fadd2(o[e], o[e + 1], o[e], o[e + 1], __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
            tc_fence_before();  // ordered before the next item's products by its group barriers
        }
        // epilogue: O / l staged over q', coalesced stores, log-sum-exp
        const float inv = 1.f / l;
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] *= inv;
        store_row_swz(q0, r, o);
        __syncwarp();
        store_rows(prm.o, q0, qtok, qvalid, warp, lane);
        if (qvalid && prm.lse != nullptr) prm.lse[qtok] = (m + lg2_approx(l)) * 0.69314718055994530942f;
    }
    cp_async_wait<0>();  // a tile staged before a failed wait: its copies land before the CTA exits
    if (r == 0) {  // every MMA issued here has completed before the columns are freed
        umma_commit(&bars->done);
        mbar_wait(&bars->done, 0, ctl, 0x63ff);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace fwd

// ------------------------------------------------------------------ backward
namespace bwd {

struct WsLayout {
    size_t acc, nrm, rowv, fac, part, part2, cnt, red, total;
    long long chunks;  // first-level dU / dW sums
};

__host__ __device__ inline size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

__host__ __device__ inline WsLayout ws_layout(const Geo& g) {
    const size_t ht = static_cast<size_t>(g.heads) * static_cast<size_t>(g.tiles);
    WsLayout L;
    L.chunks = (g.wins + kWinChunk - 1) / kWinChunk;
    size_t o = 0;
    L.acc = o;   o += round256(ht * kTile * 64 * 4);  // fp32 [heads][tiles][128][64]
    L.nrm = o;   o += round256(ht * 8);               // max |dO row|^2, max |v row|^2 per (head, tile)
    L.rowv = o;  o += round256(ht * kTile * 8);       // per slot row: lse log2(e), D
    L.fac = o;   o += round256(static_cast<size_t>(g.heads) * g.N * 2 * 32);  // [h][pos]: sqrt(d) U, W (fp16)
    L.part = o;  o += round256(ht * 8 * 16 * 4);      // d theta partials [heads][tiles][8][16]
    L.part2 = o; o += round256(static_cast<size_t>(g.heads) * 64 * 16 * 4);
    L.cnt = o;   o += round256(static_cast<size_t>(g.heads) * 4);
    L.red = o;   o += round256(static_cast<size_t>(L.chunks) * g.heads * g.N * 32 * 4);  // [chunk][h][N][32]
    L.total = o;
    return L;
}

struct Params {
    Geo g;
    const uint8_t *q, *k, *v, *o, *dout;  // bf16 [B, H, W, heads, 32]
    uint8_t *dq, *dk, *dv;
    const float *lse, *theta;  // theta may be null (no rotation)
    const float *u, *w;        // [heads][M*M][16]
    float *du, *dw;            // [heads][M*M][16]
    uint8_t* ws;
    WsLayout L;
    unsigned int* status;
    unsigned long long limit_ns;
    long long items;
    float scale;
};

// d theta terms of one token side of a 32-channel row: pos * (dx_b x_a - dx_a x_b)
// per pair, added into part[axis * 8 + k].  The 2D cross product does not change
// when both vectors turn by the same angle, so rotated or un-rotated pairs give
// the same terms.
__device__ __forceinline__ void dtheta_terms(float (&part)[16], const float (&dx)[32], const float (&x)[32], int i,
                                             int j) {
#pragma unroll
    for (int ax = 0; ax < 2; ++ax) {
        const float pos = static_cast<float>(ax ? i : j);
#pragma unroll
        for (int k = 0; k < kPairs; ++k) {
            const int a = ax * 16 + 2 * k, b = a + 1;
            part[ax * kPairs + k] += pos * (dx[b] * x[a] - dx[a] * x[b]);
        }
    }
}

// The warp's 16 d theta partials, summed over the warp in a fixed order, to
// part[((h * tiles + T) * 8 + slot)][k].
__device__ __forceinline__ void write_partials(const float (&part)[16], float* out, const Geo& g, int h, long long T,
                                               int slot, int lane) {
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        float v = part[e];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == e) out[((static_cast<long long>(h) * g.tiles + T) * 8 + slot) * 16 + e] = v;
    }
}

// prep: per (tile, head), thread = slot row: the tile's largest squared norms of
// dO and v rows, and the zeroed accumulator rows; block 0 zeroes the d theta
// reduction's counters.
__global__ void __launch_bounds__(128) prep_kernel(const Params p) {
    __shared__ float2 nrm_w[4];
    const Geo& g = p.g;
    const long long T = blockIdx.x / g.heads;
    const int h = static_cast<int>(blockIdx.x - T * g.heads);
    const long long ht = static_cast<long long>(h) * g.tiles + T;
    const int r = threadIdx.x;
    if (blockIdx.x == 0)
        for (int i = r; i < g.heads; i += blockDim.x) reinterpret_cast<unsigned int*>(p.ws + p.L.cnt)[i] = 0u;
    // the head's factor rows in fp16 (sqrt(d) U and W; 32 bytes each), written by
    // the blocks of its first tiles, one position per thread
    const long long pos = T * kTile + r;
    if (pos < g.N) {
        uint8_t* f = p.ws + p.L.fac + (static_cast<size_t>(h) * g.N + static_cast<size_t>(pos)) * 64;
        const float4* u4 = reinterpret_cast<const float4*>(p.u + (static_cast<long long>(h) * g.N + pos) * 16);
        const float4* w4 = reinterpret_cast<const float4*>(p.w + (static_cast<long long>(h) * g.N + pos) * 16);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const float4 a0 = __ldg(u4 + 2 * c), a1 = __ldg(u4 + 2 * c + 1);
            const float4 b0 = __ldg(w4 + 2 * c), b1 = __ldg(w4 + 2 * c + 1);
            reinterpret_cast<uint4*>(f)[c] =
                make_uint4(pack_f16x2(a0.x * kSqrtD, a0.y * kSqrtD), pack_f16x2(a0.z * kSqrtD, a0.w * kSqrtD),
                           pack_f16x2(a1.x * kSqrtD, a1.y * kSqrtD), pack_f16x2(a1.z * kSqrtD, a1.w * kSqrtD));
            reinterpret_cast<uint4*>(f + 32)[c] = make_uint4(pack_f16x2(b0.x, b0.y), pack_f16x2(b0.z, b0.w),
                                                             pack_f16x2(b1.x, b1.y), pack_f16x2(b1.z, b1.w));
        }
    }
    int pi, pj;
    long long tok;
    float ndo = 0.f, nv = 0.f, D = 0.f, lse2 = INFINITY;
    if (slot_token(g, T, r, h, &pi, &pj, &tok)) {
        float a[32], c[32];
        load_row32(p.dout, tok, a);
        load_row32(p.o, tok, c);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            ndo = fmaf(a[e], a[e], ndo);
            D = fmaf(a[e], c[e], D);
        }
        load_row32(p.v, tok, a);
#pragma unroll
        for (int e = 0; e < 32; ++e) nv = fmaf(a[e], a[e], nv);
        lse2 = __ldg(p.lse + tok) * 1.4426950408889634f;
    }
    reinterpret_cast<float2*>(p.ws + p.L.rowv)[ht * kTile + r] = make_float2(lse2, D);
    // the key side of d theta: the main kernel writes one slot per run of items of a
    // head in a CTA, the other slots 4..7 of the head's tiles must read zero
    if (r < 64) reinterpret_cast<float*>(p.ws + p.L.part)[(ht * 8 + 4) * 16 + r] = 0.f;
    uint4* acc = reinterpret_cast<uint4*>(p.ws + p.L.acc + (ht * kTile + r) * 64 * 4);
#pragma unroll
    for (int c = 0; c < 16; ++c) acc[c] = make_uint4(0, 0, 0, 0);
    ndo = warp_max_nonneg(ndo);
    nv = warp_max_nonneg(nv);
    if ((r & 31) == 0) nrm_w[r >> 5] = make_float2(ndo, nv);
    __syncthreads();
    if (r == 0)
        reinterpret_cast<float2*>(p.ws + p.L.nrm)[ht] =
            make_float2(fmaxf(fmaxf(nrm_w[0].x, nrm_w[1].x), fmaxf(nrm_w[2].x, nrm_w[3].x)),
                        fmaxf(fmaxf(nrm_w[0].y, nrm_w[1].y), fmaxf(nrm_w[2].y, nrm_w[3].y)));
}

// cp.async copy of a factor row (32 bytes, fp16) into row r of a factor half
// tile, channels 16..31 zero-filled.
__device__ __forceinline__ void copy_factor(uint8_t* tile, int r, const uint8_t* src) {
    uint8_t* row = tile + r * kRowBytes;
    const int sw = (r >> 1) & 3;
#pragma unroll
    for (int c = 0; c < 4; ++c) cp_async16(smem_u32(row + ((c ^ sw) << 4)), src + 16 * (c & 1), c < 2 ? 16u : 0u);
}

// Main kernel: two warpgroups of four warps; warp w serves TMEM lanes (key rows)
// 32 (w & 3) .. + 31, and the warpgroups split each step's work: the column
// halves of S^T and dP^T, the staging of rows (q and the U factors, k and its
// rotation: group 0; dO, D and lse2, v and the W factors: group 1), the dQ' and
// dU parts of the accumulator rows, and the item's end (dk and the key side of
// d theta: group 0; dv and the dW share: group 1).
constexpr int kThreads = 256;
constexpr int kKOff = 0;                           // K~ half tiles: k' and W
constexpr int kVOff = kKOff + 2 * kTileBytes;      // V tile
constexpr int kBufOff = kVOff + kTileBytes;        // two query buffers: Q~ half tiles (q', sqrt(d) U), dO tile
constexpr int kBufBytes = 3 * kTileBytes;
constexpr int kDSOff = kBufOff + 2 * kBufBytes;    // dS', MN-major 128-byte swizzle (1024-aligned)
constexpr int kVecOff = kDSOff + 4 * kTileBytes;   // per buffer: lse2[128], D[128]
constexpr int kTabOff = kVecOff + 2 * 2 * kTile * 4;
constexpr int kBarOff = kTabOff + kTabBytes;
constexpr int kSmemBytes = kBarOff + 256 + 1024;
static_assert(kDSOff % 1024 == 0, "128-byte swizzled operand must be 1024-byte aligned");
constexpr uint32_t kTmemCols = 512;
// S^T [0,128), dP^T [128,256); P'^T (bf16) [384,448) and dS'^T (fp16) [448,512),
// apart from S^T and dP^T because the two warpgroups read and write different
// column halves at once; dQ~ over S^T's consumed [64,128); dV [256,288),
// dK~ [320,384).
constexpr uint32_t kColS = 0, kColDP = 128, kColP = 384, kColDS = 448, kColDQ = 64, kColDV = 256, kColDK = 320;

struct Bars {
    uint64_t s_full, mma_done, grp, done;
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Bars) <= 256, "barrier block overflows its slot");

__global__ void __launch_bounds__(kThreads, 1) main_kernel(const __grid_constant__ Params prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars* bars = reinterpret_cast<Bars*>(smem + kBarOff);
    const Geo& g = prm.g;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->mma_done, 1);
        mbar_init(&bars->grp, 8);
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
    const int wg = warp >> 2, quad = warp & 3;
    const int r = tid & (kTile - 1);  // this thread's row (TMEM lane)
    const uint32_t tmem = bars->tmem_base;
    const uint32_t trow = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const Ctl ctl{prm.status, &bars->abort_flag, prm.limit_ns};
    const uint32_t id_s = make_idesc(kTile, kTile, false, false, true);     // fp16 K~, Q~
    const uint32_t id_dp = make_idesc(kTile, kTile, false, false, false);   // bf16 V, dO
    const uint32_t id_dv = make_idesc(kTile, kHeadDim, false, true, false); // P'^T (TMEM) x dO
    // dK~ and dQ~ take both half tiles in one N = 64 product: the MN-major B
    // operand's 64-byte swizzle atoms (32 channels) follow each other at the
    // descriptor's leading byte offset, one half tile apart
    const uint32_t id_dk = make_idesc(kTile, 2 * kHeadDim, false, true, true);  // dS'^T (TMEM) x Q~
    const uint32_t id_dq = make_idesc(kTile, 2 * kHeadDim, true, true, true);   // dS' (smem) x K~
    const uint32_t sbase = smem_u32(smem);
    const uint64_t dK0 = make_sdesc(sbase, 16, 512, kSw64);
    const uint64_t dMN0 = make_sdesc(sbase, 8192, 512, kSw64);
    const uint64_t dDS = make_sdesc(sbase + kDSOff, 16384, 1024, kSw128);
    auto u16 = [](int bytes) { return static_cast<uint64_t>(bytes >> 4); };
    const float sl2 = g.scale_log2;
    float2* tab = reinterpret_cast<float2*>(smem + kTabOff);
    const float2* rtab = prm.theta ? tab : nullptr;
    float* vec = reinterpret_cast<float*>(smem + kVecOff);  // buffer b: lse2 at [256 b], D at [256 b + 128]
    uint8_t* ds = smem + kDSOff;
    uint8_t* kh[2] = {smem + kKOff, smem + kKOff + kTileBytes};
    uint8_t* vt = smem + kVOff;
    float* acc_all = reinterpret_cast<float*>(prm.ws + prm.L.acc);
    const uint8_t* fac = prm.ws + prm.L.fac;                                // [h][pos]: sqrt(d) U, W (fp16)
    const float2* rowv = reinterpret_cast<const float2*>(prm.ws + prm.L.rowv);  // per slot row: lse2, D
    uint32_t gph = 0, sph = 0, mph = 0;
    int tab_head = -1;
    bool ok = true;
    // key side of d theta, summed over this CTA's run of items of one head (items
    // go head by head) and written once per run, to slot 4 + quad of the run's
    // first key tile
    float part[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) part[e] = 0.f;
    int run_head = -1;
    long long run_tile = 0;
    auto flush_partials = [&]() {
        if (rtab && wg == 0 && run_head >= 0)
            write_partials(part, reinterpret_cast<float*>(prm.ws + prm.L.part), g, run_head, run_tile, 4 + quad, lane);
#pragma unroll
        for (int e = 0; e < 16; ++e) part[e] = 0.f;
    };
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

    for (long long it = blockIdx.x; it < prm.items && ok; it += gridDim.x) {
        const BwdItem I = d_bwd_item(g, it);
        if (I.h != run_head) {  // a new run of items of one head
            flush_partials();
            run_head = I.h;
            run_tile = I.u;
        }
        if (rtab && I.h != tab_head) {
            if (!group_sync(0x6401)) break;
            build_table(tab, prm.theta + I.h * 2 * kPairs, g.M, tid, kThreads);
            if (!group_sync(0x6402)) break;
            tab_head = I.h;
        }
        // the gradient scaling 2^e of the item: the largest |dO| and |v| rows of its
        // window (or tile, for windows inside one tile), from the prep kernel
        float mdo = 0.f, mv = 0.f;
        {
            const float2* nrm = reinterpret_cast<const float2*>(prm.ws + prm.L.nrm) + static_cast<size_t>(I.h) * g.tiles;
            for (int n = 0; n < I.nq; ++n) {
                const float2 t = __ldcg(&nrm[I.q0 + n]);
                mdo = fmaxf(mdo, t.x);
                mv = fmaxf(mv, t.y);
            }
        }
        const int gexp = grad_scale_exp(mdo, mv);
        // this thread's key row: K rotated (group 0), V and the key factors (group 1)
        int ki, kj;
        long long ktok;
        const bool kvalid = slot_token(g, I.u, r, I.h, &ki, &kj, &ktok);
        const uint32_t keyseg = I.masked ? seg_at(d_tile_segs(g, I.u, I.win), r >> g.lBT) : 0u;
        if (!group_sync(0x6403)) break;  // the previous item's K~, V rows are read by every thread
        if (wg == 0) {
            copy_rows(kh[0], prm.k, ktok, kvalid, quad, lane);
            cp_async_commit();
            cp_async_wait<0>();
            __syncwarp();
            prep_row(kh[0], r, ki, kj, rtab);
        } else {
            copy_rows(vt, prm.v, ktok, kvalid, quad, lane);
            copy_factor(kh[1], r, fac + (static_cast<size_t>(I.h) * g.N + ki * g.M + kj) * 64 + 32);
            cp_async_commit();
        }
        bool first = true;
        // Query steps, double-buffered: the copies, factors, D and lse2 of the next
        // active query tile are issued while the current step's products run.
        auto stage = [&](int n, int b, int& qi, int& qj, bool& qvalid) {
            long long qtok;
            qvalid = slot_token(g, I.q0 + n, r, I.h, &qi, &qj, &qtok);
            uint8_t* qb = smem + kBufOff + b * kBufBytes;
            if (wg == 0) {
                copy_rows(qb, prm.q, qtok, qvalid, quad, lane);
                copy_factor(qb + kTileBytes, r, fac + (static_cast<size_t>(I.h) * g.N + qi * g.M + qj) * 64);
                cp_async_commit();
            } else {
                copy_rows(qb + 2 * kTileBytes, prm.dout, qtok, qvalid, quad, lane);
                cp_async_commit();
                // lse2 and D of the row, from the prep kernel (lse2 = +inf for a padded row)
                const float2 ld = __ldcg(rowv + ((static_cast<long long>(I.h) * g.tiles + I.q0 + n) * kTile + r));
                vec[256 * b + kTile + r] = ld.y;
                vec[256 * b + r] = ld.x - static_cast<float>(gexp);
            }
        };
        auto next_active = [&](int n) {
            while (n < I.nq && !bwd_active(g, I, n)) ++n;
            return n;
        };
        int n = next_active(0), b = 0, qi = 0, qj = 0;
        bool qvalid = false;
        if (n < I.nq) stage(n, 0, qi, qj, qvalid);
        while (n < I.nq && ok) {
            const long long T = I.q0 + n;
            const int nn = next_active(n + 1);
            const int qoff = kBufOff + b * kBufBytes, dooff = qoff + 2 * kTileBytes;
            const float* lse2v = vec + 256 * b;
            const float* dvec = lse2v + kTile;
            cp_async_wait<0>();
            __syncwarp();
            if (wg == 0) prep_row(smem + qoff, r, qi, qj, rtab);
            fence_proxy_async_smem();
            if (!group_sync(0x6404)) { ok = false; break; }  // rows staged and rotated
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < kHeadDim / 16; ++k) {
                    umma_ss(tmem + kColS, dK0 + u16(kKOff) + 2 * k, dK0 + u16(qoff) + 2 * k, id_s, k > 0);
                    umma_ss(tmem + kColDP, dK0 + u16(kVOff) + 2 * k, dK0 + u16(dooff) + 2 * k, id_dp, k > 0);
                }
                umma_ss(tmem + kColS, dK0 + u16(kKOff + kTileBytes), dK0 + u16(qoff + kTileBytes), id_s, 1u);
                umma_commit(&bars->s_full);
            }
            // the next step's rows go to the other buffer, whose products (the previous
            // step's) have completed
            int nqi = 0, nqj = 0;
            bool nqvalid = false;
            if (nn < I.nq) stage(nn, b ^ 1, nqi, nqj, nqvalid);
            const uint32_t a16 = I.masked ? d_allow16(g, keyseg, T, I.win) : 0xFFu;
            if (!wwait(&bars->s_full, sph, 0x6405)) { ok = false; break; }
            sph ^= 1;
            tc_fence_after();
            // this key row of P'^T and dS'^T: the group's 64 query columns, 32 at a time
#pragma unroll 1
            for (int c = 2 * wg; c < 2 * wg + 2; ++c) {
                uint8_t* base = ds + (c >> 1) * 16384 + (r >> 3) * 1024 + (r & 7) * 128;
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
                tmem_st16(trow + kColP + 16 * c, wp);
                tmem_st16(trow + kColDS + 16 * c, wd);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {  // dS' (queries along M, keys along K), MN-major
                    const int cc = 4 * (c & 1) + q4;
                    *reinterpret_cast<uint4*>(base + ((cc ^ (r & 7)) << 4)) =
                        make_uint4(wd[4 * q4], wd[4 * q4 + 1], wd[4 * q4 + 2], wd[4 * q4 + 3]);
                }
            }
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            if (!group_sync(0x6406)) { ok = false; break; }  // every row's P'^T, dS'^T and dS' written
            if (tid == 0) {
                tc_fence_after();
                const uint32_t acc = first ? 0u : 1u;
#pragma unroll
                for (int k = 0; k < kTile / 16; ++k)
                    umma_ts(tmem + kColDV, tmem + kColP + 8 * k, dMN0 + u16(dooff) + 64 * k, id_dv,
                            k > 0 ? 1u : acc);
#pragma unroll
                for (int k = 0; k < kTile / 16; ++k)
                    umma_ts(tmem + kColDK, tmem + kColDS + 8 * k, dMN0 + u16(qoff) + 64 * k, id_dk,
                            k > 0 ? 1u : acc);
#pragma unroll
                for (int k = 0; k < kTile / 16; ++k)
                    umma_ss(tmem + kColDQ, dDS + 128 * k, dMN0 + u16(kKOff) + 64 * k, id_dq, k > 0);
                umma_commit(&bars->mma_done);
            }
            first = false;
            if (!wwait(&bars->mma_done, mph, 0x6407)) { ok = false; break; }
            mph ^= 1;
            tc_fence_after();
            // this query row's dQ' (group 0: softmax scale and 2^-e) and dU share
            // (group 1: 2^-e), added into its accumulator row
            {
                const float down = exp2i(-gexp);
                float* accrow = acc_all + ((static_cast<long long>(I.h) * g.tiles + T) * kTile + r) * 64;
                if (wg == 0) {
                    const float sc = prm.scale * down;
                    uint32_t v[32];
                    tmem_ld32(trow + kColDQ, v);
                    tmem_wait_ld();
                    if (qvalid) {
#pragma unroll
                        for (int e = 0; e < 32; e += 4)
                            red_add_v4(accrow + e, __uint_as_float(v[e]) * sc, __uint_as_float(v[e + 1]) * sc,
                                       __uint_as_float(v[e + 2]) * sc, __uint_as_float(v[e + 3]) * sc);
                    }
                } else {
                    uint32_t v16[16];
                    tmem_ld16(trow + kColDQ + kHeadDim, v16);
                    tmem_wait_ld();
                    // a padded token's row adds nothing: its dS' row is zero (lse2 = +inf)
#pragma unroll
                    for (int e = 0; e < 16; e += 4)
                        red_add_v4(accrow + 32 + e, __uint_as_float(v16[e]) * down,
                                   __uint_as_float(v16[e + 1]) * down, __uint_as_float(v16[e + 2]) * down,
                                   __uint_as_float(v16[e + 3]) * down);
                }
            }
            tc_fence_before();  // ordered before the next step's products by its group barrier
            n = nn;
            b ^= 1;
            qi = nqi;
            qj = nqj;
            qvalid = nqvalid;
        }
        if (!ok) break;
        // item end: group 0 dk (dK' un-rotated) and the key side of d theta, group 1
        // dv and the row's dW share
        const float down = exp2i(-gexp);
        if (first) {  // no query tile attends these keys (cannot happen: a key attends itself)
            float z[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) z[e] = 0.f;
            store_row_swz(wg == 0 ? kh[0] : vt, r, z);
        } else if (wg == 0) {
            uint32_t t[32];
            float dx[32], x[32];
            tmem_ld32(trow + kColDK, t);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) dx[e] = __uint_as_float(t[e]) * (prm.scale * down);
            if (rtab) {
                load_row_swz(kh[0], r, x, true);  // rotated k' (fp16)
                if (kvalid) dtheta_terms(part, dx, x, ki, kj);
                rope_row(dx, ki, kj, rtab, true);
            }
            store_row_swz(kh[0], r, dx);  // dk (bf16), staged over k'
        } else {
            uint32_t t16[16];
            tmem_ld16(trow + kColDK + kHeadDim, t16);
            tmem_wait_ld();
            float4* dst = reinterpret_cast<float4*>(
                acc_all + ((static_cast<long long>(I.h) * g.tiles + I.u) * kTile + r) * 64 + 48);
            const float f = prm.scale * down;
#pragma unroll
            for (int c = 0; c < 4; ++c)
                dst[c] = make_float4(__uint_as_float(t16[4 * c]) * f, __uint_as_float(t16[4 * c + 1]) * f,
                                     __uint_as_float(t16[4 * c + 2]) * f, __uint_as_float(t16[4 * c + 3]) * f);
            uint32_t t[32];
            float x[32];
            tmem_ld32(trow + kColDV, t);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] = __uint_as_float(t[e]) * down;
            store_row_swz(vt, r, x);  // dv, staged over v
        }
        tc_fence_before();
        __syncwarp();
        if (wg == 0) {
            store_rows(prm.dk, kh[0], ktok, kvalid, quad, lane);
        } else {
            store_rows(prm.dv, vt, ktok, kvalid, quad, lane);
        }
    }
    flush_partials();
    cp_async_wait<0>();  // a step staged before a failed wait: its copies land before the CTA exits
    if (tid == 0) {
        umma_commit(&bars->done);
        mbar_wait(&bars->done, 0, ctl, 0x64ff);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// post: per (tile, head), thread = slot row: dq (the accumulated dQ' un-rotated)
// and the query side of d theta.
__global__ void __launch_bounds__(128) post_kernel(const Params p) {
    __shared__ float2 tab[2 * kPairs * 64];
    const Geo& g = p.g;
    const long long T = blockIdx.x / g.heads;
    const int h = static_cast<int>(blockIdx.x - T * g.heads);
    const long long ht = static_cast<long long>(h) * g.tiles + T;
    if (p.theta) build_table(tab, p.theta + h * 2 * kPairs, g.M, threadIdx.x, blockDim.x);
    __syncthreads();
    const int r = threadIdx.x, lane = r & 31, warp = r >> 5;
    int pi, pj;
    long long tok;
    float part[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) part[e] = 0.f;
    if (slot_token(g, T, r, h, &pi, &pj, &tok)) {
        const float* acc = reinterpret_cast<const float*>(p.ws + p.L.acc) + (ht * kTile + r) * 64;
        float dx[32];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
            const float4 a4 = *reinterpret_cast<const float4*>(acc + e);
            dx[e] = a4.x;
            dx[e + 1] = a4.y;
            dx[e + 2] = a4.z;
            dx[e + 3] = a4.w;
        }
        if (p.theta) {
            rope_row(dx, pi, pj, tab, true);
            float q[32];
            load_row32(p.q, tok, q);
            dtheta_terms(part, dx, q, pi, pj);  // the cross products are the same before rotation
        }
        uint4* dst = reinterpret_cast<uint4*>(p.dq + tok * kRowBytes);
#pragma unroll
        for (int c = 0; c < 4; ++c) dst[c] = pack_chunk(dx, c);
    }
    if (p.theta) write_partials(part, reinterpret_cast<float*>(p.ws + p.L.part), g, h, T, warp, lane);
}

// dU / dW sum, level 1: block (chunk, head) sums the shares of windows
// [chunk * 16, chunk * 16 + 16) slot by slot, in window order:
// red[chunk][h][slot sigma][32] (sigma = the slot of a token inside its window).
__global__ void __launch_bounds__(256) bias_sum1_kernel(const Params p) {
    const Geo& g = p.g;
    const long long chunk = blockIdx.x;
    const int h = blockIdx.y;
    const long long w0 = chunk * kWinChunk;
    const long long w1 = w0 + kWinChunk < g.wins ? w0 + kWinChunk : g.wins;
    const float* acc = reinterpret_cast<const float*>(p.ws + p.L.acc) + static_cast<long long>(h) * g.tiles * kTile * 64;
    float4* out = reinterpret_cast<float4*>(p.ws + p.L.red) + (chunk * g.heads + h) * static_cast<long long>(g.N) * 8;
    for (int idx = threadIdx.x; idx < g.N * 8; idx += blockDim.x) {
        const int sigma = idx >> 3, qd = idx & 7;
        float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
        for (long long w = w0; w < w1; ++w) {
            const long long slot = w * g.N + sigma;  // slot of the head's token enumeration (tile * 128 + row)
            const float4 a = __ldcg(reinterpret_cast<const float4*>(acc + slot * 64 + 32 + 4 * qd));
            s.x += a.x;
            s.y += a.y;
            s.z += a.z;
            s.w += a.w;
        }
        out[idx] = s;
    }
}

// Level 2: warp (head, slot sigma, quarter) sums the chunks, lane l those with
// c = l mod 32 in increasing order, then the 32 lane sums in a fixed butterfly,
// and writes dU (quarters 0-3) or dW (4-7) at the slot's window position
// t = i M + j.
__global__ void __launch_bounds__(256) bias_sum2_kernel(const Params p) {
    const Geo& g = p.g;
    const int lane = threadIdx.x & 31;
    const long long gw = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (gw >= static_cast<long long>(g.heads) * g.N * 8) return;  // whole warps leave together
    const int h = static_cast<int>(gw / (g.N * 8));
    const int idx = static_cast<int>(gw - static_cast<long long>(h) * g.N * 8);
    const int sigma = idx >> 3, qd = idx & 7;
    const float4* red = reinterpret_cast<const float4*>(p.ws + p.L.red);
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    for (long long c = lane; c < p.L.chunks; c += 32) {
        const float4 a = __ldcg(red + (c * g.heads + h) * static_cast<long long>(g.N) * 8 + idx);
        s.x += a.x;
        s.y += a.y;
        s.z += a.z;
        s.w += a.w;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        s.x += __shfl_xor_sync(0xffffffffu, s.x, o);
        s.y += __shfl_xor_sync(0xffffffffu, s.y, o);
        s.z += __shfl_xor_sync(0xffffffffu, s.z, o);
        s.w += __shfl_xor_sync(0xffffffffu, s.w, o);
    }
    if (lane) return;
    int i, j;
    tile_row_pos(g, sigma >> 7, sigma & (kTile - 1), &i, &j);
    float* dst = qd < 4 ? p.du : p.dw;
    reinterpret_cast<float4*>(dst + (static_cast<long long>(h) * g.N + i * g.M + j) * 16)[qd & 3] = s;
}

}  // namespace bwd

}  // namespace lrbk

size_t lrbias_bwd_workspace_bytes(const Geo& g) { return lrbk::bwd::ws_layout(g).total; }

cudaError_t launch_lrbias_fwd(const Geo& g, const LrbPtrs& p, unsigned int* status, unsigned long long limit_ns,
                              int num_sms, cudaStream_t stream, cudaEvent_t const* events) {
    using namespace lrbk;
    static SmemOptIn optin;
    if (cudaError_t e = optin.ensure(reinterpret_cast<const void*>(fwd::fwd_kernel), fwd::kSmemBytes)) return e;
    fwd::Params prm;
    prm.g = g;
    prm.q = static_cast<const uint8_t*>(p.q);
    prm.k = static_cast<const uint8_t*>(p.k);
    prm.v = static_cast<const uint8_t*>(p.v);
    prm.o = static_cast<uint8_t*>(p.o_out);
    prm.theta = p.theta;
    prm.u = p.u;
    prm.w = p.w;
    prm.lse = p.lse_out;
    prm.status = status;
    prm.limit_ns = limit_ns;
    prm.items = fwd_item_count(g);
    if (prm.items == 0) return cudaSuccess;
    const long long grid = prm.items < 2ll * num_sms ? prm.items : 2ll * num_sms;  // two CTAs per SM (TMEM)
    cudaError_t e = events ? cudaEventRecord(events[0], stream) : cudaSuccess;
    if (e != cudaSuccess) return e;
    fwd::fwd_kernel<<<static_cast<unsigned>(grid), fwd::kThreads, fwd::kSmemBytes, stream>>>(prm);
    e = cudaGetLastError();
    if (e == cudaSuccess && events) e = cudaEventRecord(events[1], stream);
    return e;
}

cudaError_t launch_lrbias_bwd(const Geo& g, const LrbPtrs& p, unsigned int* status, unsigned long long limit_ns,
                              int num_sms, cudaStream_t stream, cudaEvent_t const* events) {
    using namespace lrbk;
    static SmemOptIn optin;
    if (cudaError_t e = optin.ensure(reinterpret_cast<const void*>(bwd::main_kernel), bwd::kSmemBytes)) return e;
    const bwd::WsLayout L = bwd::ws_layout(g);
    bwd::Params prm;
    prm.g = g;
    prm.q = static_cast<const uint8_t*>(p.q);
    prm.k = static_cast<const uint8_t*>(p.k);
    prm.v = static_cast<const uint8_t*>(p.v);
    prm.o = static_cast<const uint8_t*>(p.o);
    prm.dout = static_cast<const uint8_t*>(p.dout);
    prm.dq = static_cast<uint8_t*>(p.dq);
    prm.dk = static_cast<uint8_t*>(p.dk);
    prm.dv = static_cast<uint8_t*>(p.dv);
    prm.lse = p.lse;
    prm.theta = p.theta;
    prm.u = p.u;
    prm.w = p.w;
    prm.du = p.du;
    prm.dw = p.dw;
    prm.ws = p.ws;
    prm.L = L;
    prm.status = status;
    prm.limit_ns = limit_ns;
    prm.items = bwd_item_count(g);
    prm.scale = 0.17677669529663688f;  // 1/sqrt(32)
    const long long ht = static_cast<long long>(g.heads) * g.tiles;
    cudaError_t e = cudaSuccess;
    auto mark = [&](int i) {
        if (events && e == cudaSuccess) e = cudaEventRecord(events[i], stream);
    };
    mark(0);
    bwd::prep_kernel<<<static_cast<unsigned>(ht), 128, 0, stream>>>(prm);
    if (e == cudaSuccess) e = cudaGetLastError();
    mark(1);
    const long long grid = prm.items < num_sms ? prm.items : num_sms;
    bwd::main_kernel<<<static_cast<unsigned>(grid), bwd::kThreads, bwd::kSmemBytes, stream>>>(prm);
    if (e == cudaSuccess) e = cudaGetLastError();
    mark(2);
    bwd::post_kernel<<<static_cast<unsigned>(ht), 128, 0, stream>>>(prm);
    if (e == cudaSuccess) e = cudaGetLastError();
    mark(3);
    // d theta: [heads] sums of [tiles * 8][16] partials
    if (e == cudaSuccess && p.theta)
        e = bwdk::launch_dtheta(reinterpret_cast<const float*>(p.ws + L.part), g.tiles * 8, g.heads,
                                reinterpret_cast<float*>(p.ws + L.part2), reinterpret_cast<unsigned int*>(p.ws + L.cnt),
                                p.dtheta, stream);
    // dU, dW: two fixed-order levels over the windows of the batch
    if (e == cudaSuccess) {
        bwd::bias_sum1_kernel<<<dim3(static_cast<unsigned>(L.chunks), static_cast<unsigned>(g.heads)), 256, 0, stream>>>(
            prm);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) {  // one warp per (head, slot, quarter), eight warps per block
        const long long warps = static_cast<long long>(g.heads) * g.N * 8;
        bwd::bias_sum2_kernel<<<static_cast<unsigned>((warps + 7) / 8), 256, 0, stream>>>(prm);
        e = cudaGetLastError();
    }
    mark(4);
    return e;
}

}  // namespace fswin
