// Kernels for heads of d = 64 channels, every window size.
//
// A 64-channel token row (128 bytes) is held as two 32-channel half rows in two
// half tiles, each laid out like the d = 32 tiles (64-byte rows, 64-byte
// swizzle), so the same tile helpers and MMA descriptors apply.  The halves are
// also the two RoPE axes: channel pairs of the first half turn by the column
// position j with theta[h][0][k], those of the second half by the row position i
// with theta[h][1][k], k = 0 .. 15.
//
// The kernels are plain one-tile pipelines (one CTA of row warps walks its work
// items, four in the forward, eight in the backward's main kernel; thread 0
// issues the MMAs): copies, rotation, products and softmax follow each other
// without overlap across items.
//   forward:  item = (query tile, head); the key tiles of its group in turn,
//             online softmax with O in registers;
//   backward: prep (per tile and head: the largest |dO row| and |v row| for the
//             gradient scaling, zeroed dQ' accumulator), main (eight warps in two
//             warpgroups; item = (key tile, head); the query tiles of its group
//             in turn, double-buffered: S^T, dP^T, P'^T and dS'^T, dV and dK'
//             accumulated in TMEM, dQ' added with 16-byte fp32 vector
//             reductions; dk, dv and the key side of d theta at the item's end),
//             post (dq and the query side of d theta), and the fixed-order
//             d theta sum of the d = 32 backward.
#include <cuda.h>
#include <cuda_runtime.h>

#include "dgeo.cuh"
#include "geometry.cuh"
#include "kernels.cuh"
#include "ptx.cuh"
#include "rows.cuh"
#include "schedule.cuh"

namespace fswin {

namespace widek {

constexpr int kHalves = 2;                      // 32-channel halves of a 64-channel row
constexpr int kWideRowBytes = kHalves * kRowBytes;  // 128 bytes in memory
constexpr int kPairs = 16;                      // RoPE pairs per axis
constexpr int kTabBytes = 2 * kPairs * 64 * 8;  // [axis][pair][position < 64] float2

// cos/sin of pos * theta[h][axis][k], pos < M, as [axis * 16 + k][64 positions].
__device__ __forceinline__ void build_table(float2* tab, const float* theta_h, int M, int t, int nt) {
    for (int e = t; e < 2 * kPairs * M; e += nt) {
        const int ak = e / M, pos = e - ak * M;
        float sn, cs;
        sincosf(static_cast<float>(pos) * theta_h[ak], &sn, &cs);
        tab[ak * 64 + pos] = make_float2(cs, sn);
    }
}

// Rotates (inv: un-rotates) the 16 pairs of one 32-channel half by one position.
__device__ __forceinline__ void rope_half(float (&x)[32], int pos, const float2* tab_axis, bool inv) {
#pragma unroll
    for (int k = 0; k < kPairs; ++k) {
        const float2 cs = tab_axis[k * 64 + pos];
        const float sn = inv ? -cs.y : cs.y;
        const float a = x[2 * k], b = x[2 * k + 1];
        x[2 * k] = a * cs.x - b * sn;
        x[2 * k + 1] = a * sn + b * cs.x;
    }
}

// cp.async copies of the warp's 32 rows of a [.., 64] bf16 tensor into the two
// half tiles: lane l moves 16-byte chunk l % 8 of rows l / 8 + 4 i, so each
// instruction moves four whole 128-byte rows.  tok / valid: this lane's own row.
__device__ __forceinline__ void copy_rows(uint8_t* half0, uint8_t* half1, const uint8_t* src, long long tok,
                                          bool valid, int warp, int lane) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int rl = (lane >> 3) + 4 * i, c = lane & 7;
        const long long tk = __shfl_sync(0xFFFFFFFFu, tok, rl);
        const bool vd = __shfl_sync(0xFFFFFFFFu, valid ? 1 : 0, rl) != 0;
        const int row = warp * 32 + rl, cc = c & 3;
        uint8_t* dst = (c < 4 ? half0 : half1) + row * kRowBytes + ((cc ^ ((row >> 1) & 3)) << 4);
        cp_async16(smem_u32(dst), vd ? src + tk * kWideRowBytes + 16 * c : src, vd ? 16u : 0u);
    }
}

// Coalesced 16-byte stores of the warp's 32 staged rows (valid ones only).
__device__ __forceinline__ void store_rows(uint8_t* dst, const uint8_t* half0, const uint8_t* half1, long long tok,
                                           bool valid, int warp, int lane) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int rl = (lane >> 3) + 4 * i, c = lane & 7;
        const long long tk = __shfl_sync(0xFFFFFFFFu, tok, rl);
        const bool vd = __shfl_sync(0xFFFFFFFFu, valid ? 1 : 0, rl) != 0;
        const int row = warp * 32 + rl, cc = c & 3;
        const uint8_t* s = (c < 4 ? half0 : half1) + row * kRowBytes + ((cc ^ ((row >> 1) & 3)) << 4);
        if (vd) *reinterpret_cast<uint4*>(dst + tk * kWideRowBytes + 16 * c) = *reinterpret_cast<const uint4*>(s);
    }
}

// ------------------------------------------------------------------ forward
namespace fwd {

constexpr int kThreads = 128;
constexpr int kQOff = 0;                             // Q' half tiles (then the staged O)
constexpr int kKVOff = kQOff + kHalves * kTileBytes;  // two key buffers: K' half tiles, V half tiles
constexpr int kKVBytes = 2 * kHalves * kTileBytes;
constexpr int kTabOff = kKVOff + 2 * kKVBytes;
constexpr int kBarOff = kTabOff + kTabBytes;
constexpr int kSmemBytes = kBarOff + 256 + 1024;  // + alignment of the base
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS = 0, kColP = 0, kColO = 128;  // O tile halves at 128, 160

struct Bars {
    uint64_t s_full, o_full, grp, done;
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Bars) <= 256, "barrier block overflows its slot");

struct Params {
    Geo g;
    const uint8_t *q, *k, *v;  // bf16 [B, H, W, heads, 64]
    uint8_t* o;
    const float* theta;  // [heads][2][16]
    float* lse;          // [B, H, W, heads] or null
    unsigned int* status;
    unsigned long long limit_ns;
    long long items;
};

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
    const uint32_t id_s = make_idesc(kTile, kTile, false, false, true);    // fp16 Q', K'
    // P (TMEM) x V over both half tiles in one N = 64 product (the MN-major
    // operand's two swizzle atoms one half tile apart)
    const uint32_t id_pv = make_idesc_bf16(kTile, 2 * kHeadDim, false, true);
    const uint32_t sbase = smem_u32(smem);
    const uint64_t dK0 = make_sdesc(sbase, 16, 512, kSw64);     // K-major, 64-byte rows
    const uint64_t dMN0 = make_sdesc(sbase, 8192, 512, kSw64);  // MN-major, 64-byte rows
    const float sl2 = g.scale_log2;
    float2* tab = reinterpret_cast<float2*>(smem + kTabOff);
    uint8_t* q0 = smem + kQOff;
    uint8_t* q1 = q0 + kTileBytes;
    uint32_t gph = 0, sph = 0, oph = 0;
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
    // rotates this thread's row of a half-tile pair in place (bf16 in, fp16 out)
    auto rotate_row = [&](uint8_t* h0, uint8_t* h1, int pi, int pj) {
        float x[32];
        load_row_swz(h0, r, x, false);
        rope_half(x, pj, tab, false);
        store_row_swz(h0, r, x, true);
        load_row_swz(h1, r, x, false);
        rope_half(x, pi, tab + kPairs * 64, false);
        store_row_swz(h1, r, x, true);
    };

    for (long long it = blockIdx.x; it < prm.items && ok; it += gridDim.x) {
        const FwdItem I = d_fwd_item(g, it);
        if (I.h != tab_head) {
            if (!group_sync(0x6101)) break;  // no row still rotates with the old table
            build_table(tab, prm.theta + I.h * 2 * kPairs, g.M, r, kThreads);
            if (!group_sync(0x6102)) break;
            tab_head = I.h;
        }
        // this thread's query row, its token and its segment byte
        int pi, pj;
        long long qtok;
        const bool qvalid = slot_token(g, I.X, r, I.h, &pi, &pj, &qtok);
        const uint32_t myseg = I.masked ? seg_at(d_tile_segs(g, I.X, I.win), r >> g.lBT) : 0u;
        if (!group_sync(0x6103)) break;  // the previous item's staged O rows are stored
        // Key tiles, double-buffered: the next active tile's K, V rows are copied
        // while the current tile's softmax runs.
        auto kv_stage = [&](int u, int b, int& ki, int& kj) {
            long long ktok;
            const bool kvalid = slot_token(g, I.kv0 + u, r, I.h, &ki, &kj, &ktok);
            uint8_t* kb = smem + kKVOff + b * kKVBytes;
            copy_rows(kb, kb + kTileBytes, prm.k, ktok, kvalid, warp, lane);
            copy_rows(kb + 2 * kTileBytes, kb + 3 * kTileBytes, prm.v, ktok, kvalid, warp, lane);
            cp_async_commit();
        };
        auto next_kv = [&](int u) {
            while (u < I.nkv && !((I.act >> u) & 1u)) ++u;
            return u;
        };
        copy_rows(q0, q1, prm.q, qtok, qvalid, warp, lane);
        cp_async_commit();
        int u = next_kv(0), b = 0, ki = 0, kj = 0;
        if (u < I.nkv) kv_stage(u, 0, ki, kj);
        cp_async_wait<0>();
        __syncwarp();
        rotate_row(q0, q1, pi, pj);
        float o[64];
#pragma unroll
        for (int e = 0; e < 64; ++e) o[e] = 0.f;
        float m = -INFINITY, l = 0.f;
        while (u < I.nkv && ok) {
            const long long kt = I.kv0 + u;
            const int un = next_kv(u + 1);
            const int koff = kKVOff + b * kKVBytes;
            cp_async_wait<0>();
            __syncwarp();
            rotate_row(smem + koff, smem + koff + kTileBytes, ki, kj);
            fence_proxy_async_smem();
            if (!group_sync(0x6104)) { ok = false; break; }  // every Q' and K' row rotated
            if (r == 0) {
                tc_fence_after();
#pragma unroll
                for (int hf = 0; hf < kHalves; ++hf)
#pragma unroll
                    for (int k = 0; k < kHeadDim / 16; ++k)
                        umma_ss(tmem + kColS, dK0 + ((kQOff + hf * kTileBytes) >> 4) + 2 * k,
                                dK0 + ((koff + hf * kTileBytes) >> 4) + 2 * k, id_s, (hf | k) != 0);
                umma_commit(&bars->s_full);
            }
            // the next tile's rows go to the other buffer, whose products (the
            // previous tile's) have completed
            int nki = 0, nkj = 0;
            if (un < I.nkv) kv_stage(un, b ^ 1, nki, nkj);
            const uint32_t a16 = I.masked ? d_allow16(g, myseg, kt, I.win) : 0xFFu;
            if (!wwait(&bars->s_full, sph, 0x6105)) { ok = false; break; }
            sph ^= 1;
            tc_fence_after();
            // row maximum of the attended raw scores
            float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t v[32];
                tmem_ld32(trow + kColS + 32 * c, v);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    if (!((a16 >> (2 * c + (e >> 4))) & 1u)) v[e] = __float_as_uint(-INFINITY);
#pragma unroll
                for (int e = 0; e < 32; e += 2)
                    mx4[(e >> 1) & 3] = fmax3(mx4[(e >> 1) & 3], __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
            }
            const float m_tile = fmaxf(fmax3(mx4[0], mx4[1], mx4[2]), mx4[3]) * sl2;
            if (m_tile > m + 8.f) {  // the conditional rescale of the d = 32 forward
                const float alpha = ex2_approx(m - m_tile);
#pragma unroll
                for (int e = 0; e < 64; ++e) o[e] *= alpha;
                l *= alpha;
                m = m_tile;
            }
            const float mu = (m == -INFINITY) ? 0.f : m;
            float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t v[32];
                tmem_ld32(trow + kColS + 32 * c, v);
                tmem_wait_ld();
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
                tmem_st16(trow + kColP + 16 * c, w);  // over columns of S already read
            }
            l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
            tmem_wait_st();
            tc_fence_before();
            if (!group_sync(0x6106)) { ok = false; break; }  // every row's P written
            if (r == 0) {
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < kTile / 16; ++k)
                    umma_ts(tmem + kColO, tmem + kColP + 8 * k, dMN0 + ((koff + 2 * kTileBytes) >> 4) + 64 * k, id_pv,
                            k > 0);
                umma_commit(&bars->o_full);
            }
            if (!wwait(&bars->o_full, oph, 0x6107)) { ok = false; break; }
            oph ^= 1;
            tc_fence_after();
#pragma unroll
            for (int hf = 0; hf < kHalves; ++hf) {
                uint32_t v[32];
                tmem_ld32(trow + kColO + kHeadDim * hf, v);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) o[32 * hf + e] += __uint_as_float(v[e]);
            }
            tc_fence_before();  // ordered before the next tile's products by its group barrier
            u = un;
            b ^= 1;
            ki = nki;
            kj = nkj;
        }
        if (!ok) break;
        // epilogue: O / l staged over Q', coalesced stores, log-sum-exp
        const float inv = 1.f / l;
        {
            float x[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] = o[e] * inv;
            store_row_swz(q0, r, x);
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] = o[32 + e] * inv;
            store_row_swz(q1, r, x);
        }
        __syncwarp();
        store_rows(prm.o, q0, q1, qtok, qvalid, warp, lane);
        if (qvalid && prm.lse != nullptr) prm.lse[qtok] = (m + lg2_approx(l)) * 0.69314718055994530942f;
    }
    cp_async_wait<0>();  // a tile staged before a failed wait: its copies land before the CTA exits
    if (r == 0) {  // every MMA issued here has completed before the columns are freed
        umma_commit(&bars->done);
        mbar_wait(&bars->done, 0, ctl, 0x61ff);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace fwd

// ------------------------------------------------------------------ backward
namespace bwd {

// workspace: the dQ' accumulator, per-tile norms, d theta partials and scratch
struct WsLayout {
    size_t dqacc, nrm, rowv, part, part2, cnt, total;
};

__host__ __device__ inline size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

__host__ __device__ inline WsLayout ws_layout(const Geo& g) {
    const size_t ht = static_cast<size_t>(g.heads) * static_cast<size_t>(g.tiles);
    WsLayout L;
    size_t o = 0;
    L.dqacc = o; o += round256(ht * kTile * 64 * 4);   // fp32 [heads][tiles][128][64]
    L.nrm = o;   o += round256(ht * 8);                // max |dO row|^2, max |v row|^2 per (head, tile)
    L.rowv = o;  o += round256(ht * kTile * 8);        // per slot row: lse log2(e), D
    L.part = o;  o += round256(ht * 2 * 8 * 16 * 4);   // [heads][2 axes][tiles][8][16]
    L.part2 = o; o += round256(static_cast<size_t>(g.heads) * 2 * 64 * 16 * 4);
    L.cnt = o;   o += round256(static_cast<size_t>(g.heads) * 2 * 4);
    L.total = o;
    return L;
}

struct Params {
    Geo g;
    const uint8_t *q, *k, *v, *o, *dout;  // bf16 [B, H, W, heads, 64]
    uint8_t *dq, *dk, *dv;
    const float *lse, *theta;
    uint8_t* ws;
    WsLayout L;
    unsigned int* status;
    unsigned long long limit_ns;
    long long items;
    float scale;
};

__device__ __forceinline__ void load_row64(const uint8_t* base, long long tok, float (&a)[32], float (&b)[32]) {
    const uint4* p = reinterpret_cast<const uint4*>(base + tok * kWideRowBytes);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint4 v = p[c];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float* x = c < 4 ? a : b;
            const int i = 8 * (c & 3) + 2 * e;
            x[i] = bf16lo_to_f32(w[e]);
            x[i + 1] = bf16hi_to_f32(w[e]);
        }
    }
}

// d theta terms of one token side: pos * (dx_b x_a - dx_a x_b) per pair, the
// rotation-invariant cross product, added into part[axis * 16 + k].
__device__ __forceinline__ void dtheta_terms(float (&part)[32], const float (&dx)[32], const float (&x)[32], float pos,
                                             int axis) {
#pragma unroll
    for (int k = 0; k < kPairs; ++k)
        part[axis * kPairs + k] += pos * (dx[2 * k + 1] * x[2 * k] - dx[2 * k] * x[2 * k + 1]);
}

// The warp's 32 d theta partials, summed over the warp in a fixed order, to
// part[((h * 2 + axis) * tiles + T) * 8 + slot][k].
__device__ __forceinline__ void write_partials(const float (&part)[32], float* out, const Geo& g, int h, long long T,
                                               int slot, int lane) {
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        float v = part[e];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        const int axis = e >> 4, k = e & 15;
        if (lane == k)
            out[(((static_cast<long long>(h) * 2 + axis) * g.tiles + T) * 8 + slot) * 16 + k] = v;
    }
}

// prep: per (tile, head), thread = slot row: the tile's largest squared norms of
// dO and v rows, and the zeroed dQ' accumulator rows; block 0 zeroes the d theta
// reduction's counters.
__global__ void __launch_bounds__(128) prep_kernel(const Params p) {
    __shared__ float2 nrm_w[4];
    const Geo& g = p.g;
    const long long T = blockIdx.x / g.heads;
    const int h = static_cast<int>(blockIdx.x - T * g.heads);
    const long long ht = static_cast<long long>(h) * g.tiles + T;
    const int r = threadIdx.x;
    if (blockIdx.x == 0)
        for (int i = r; i < 2 * g.heads; i += blockDim.x) reinterpret_cast<unsigned int*>(p.ws + p.L.cnt)[i] = 0u;
    int pi, pj;
    long long tok;
    float ndo = 0.f, nv = 0.f, D = 0.f, lse2 = INFINITY;
    if (slot_token(g, T, r, h, &pi, &pj, &tok)) {
        float a[32], b[32], c[32], d[32];
        load_row64(p.dout, tok, a, b);
        load_row64(p.o, tok, c, d);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            ndo = fmaf(a[e], a[e], fmaf(b[e], b[e], ndo));
            D = fmaf(a[e], c[e], fmaf(b[e], d[e], D));
        }
        load_row64(p.v, tok, a, b);
#pragma unroll
        for (int e = 0; e < 32; ++e) nv = fmaf(a[e], a[e], fmaf(b[e], b[e], nv));
        lse2 = __ldg(p.lse + tok) * 1.4426950408889634f;
    }
    // D = dO . O and lse in log2 units per slot row, staged by the main kernel
    reinterpret_cast<float2*>(p.ws + p.L.rowv)[ht * kTile + r] = make_float2(lse2, D);
    // the key side of d theta: the main kernel writes one slot per run of items of a
    // head in a CTA, the other slots 4..7 of the head's tiles must read zero
    {
        const int axis = r >> 6, i = r & 63;
        reinterpret_cast<float*>(p.ws + p.L.part)[(((static_cast<long long>(h) * 2 + axis) * g.tiles + T) * 8 + 4) * 16 + i] =
            0.f;
    }
    uint4* acc = reinterpret_cast<uint4*>(p.ws + p.L.dqacc + (ht * kTile + r) * 64 * 4);
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

// Main kernel: two warpgroups of four warps; warp w serves TMEM lanes (key rows)
// 32 (w & 3) .. + 31, and the warpgroups split each step's work: the column
// halves of S^T and dP^T, the row staging (k and q with their rotation: group
// 0; v, dO, D and lse2: group 1), the two 32-channel halves of dQ', and the
// item's end (dk and d theta: group 0; dv: group 1).
constexpr int kThreads = 256;
constexpr int kKOff = 0;                               // K' half tiles
constexpr int kVOff = kKOff + kHalves * kTileBytes;    // V half tiles
constexpr int kBufOff = kVOff + kHalves * kTileBytes;  // two query buffers: Q' half tiles, dO half tiles
constexpr int kBufBytes = 2 * kHalves * kTileBytes;
constexpr int kDSOff = kBufOff + 2 * kBufBytes;        // dS', MN-major 128-byte swizzle (1024-aligned)
constexpr int kVecOff = kDSOff + 4 * kTileBytes;       // per buffer: lse2[128], D[128]
constexpr int kTabOff = kVecOff + 2 * 2 * kTile * 4;
constexpr int kBarOff = kTabOff + kTabBytes;
constexpr int kSmemBytes = kBarOff + 256 + 1024;
static_assert(kDSOff % 1024 == 0, "128-byte swizzled operand must be 1024-byte aligned");
constexpr uint32_t kTmemCols = 512;
// S^T [0,128), dP^T [128,256); dV [256,320), dK' [320,384); P'^T (bf16) [384,448)
// and dS'^T (fp16) [448,512), apart from S^T and dP^T because the two
// warpgroups read and write different column halves at once; dQ' over S^T's
// consumed [64,128).
constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 320, kColP = 384, kColDS = 448, kColDQ = 64;

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
    const uint32_t id_s = make_idesc(kTile, kTile, false, false, true);    // fp16 K', Q'
    const uint32_t id_dp = make_idesc(kTile, kTile, false, false, false);  // bf16 V, dO
    // the gradient products take both half tiles in one N = 64 product: the
    // MN-major B operand's 64-byte swizzle atoms (32 channels) follow each other
    // at the descriptor's leading byte offset, one half tile apart
    const uint32_t id_dv = make_idesc(kTile, 64, false, true, false);  // P'^T (TMEM) x dO
    const uint32_t id_dk = make_idesc(kTile, 64, false, true, true);   // dS'^T (TMEM) x Q'
    const uint32_t id_dq = make_idesc(kTile, 64, true, true, true);    // dS' (smem) x K'
    const uint32_t sbase = smem_u32(smem);
    const uint64_t dK0 = make_sdesc(sbase, 16, 512, kSw64);
    const uint64_t dMN0 = make_sdesc(sbase, 8192, 512, kSw64);
    const uint64_t dDS = make_sdesc(sbase + kDSOff, 16384, 1024, kSw128);
    auto u16 = [](int bytes) { return static_cast<uint64_t>(bytes >> 4); };
    const float sl2 = g.scale_log2;
    float2* tab = reinterpret_cast<float2*>(smem + kTabOff);
    float* vec = reinterpret_cast<float*>(smem + kVecOff);  // buffer b: lse2 at [256 b], D at [256 b + 128]
    uint8_t* ds = smem + kDSOff;
    uint8_t* kh[2] = {smem + kKOff, smem + kKOff + kTileBytes};
    uint8_t* vh[2] = {smem + kVOff, smem + kVOff + kTileBytes};
    float* dqacc = reinterpret_cast<float*>(prm.ws + prm.L.dqacc);
    uint32_t gph = 0, sph = 0, mph = 0;
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
    auto rotate_row = [&](uint8_t* h0, uint8_t* h1, int pi, int pj) {
        float x[32];
        load_row_swz(h0, r, x, false);
        rope_half(x, pj, tab, false);
        store_row_swz(h0, r, x, true);
        load_row_swz(h1, r, x, false);
        rope_half(x, pi, tab + kPairs * 64, false);
        store_row_swz(h1, r, x, true);
    };
    // key side of d theta, summed over this CTA's run of items of one head (items
    // go head by head) and written once per run, to slot 4 + quad of the run's
    // first key tile
    float part[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) part[e] = 0.f;
    int run_head = -1;
    long long run_tile = 0;
    auto flush_partials = [&]() {
        if (wg == 0 && run_head >= 0)
            write_partials(part, reinterpret_cast<float*>(prm.ws + prm.L.part), g, run_head, run_tile, 4 + quad, lane);
#pragma unroll
        for (int e = 0; e < 32; ++e) part[e] = 0.f;
    };

    for (long long it = blockIdx.x; it < prm.items && ok; it += gridDim.x) {
        const BwdItem I = d_bwd_item(g, it);
        if (I.h != run_head) {  // a new run of items of one head
            flush_partials();
            run_head = I.h;
            run_tile = I.u;
        }
        if (I.h != tab_head) {
            if (!group_sync(0x6201)) break;
            build_table(tab, prm.theta + I.h * 2 * kPairs, g.M, tid, kThreads);
            if (!group_sync(0x6202)) break;
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
        // this thread's key row: K rotated (group 0), V (group 1)
        int ki, kj;
        long long ktok;
        const bool kvalid = slot_token(g, I.u, r, I.h, &ki, &kj, &ktok);
        const uint32_t keyseg = I.masked ? seg_at(d_tile_segs(g, I.u, I.win), r >> g.lBT) : 0u;
        if (!group_sync(0x6203)) break;  // the previous item's K', V rows are read by every thread
        if (wg == 0) {
            copy_rows(kh[0], kh[1], prm.k, ktok, kvalid, quad, lane);
            cp_async_commit();
            cp_async_wait<0>();
            __syncwarp();
            rotate_row(kh[0], kh[1], ki, kj);
        } else {
            copy_rows(vh[0], vh[1], prm.v, ktok, kvalid, quad, lane);
            cp_async_commit();
        }
        bool first = true;
        // Query steps, double-buffered: the copies, D and lse2 of the next active
        // query tile are issued while the current step's products run.
        auto stage = [&](int n, int b, int& qi, int& qj, bool& qvalid) {
            long long qtok;
            qvalid = slot_token(g, I.q0 + n, r, I.h, &qi, &qj, &qtok);
            uint8_t* qb = smem + kBufOff + b * kBufBytes;
            if (wg == 0) {
                copy_rows(qb, qb + kTileBytes, prm.q, qtok, qvalid, quad, lane);
                cp_async_commit();
            } else {
                copy_rows(qb + 2 * kTileBytes, qb + 3 * kTileBytes, prm.dout, qtok, qvalid, quad, lane);
                cp_async_commit();
                // lse2 and D of the row, from the prep kernel (lse2 = +inf for a padded row)
                const float2 ld = __ldcg(reinterpret_cast<const float2*>(prm.ws + prm.L.rowv) +
                                         ((static_cast<long long>(I.h) * g.tiles + I.q0 + n) * kTile + r));
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
            if (wg == 0) rotate_row(smem + qoff, smem + qoff + kTileBytes, qi, qj);
            fence_proxy_async_smem();
            if (!group_sync(0x6204)) { ok = false; break; }  // rows staged and rotated
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int hf = 0; hf < kHalves; ++hf)
#pragma unroll
                    for (int k = 0; k < kHeadDim / 16; ++k) {
                        umma_ss(tmem + kColS, dK0 + u16(kKOff + hf * kTileBytes) + 2 * k,
                                dK0 + u16(qoff + hf * kTileBytes) + 2 * k, id_s, (hf | k) != 0);
                        umma_ss(tmem + kColDP, dK0 + u16(kVOff + hf * kTileBytes) + 2 * k,
                                dK0 + u16(dooff + hf * kTileBytes) + 2 * k, id_dp, (hf | k) != 0);
                    }
                umma_commit(&bars->s_full);
            }
            // the next step's rows go to the other buffer, whose products (the previous
            // step's) have completed
            int nqi = 0, nqj = 0;
            bool nqvalid = false;
            if (nn < I.nq) stage(nn, b ^ 1, nqi, nqj, nqvalid);
            const uint32_t a16 = I.masked ? d_allow16(g, keyseg, T, I.win) : 0xFFu;
            if (!wwait(&bars->s_full, sph, 0x6205)) { ok = false; break; }
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
            if (!group_sync(0x6206)) { ok = false; break; }  // every row's P'^T, dS'^T and dS' written
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
            if (!wwait(&bars->mma_done, mph, 0x6207)) { ok = false; break; }
            mph ^= 1;
            tc_fence_after();
            // this query row's dQ' half (the group's 32 channels), softmax scale and
            // 2^-e applied, added into the accumulator
            {
                const float sc = prm.scale * exp2i(-gexp);
                float* accrow = dqacc + ((static_cast<long long>(I.h) * g.tiles + T) * kTile + r) * 64 + 32 * wg;
                uint32_t v[32];
                tmem_ld32(trow + kColDQ + kHeadDim * wg, v);
                tmem_wait_ld();
                if (qvalid) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        red_add_v4(accrow + e, __uint_as_float(v[e]) * sc, __uint_as_float(v[e + 1]) * sc,
                                   __uint_as_float(v[e + 2]) * sc, __uint_as_float(v[e + 3]) * sc);
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
        // item end: group 0 dk (dK' un-rotated) and the key side of d theta, group 1 dv
        const float down = exp2i(-gexp);
        uint8_t* const* st = wg == 0 ? kh : vh;
        if (first) {  // no query tile attends these keys (cannot happen: a key attends itself)
            float z[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) z[e] = 0.f;
            store_row_swz(st[0], r, z);
            store_row_swz(st[1], r, z);
        } else {
#pragma unroll 1
            for (int hf = 0; hf < kHalves; ++hf) {
                uint32_t t[32];
                float dx[32];
                tmem_ld32(trow + (wg == 0 ? kColDK : kColDV) + kHeadDim * hf, t);
                tmem_wait_ld();
                if (wg == 0) {
                    float x[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) dx[e] = __uint_as_float(t[e]) * (prm.scale * down);
                    load_row_swz(kh[hf], r, x, true);  // rotated k' (fp16)
                    if (kvalid) dtheta_terms(part, dx, x, static_cast<float>(hf ? ki : kj), hf);
                    rope_half(dx, hf ? ki : kj, tab + hf * kPairs * 64, true);
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) dx[e] = __uint_as_float(t[e]) * down;
                }
                store_row_swz(st[hf], r, dx);  // dk staged over k', dv over v (bf16)
            }
        }
        tc_fence_before();
        __syncwarp();
        store_rows(wg == 0 ? prm.dk : prm.dv, st[0], st[1], ktok, kvalid, quad, lane);
    }
    flush_partials();
    cp_async_wait<0>();  // a step staged before a failed wait: its copies land before the CTA exits
    if (tid == 0) {
        umma_commit(&bars->done);
        mbar_wait(&bars->done, 0, ctl, 0x62ff);
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
    build_table(tab, p.theta + h * 2 * kPairs, g.M, threadIdx.x, blockDim.x);
    __syncthreads();
    const int r = threadIdx.x, lane = r & 31, warp = r >> 5;
    int pi, pj;
    long long tok;
    float part[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) part[e] = 0.f;
    if (slot_token(g, T, r, h, &pi, &pj, &tok)) {
        const float* acc = reinterpret_cast<const float*>(p.ws + p.L.dqacc) + (ht * kTile + r) * 64;
        float q0[32], q1[32];
        load_row64(p.q, tok, q0, q1);
        uint4* dst = reinterpret_cast<uint4*>(p.dq + tok * kWideRowBytes);
#pragma unroll 1
        for (int hf = 0; hf < kHalves; ++hf) {
            float dx[32];
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
                const float4 a4 = *reinterpret_cast<const float4*>(acc + 32 * hf + e);
                dx[e] = a4.x;
                dx[e + 1] = a4.y;
                dx[e + 2] = a4.z;
                dx[e + 3] = a4.w;
            }
            rope_half(dx, hf ? pi : pj, tab + hf * kPairs * 64, true);
            dtheta_terms(part, dx, hf ? q1 : q0, static_cast<float>(hf ? pi : pj), hf);
#pragma unroll
            for (int c = 0; c < 4; ++c) dst[4 * hf + c] = pack_chunk(dx, c);
        }
    }
    write_partials(part, reinterpret_cast<float*>(p.ws + p.L.part), g, h, T, warp, lane);
}

}  // namespace bwd

}  // namespace widek

size_t wide_bwd_workspace_bytes(const Geo& g) { return widek::bwd::ws_layout(g).total; }

cudaError_t launch_wide_fwd(const Geo& g, const void* q, const void* k, const void* v, const float* theta, void* o,
                            float* lse, unsigned int* status, unsigned long long limit_ns, int num_sms,
                            cudaStream_t stream, cudaEvent_t const* events) {
    using namespace widek;
    static SmemOptIn optin;
    if (cudaError_t e = optin.ensure(reinterpret_cast<const void*>(fwd::fwd_kernel), fwd::kSmemBytes)) return e;
    fwd::Params prm;
    prm.g = g;
    prm.q = static_cast<const uint8_t*>(q);
    prm.k = static_cast<const uint8_t*>(k);
    prm.v = static_cast<const uint8_t*>(v);
    prm.o = static_cast<uint8_t*>(o);
    prm.theta = theta;
    prm.lse = lse;
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

cudaError_t launch_wide_bwd(const Geo& g, const BwdPtrs& p, unsigned int* status, unsigned long long limit_ns,
                            int num_sms, cudaStream_t stream, cudaEvent_t const* events) {
    using namespace widek;
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
    prm.ws = p.ws;
    prm.L = L;
    prm.status = status;
    prm.limit_ns = limit_ns;
    prm.items = bwd_item_count(g);
    prm.scale = 0.125f;  // 1/sqrt(64)
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
    // d theta: [heads][2 axes] sums of [tiles * 8][16] partials, as heads * 2 rows of 16
    if (e == cudaSuccess)
        e = bwdk::launch_dtheta(reinterpret_cast<const float*>(p.ws + L.part), g.tiles * 8, 2 * g.heads,
                                reinterpret_cast<float*>(p.ws + L.part2), reinterpret_cast<unsigned int*>(p.ws + L.cnt),
                                p.dtheta, stream);
    mark(4);
    return e;
}

}  // namespace fswin
