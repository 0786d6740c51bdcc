// Window / box / tile geometry of the shifted-window token grid.
//
// Tokens of one head are enumerated window by window (windows in the rolled
// frame, image-major), and inside a window box by box, where a box is a
// bh x bw rectangle of tokens that never straddles the wrap-around of the
// cyclic shift.  A "tile" is 128 consecutive token slots of that enumeration:
// the row block of one tcgen05 MMA.  Attention happens inside a "group": a
// window when a window holds >= 128 tokens (several tiles per window), or a
// tile when windows are smaller (several windows per tile, separated by a
// block-diagonal mask).  Two tokens attend to each other iff they share the
// window and the shift-region label (the Swin shifted-window rule).
//
// A grid whose H or W is not a multiple of M is padded at the bottom and right
// to Hp x Wp (the next multiples of M) with zero tokens, as a Swin layer pads
// its input: windows, the roll and the region labels refer to the padded grid,
// padded tokens take part in the softmax, and only real positions are read
// from or written to memory.
//
// Every extent below is a power of two, so the per-row and per-tile helpers
// use shifts and masks.  The few divisions by other set-up constants (windows
// per image, tiles per head) use 32-bit division by invariant integers.
#pragma once

#include <cstdint>

namespace fswin {

// Unsigned 32-bit division by a divisor fixed at set-up: one multiply-high, a
// subtract, an add and two shifts (T. Granlund and P. L. Montgomery, "Division
// by invariant integers using multiplication", PLDI 1994, section 4: the
// multiplier m' = floor(2^32 (2^l - d) / d) + 1 with l = ceil(log2 d)).
struct FastDiv {
    uint32_t d, m, s1, s2;
};

inline FastDiv make_fastdiv(uint32_t d) {  // 1 <= d <= 2^31
    FastDiv f;
    f.d = d;
    int l = 0;
    while ((1ull << l) < d) ++l;
    f.m = static_cast<uint32_t>(((1ull << 32) * ((1ull << l) - d)) / d + 1);
    f.s1 = l > 0 ? 1u : 0u;
    f.s2 = l > 0 ? static_cast<uint32_t>(l - 1) : 0u;
    return f;
}

__host__ __device__ inline uint32_t fdiv(const FastDiv& f, uint32_t n) {
#ifdef __CUDA_ARCH__
    const uint32_t t = __umulhi(f.m, n);
#else
    const uint32_t t = static_cast<uint32_t>((static_cast<uint64_t>(f.m) * n) >> 32);
#endif
    return (t + ((n - t) >> f.s1)) >> f.s2;
}

constexpr int kTile = 128;                  // token rows per tile
constexpr int kHeadDim = 32;                // channels of one tile row (a d = 64 head takes two)
constexpr int kRowBytes = kHeadDim * 2;     // one 16-bit token row
constexpr int kTileBytes = kTile * kRowBytes;

struct Geo {
    int B, H, W, heads, M, s;   // H, W: the tokens in memory
    int Hp, Wp;         // the grid padded to multiples of M
    int nWw, nW;        // windows per image row, per image
    int N;              // tokens per window
    int bh, bw, BT;     // box rows, box cols, tokens per box
    int nbc, nbw;       // boxes per window row, per window
    int bpt;            // boxes per tile
    int tpw;            // tiles per window (N >= 128), else 0
    int wpt;            // windows per tile (N < 128), else 0
    int lbh, lbw, lBT, lnbc, lnbw, lbpt, ltpw, lwpt;  // log2 of the above
    long long wins;     // windows in the batch
    long long tiles;    // tiles per head
    float scale_log2;   // log2(e) / sqrt(d)
    FastDiv fd_nW, fd_nWw, fd_tiles, fd_heads;  // window, tile and item indices fit 32 bits
    int d;              // head dimension: 32, or 64 (the wide kernels)
};

__host__ __device__ inline int ilog2_exact(int x) {
    int l = 0;
    while ((1 << l) < x) ++l;
    return l;
}

// Builds the geometry of a problem.  Returns 0 on success, 2 for an
// unsupported shape (the FS_ERR_SHAPE code of the C ABI).
inline int geo_init(Geo* g, int B, int H, int W, int heads, int d, int M, int s) {
    if (d != 32 && d != 64) return 2;
    if (!(M == 4 || M == 8 || M == 16 || M == 32 || M == 64)) return 2;
    if (B < 0 || heads < 1 || H < M || W < M) return 2;
    if (s < 0 || s >= M || s % 4) return 2;
    if (H > (1 << 24) || W > (1 << 24) || heads > 4096) return 2;
    const int Hp = (H + M - 1) / M * M, Wp = (W + M - 1) / M * M;
    // token, window, tile and work-item indices of one head stay below 2^31
    if (static_cast<long long>(B) * Hp * Wp > (1ll << 31)) return 2;
    if (static_cast<long long>(B) * Hp * Wp * heads > (1ll << 37)) return 2;
    int a = M, b = s;  // box side: gcd(M, s), or M without shift
    while (b) {
        const int t = a % b;
        a = b;
        b = t;
    }
    const int side = s ? a : M;
    Geo x{};
    x.B = B;
    x.H = H;
    x.W = W;
    x.Hp = Hp;
    x.Wp = Wp;
    x.heads = heads;
    x.d = d;
    x.M = M;
    x.s = s;
    x.nWw = Wp / M;
    x.nW = (Hp / M) * (Wp / M);
    x.N = M * M;
    x.bw = side < kTile ? side : kTile;
    x.bh = side < kTile / x.bw ? side : kTile / x.bw;
    x.BT = x.bh * x.bw;
    x.nbc = M / x.bw;
    x.nbw = (M / x.bh) * (M / x.bw);
    x.bpt = kTile / x.BT;
    x.tpw = x.N >= kTile ? x.N / kTile : 0;
    x.wpt = x.N < kTile ? kTile / x.N : 0;
    x.lbh = ilog2_exact(x.bh);
    x.lbw = ilog2_exact(x.bw);
    x.lBT = ilog2_exact(x.BT);
    x.lnbc = ilog2_exact(x.nbc);
    x.lnbw = ilog2_exact(x.nbw);
    x.lbpt = ilog2_exact(x.bpt);
    x.ltpw = x.tpw ? ilog2_exact(x.tpw) : 0;
    x.lwpt = x.wpt ? ilog2_exact(x.wpt) : 0;
    x.wins = static_cast<long long>(B) * x.nW;
    x.tiles = (x.wins * x.N + kTile - 1) / kTile;
    x.scale_log2 = 1.4426950408889634f / (d == 64 ? 8.0f : 5.656854249492380195f);  // log2(e) / sqrt(d)
    x.fd_nW = make_fastdiv(static_cast<uint32_t>(x.nW));
    x.fd_nWw = make_fastdiv(static_cast<uint32_t>(x.nWw));
    x.fd_tiles = make_fastdiv(static_cast<uint32_t>(x.tiles > 0 ? x.tiles : 1));
    x.fd_heads = make_fastdiv(static_cast<uint32_t>(heads));
    *g = x;
    return 0;
}

__host__ __device__ inline int region_of(int X, int M, int s, int x) {
    return x < X - M ? 0 : (x < X - s ? 1 : 2);
}

// A window of the batch in the rolled frame.
struct Win {
    long long gw;
    int b, wr, wc;
    bool valid;
};

__host__ __device__ inline Win win_of(const Geo& g, long long gw) {
    Win w;
    w.gw = gw;
    w.valid = gw < g.wins;
    const uint32_t g32 = static_cast<uint32_t>(gw);
    w.b = static_cast<int>(fdiv(g.fd_nW, g32));  // >= B for padding windows: TMA then zero-fills
    const uint32_t r = g32 - static_cast<uint32_t>(w.b) * g.nW;
    w.wr = static_cast<int>(fdiv(g.fd_nWw, r));
    w.wc = static_cast<int>(r) - w.wr * g.nWw;
    return w;
}

// Box x (0 .. bpt-1) of a tile: its window and its index k inside the window.
__host__ __device__ inline void tile_box(const Geo& g, long long tile, int x, long long* gw, int* k) {
    if (g.tpw) {
        *gw = tile >> g.ltpw;
        *k = (static_cast<int>(tile & (g.tpw - 1)) << g.lbpt) + x;
    } else {
        *gw = (tile << g.lwpt) + (x >> g.lnbw);
        *k = x & (g.nbw - 1);
    }
}

// Rolled coordinates of the first token of box k of window w.
__host__ __device__ inline int box_r(const Geo& g, const Win& w, int k) { return w.wr * g.M + ((k >> g.lnbc) << g.lbh); }
__host__ __device__ inline int box_c(const Geo& g, const Win& w, int k) {
    return w.wc * g.M + ((k & (g.nbc - 1)) << g.lbw);
}

__host__ __device__ inline int box_label(const Geo& g, const Win& w, int k) {
    if (!g.s) return 0;
    return 3 * region_of(g.Hp, g.M, g.s, box_r(g, w, k)) + region_of(g.Wp, g.M, g.s, box_c(g, w, k));
}

// Original (un-rolled) coordinates of the first token of box k of window w, in
// the padded grid: the box lies wholly or partly outside the H x W tokens in
// memory when row0 + bh > H or col0 + bw > W (a box never straddles the wrap:
// Hp - s and Wp - s are multiples of the box side).
__host__ __device__ inline void box_origin(const Geo& g, const Win& w, int k, int* row0, int* col0) {
    int r = box_r(g, w, k) + g.s, c = box_c(g, w, k) + g.s;
    if (r >= g.Hp) r -= g.Hp;
    if (c >= g.Wp) c -= g.Wp;
    *row0 = r;
    *col0 = c;
}

// In-window position (i = row, j = column) of token slot p of a tile.
__host__ __device__ inline void tile_row_pos(const Geo& g, long long tile, int p, int* i, int* j) {
    const int k = g.tpw ? (static_cast<int>(tile & (g.tpw - 1)) << g.lbpt) + (p >> g.lBT) : (p & (g.N - 1)) >> g.lBT;
    const int q = p & (g.BT - 1);
    *i = ((k >> g.lnbc) << g.lbh) + (q >> g.lbw);
    *j = ((k & (g.nbc - 1)) << g.lbw) + (q & (g.bw - 1));
}

// Segment byte of every box of a tile: (window index inside the tile << 4) |
// region label.  Two tokens of one group attend iff their boxes' bytes match.
// `w0` is the tile's (first) window, computed by the caller with win_of.
__host__ __device__ inline uint64_t tile_segs(const Geo& g, long long tile, const Win& w0) {
    uint64_t out = 0;
    if (g.tpw) {
        if (!g.s) return 0;
        const int k0 = static_cast<int>(tile & (g.tpw - 1)) << g.lbpt;
        for (int x = 0; x < g.bpt; ++x) out |= static_cast<uint64_t>(box_label(g, w0, k0 + x)) << (8 * x);
        return out;
    }
    Win w = w0;
    for (int x = 0; x < g.bpt; ++x) {
        const int widx = x >> g.lnbw, k = x & (g.nbw - 1);
        if (k == 0 && widx > 0) w = win_of(g, w0.gw + widx);
        out |= static_cast<uint64_t>((widx << 4) | box_label(g, w, k)) << (8 * x);
    }
    return out;
}

// First window of a tile.
__host__ __device__ inline Win tile_win(const Geo& g, long long tile) {
    return win_of(g, g.tpw ? (tile >> g.ltpw) : (tile << g.lwpt));
}

__host__ __device__ inline uint32_t seg_at(uint64_t segs, int box) { return static_cast<uint32_t>(segs >> (8 * box)) & 0xFFu; }

// Does some token of tile a attend some token of tile b (same group)?
__host__ __device__ inline bool segs_meet(const Geo& g, uint64_t a, uint64_t b) {
    for (int x = 0; x < g.bpt; ++x)
        for (int y = 0; y < g.bpt; ++y)
            if (seg_at(a, x) == seg_at(b, y)) return true;
    return false;
}

// Bit c (0..7): may a token with segment byte `my` attend the 16 tokens in
// slots [16 c, 16 c + 16) of a tile with segment bytes `segs`?  (Boxes hold
// >= 16 tokens, so a 16-slot group never spans two boxes.)
__host__ __device__ inline uint32_t allow16(const Geo& g, uint32_t my, uint64_t segs) {
    uint32_t m = 0;
    for (int c = 0; c < 8; ++c)
        if (seg_at(segs, (c << 4) >> g.lBT) == my) m |= 1u << c;
    return m;
}

// ----------------------------------------------------------------- slow path
// Full description of a box / token slot (used once per work item at most).
struct Box {
    int b;            // image (>= B for padding boxes)
    int row0, col0;   // original coordinates of the first token
    int i0, j0;       // in-window coordinates of the first token
    long long gw;     // window index within the batch
    int label;        // shift-region label (0 when s == 0)
    bool valid;
};

__host__ __device__ inline Box box_of(const Geo& g, long long gbox) {
    Box x;
    long long gw;
    int k;
    tile_box(g, gbox >> g.lbpt, static_cast<int>(gbox & (g.bpt - 1)), &gw, &k);
    const Win w = win_of(g, gw);
    x.gw = gw;
    x.valid = w.valid;
    x.b = w.b;
    x.i0 = (k >> g.lnbc) << g.lbh;
    x.j0 = (k & (g.nbc - 1)) << g.lbw;
    x.label = box_label(g, w, k);
    box_origin(g, w, k, &x.row0, &x.col0);
    return x;
}

struct Slot {
    Box box;
    int i, j;        // in-window coordinates (RoPE positions: y = i, x = j)
    int row, col;    // original coordinates (in the padded grid)
    bool valid;      // a real token: a real window and row < H, col < W
};

__host__ __device__ inline Slot slot_of(const Geo& g, long long tile, int p) {
    Slot s;
    s.box = box_of(g, tile * g.bpt + (p >> g.lBT));
    const int q = p & (g.BT - 1), bi = q >> g.lbw, bj = q & (g.bw - 1);
    s.i = s.box.i0 + bi;
    s.j = s.box.j0 + bj;
    s.row = s.box.row0 + bi;
    s.col = s.box.col0 + bj;
    s.valid = s.box.valid && s.row < g.H && s.col < g.W;
    return s;
}

}  // namespace fswin
