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
#pragma once

#include <cstdint>

namespace fswin {

constexpr int kTile = 128;                  // token rows per tile
constexpr int kHeadDim = 32;                // supported head dimension
constexpr int kRowBytes = kHeadDim * 2;     // one bf16 token row
constexpr int kTileBytes = kTile * kRowBytes;

struct Geo {
    int B, H, W, heads, M, s;
    int nWw, nW;        // windows per image row, per image
    int N;              // tokens per window
    int bh, bw, BT;     // box rows, box cols, tokens per box
    int nbc, nbw;       // boxes per window row, per window
    int bpt;            // boxes per tile
    int tpw;            // tiles per window (N >= 128), else 0
    long long wins;     // windows in the batch
    long long tiles;    // tiles per head
    float scale_log2;   // log2(e) / sqrt(d)
};

// Builds the geometry of a problem.  Returns 0 on success, 2 for an
// unsupported shape (the FS_ERR_SHAPE code of the C ABI).
inline int geo_init(Geo* g, int B, int H, int W, int heads, int d, int M, int s) {
    if (d != kHeadDim) return 2;
    if (!(M == 4 || M == 8 || M == 16 || M == 32 || M == 64)) return 2;
    if (B < 0 || heads < 1 || H < M || W < M || H % M || W % M) return 2;
    if (s < 0 || s >= M || s % 4) return 2;
    if (H > (1 << 24) || W > (1 << 24) || heads > 4096) return 2;
    if (static_cast<long long>(B) * H * W * heads > (1ll << 40)) return 2;
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
    x.heads = heads;
    x.M = M;
    x.s = s;
    x.nWw = W / M;
    x.nW = (H / M) * (W / M);
    x.N = M * M;
    x.bw = side < kTile ? side : kTile;
    x.bh = side < kTile / x.bw ? side : kTile / x.bw;
    x.BT = x.bh * x.bw;
    x.nbc = M / x.bw;
    x.nbw = (M / x.bh) * (M / x.bw);
    x.bpt = kTile / x.BT;
    x.tpw = x.N >= kTile ? x.N / kTile : 0;
    x.wins = static_cast<long long>(B) * x.nW;
    x.tiles = (x.wins * x.N + kTile - 1) / kTile;
    x.scale_log2 = 1.4426950408889634f / 5.656854249492380195f;  // log2(e) / sqrt(32)
    *g = x;
    return 0;
}

__host__ __device__ inline int region_of(int X, int M, int s, int x) {
    return x < X - M ? 0 : (x < X - s ? 1 : 2);
}

struct Box {
    int b;            // image (>= B for padding boxes: TMA then zero-fills)
    int row0, col0;   // original (un-rolled) coordinates of the first token
    int i0, j0;       // in-window coordinates of the first token
    long long gw;     // window index within the batch
    int label;        // shift-region label (0 when s == 0)
    bool valid;
};

__host__ __device__ inline Box box_of(const Geo& g, long long gbox) {
    Box x;
    x.gw = gbox / g.nbw;
    const int k = static_cast<int>(gbox - x.gw * g.nbw);
    x.valid = x.gw < g.wins;
    x.b = static_cast<int>(x.gw / g.nW);
    const int w = static_cast<int>(x.gw - static_cast<long long>(x.b) * g.nW);
    const int wr = w / g.nWw, wc = w - (w / g.nWw) * g.nWw;
    const int br = k / g.nbc, bc = k - br * g.nbc;
    x.i0 = br * g.bh;
    x.j0 = bc * g.bw;
    const int r = wr * g.M + x.i0, c = wc * g.M + x.j0;
    x.label = g.s ? 3 * region_of(g.H, g.M, g.s, r) + region_of(g.W, g.M, g.s, c) : 0;
    x.row0 = (r + g.s) % g.H;
    x.col0 = (c + g.s) % g.W;
    return x;
}

// Segment key: tokens attend iff their segment keys are equal.
__host__ __device__ inline long long seg_of(const Box& x) { return x.gw * 9 + x.label; }

// Bit set of the region labels present in a tile.
__host__ __device__ inline uint32_t tile_labels(const Geo& g, long long tile) {
    uint32_t m = 0;
    for (int i = 0; i < g.bpt; ++i) m |= 1u << box_of(g, tile * g.bpt + i).label;
    return m;
}

// Token slot p (0..127) of a tile: its box and the in-box offset.
struct Slot {
    Box box;
    int i, j;        // in-window coordinates (RoPE positions: y = i, x = j)
    int row, col;    // original coordinates
};

__host__ __device__ inline Slot slot_of(const Geo& g, long long tile, int p) {
    Slot s;
    s.box = box_of(g, tile * g.bpt + p / g.BT);
    const int q = p % g.BT, bi = q / g.bw, bj = q - (q / g.bw) * g.bw;
    s.i = s.box.i0 + bi;
    s.j = s.box.j0 + bj;
    s.row = s.box.row0 + bi;
    s.col = s.box.col0 + bj;
    return s;
}

// For a query (or key) box segment `seg` and the boxes of another tile,
// the bit set of that tile's boxes whose tokens it may attend.
__host__ __device__ inline uint32_t allow_mask(const Geo& g, long long seg, long long other_tile) {
    uint32_t m = 0;
    for (int i = 0; i < g.bpt; ++i)
        if (seg_of(box_of(g, other_tile * g.bpt + i)) == seg) m |= 1u << i;
    return m;
}

}  // namespace fswin
