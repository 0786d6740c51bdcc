// Work items of the forward and backward kernels (host/device, so the
// scheduling can be checked on the CPU).  Each item carries bit masks of the
// (query tile, key tile) pairs that hold at least one attending token pair,
// computed once per item; the kernels' inner loops only test bits.
#pragma once

#include "geometry.cuh"

namespace fswin {

// Forward: a pair of 128-row query tiles A and B (B < 0: none) sharing one
// stream of key/value tiles.  Windows of >= 256 tokens: two query tiles of one
// window, key/value tiles = the window's tiles.  Smaller windows: two
// consecutive tiles, each attending only to itself.
struct FwdItem {
    int h;
    long long tA, tB;
    long long kv0;    // first key/value tile of the list
    int nkv;          // length of the key/value list (<= 32)
    bool paired;      // small windows: entry u of the list serves query tile u only
    uint32_t act[2];  // bit u: list entry u is used by query tile A / B
    Win win;          // the window (>= 256 tokens) or the first window of tile A
};

__host__ __device__ inline long long fwd_item_count(const Geo& g) {
    if (g.N >= 2 * kTile) return g.wins * g.heads * (g.tpw / 2);
    return ((g.tiles + 1) / 2) * g.heads;
}

__host__ __device__ inline uint32_t low_bits(int n) { return n >= 32 ? 0xFFFFFFFFu : ((1u << n) - 1u); }

// Items are ordered head-major: a persistent CTA walks items with a stride of
// the grid size, so consecutive items of a CTA almost always share the head
// (and its RoPE table).
__host__ __device__ inline FwdItem fwd_item(const Geo& g, long long it) {
    FwdItem I;
    if (g.N >= 2 * kTile) {
        const int pairs = g.tpw / 2;
        const long long per_head = g.wins * pairs;
        I.h = static_cast<int>(it / per_head);
        const long long rem = it - static_cast<long long>(I.h) * per_head;
        const long long gw = rem / pairs;
        const int pr = static_cast<int>(rem - gw * pairs);
        I.kv0 = gw * g.tpw;
        I.tA = I.kv0 + 2 * pr;
        I.tB = I.tA + 1;
        I.nkv = g.tpw;
        I.paired = false;
        I.win = win_of(g, gw);
        I.act[0] = I.act[1] = low_bits(g.tpw);
        if (g.s && (I.win.wr == g.H / g.M - 1 || I.win.wc == g.nWw - 1)) {
            const uint64_t sa = tile_segs(g, I.tA, I.win), sb = tile_segs(g, I.tB, I.win);
            I.act[0] = I.act[1] = 0;
            for (int u = 0; u < g.tpw; ++u) {
                const uint64_t su = tile_segs(g, I.kv0 + u, I.win);
                if (segs_meet(g, sa, su)) I.act[0] |= 1u << u;
                if (segs_meet(g, sb, su)) I.act[1] |= 1u << u;
            }
        }
    } else {
        const long long per_head = (g.tiles + 1) / 2;
        I.h = static_cast<int>(it / per_head);
        const long long x = it - static_cast<long long>(I.h) * per_head;
        I.tA = 2 * x;
        I.tB = 2 * x + 1 < g.tiles ? 2 * x + 1 : -1;
        I.kv0 = I.tA;
        I.nkv = I.tB >= 0 ? 2 : 1;
        I.paired = true;
        I.win = tile_win(g, I.tA);
        I.act[0] = 1u;
        I.act[1] = I.tB >= 0 ? 2u : 0u;
    }
    return I;
}

// Is key/value list entry u used by query tile T (0 = A, 1 = B)?
__host__ __device__ inline bool fwd_active(const Geo&, const FwdItem& I, int T, int u) {
    return (I.act[T] >> u) & 1u;
}

// Backward: one 128-key tile u and the query tiles of its group.
struct BwdItem {
    int h;
    long long u;    // key/value tile
    long long q0;   // first candidate query tile
    int nq;         // candidate query tiles (<= 32)
    bool paired;    // small windows: the only query tile is u
    uint32_t act;   // bit n: query tile q0 + n attends to u
    Win win;        // the window (>= 256 tokens) or the first window of tile u
};

__host__ __device__ inline long long bwd_item_count(const Geo& g) {
    if (g.N >= 2 * kTile) return g.wins * g.heads * g.tpw;
    return g.tiles * g.heads;
}

__host__ __device__ inline BwdItem bwd_item(const Geo& g, long long it) {
    BwdItem I;
    if (g.N >= 2 * kTile) {
        const long long per_head = g.wins * g.tpw;
        I.h = static_cast<int>(it / per_head);
        const long long rem = it - static_cast<long long>(I.h) * per_head;
        const long long gw = rem / g.tpw;
        I.q0 = gw * g.tpw;
        I.u = I.q0 + (rem - gw * g.tpw);
        I.nq = g.tpw;
        I.paired = false;
        I.win = win_of(g, gw);
        I.act = low_bits(g.tpw);
        if (g.s && (I.win.wr == g.H / g.M - 1 || I.win.wc == g.nWw - 1)) {
            const uint64_t su = tile_segs(g, I.u, I.win);
            I.act = 0;
            for (int n = 0; n < g.tpw; ++n)
                if (segs_meet(g, tile_segs(g, I.q0 + n, I.win), su)) I.act |= 1u << n;
        }
    } else {
        I.h = static_cast<int>(it / g.tiles);
        const long long T = it - static_cast<long long>(I.h) * g.tiles;
        I.u = T;
        I.q0 = T;
        I.nq = 1;
        I.paired = true;
        I.win = tile_win(g, T);
        I.act = 1u;
    }
    return I;
}

__host__ __device__ inline bool bwd_active(const Geo&, const BwdItem& I, int n) { return (I.act >> n) & 1u; }

}  // namespace fswin
