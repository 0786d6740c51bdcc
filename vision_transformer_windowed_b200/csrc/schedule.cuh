// Work items of the forward and backward kernels (host/device, so the
// scheduling can be checked on the CPU).  Each item carries bit masks of the
// (query tile, key tile) pairs that hold at least one attending token pair,
// computed once per item; the kernels' inner loops only test bits.
#pragma once

#include "geometry.cuh"

namespace fswin {

// Forward: one 128-row query tile X and the key/value tiles of its group
// (the window's tiles for windows of >= 128 tokens, X itself for smaller
// windows).  Items are ordered head-major: a persistent CTA walks items with a
// stride of the grid size, so consecutive items of a CTA almost always share
// the head (and its RoPE table).
struct FwdItem {
    int h;
    long long X;      // query tile
    long long kv0;    // first key/value tile of the group
    int nkv;          // key/value tiles in the group (<= 32)
    uint32_t act;     // bit u: tile kv0 + u holds keys that query tile X attends
    bool masked;      // some pairs of the group do not attend (the shift-region mask, or several windows per tile)
    Win win;          // the window (>= 128 tokens) or the first window of tile X
};

__host__ __device__ inline long long fwd_item_count(const Geo& g) { return g.tiles * g.heads; }

__host__ __device__ inline uint32_t low_bits(int n) { return n >= 32 ? 0xFFFFFFFFu : ((1u << n) - 1u); }

__host__ __device__ inline FwdItem fwd_item(const Geo& g, long long it) {
    FwdItem I;
    I.h = static_cast<int>(fdiv(g.fd_tiles, static_cast<uint32_t>(it)));
    I.X = it - static_cast<long long>(I.h) * g.tiles;
    if (g.tpw) {
        const long long gw = I.X >> g.ltpw;
        I.kv0 = gw * g.tpw;
        I.nkv = g.tpw;
        I.win = win_of(g, gw);
        I.act = low_bits(g.tpw);
        I.masked = g.s && (I.win.wr == g.Hp / g.M - 1 || I.win.wc == g.nWw - 1);
        if (I.masked) {
            const uint64_t sx = tile_segs(g, I.X, I.win);
            I.act = 0;
            for (int u = 0; u < g.tpw; ++u)
                if (segs_meet(g, sx, tile_segs(g, I.kv0 + u, I.win))) I.act |= 1u << u;
        }
    } else {
        I.kv0 = I.X;
        I.nkv = 1;
        I.win = tile_win(g, I.X);
        I.act = 1u;
        I.masked = true;
    }
    return I;
}

// Backward: one 128-key tile u and the query tiles of its group.
struct BwdItem {
    int h;
    long long u;    // key/value tile
    long long q0;   // first candidate query tile
    int nq;         // candidate query tiles (<= 32)
    bool paired;    // small windows: the only query tile is u
    uint32_t act;   // bit n: query tile q0 + n attends to u
    bool masked;    // some pairs of the group do not attend (the shift-region mask, or several windows per tile)
    Win win;        // the window (>= 256 tokens) or the first window of tile u
};

__host__ __device__ inline long long bwd_item_count(const Geo& g) {
    if (g.N >= 2 * kTile) return g.wins * g.heads * g.tpw;
    return g.tiles * g.heads;
}

__host__ __device__ inline BwdItem bwd_item(const Geo& g, long long it) {
    BwdItem I;
    if (g.N >= 2 * kTile) {
        // windows of >= 256 tokens: tiles per head = windows x tiles per window
        I.h = static_cast<int>(fdiv(g.fd_tiles, static_cast<uint32_t>(it)));
        const long long rem = it - static_cast<long long>(I.h) * g.tiles;
        const long long gw = rem >> g.ltpw;
        I.q0 = gw * g.tpw;
        I.u = I.q0 + (rem - gw * g.tpw);
        I.nq = g.tpw;
        I.paired = false;
        I.win = win_of(g, gw);
        I.act = low_bits(g.tpw);
        I.masked = g.s && (I.win.wr == g.Hp / g.M - 1 || I.win.wc == g.nWw - 1);
        if (I.masked) {
            const uint64_t su = tile_segs(g, I.u, I.win);
            I.act = 0;
            for (int n = 0; n < g.tpw; ++n)
                if (segs_meet(g, tile_segs(g, I.q0 + n, I.win), su)) I.act |= 1u << n;
        }
    } else {
        I.h = static_cast<int>(fdiv(g.fd_tiles, static_cast<uint32_t>(it)));
        const long long T = it - static_cast<long long>(I.h) * g.tiles;
        I.u = T;
        I.q0 = T;
        I.nq = 1;
        I.paired = true;
        I.win = tile_win(g, T);
        I.act = 1u;
        I.masked = true;
    }
    return I;
}

__host__ __device__ inline bool bwd_active(const Geo&, const BwdItem& I, int n) { return (I.act >> n) & 1u; }

}  // namespace fswin
