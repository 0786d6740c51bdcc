// Work items of the forward and backward kernels (host/device, so the
// scheduling can be checked on the CPU).
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
    long long kv0;  // first key/value tile of the list
    int nkv;        // length of the key/value list
    bool paired;    // small windows: entry u of the list serves query tile u only
};

__host__ __device__ inline long long fwd_item_count(const Geo& g) {
    if (g.N >= 2 * kTile) return g.wins * g.heads * (g.tpw / 2);
    return ((g.tiles + 1) / 2) * g.heads;
}

__host__ __device__ inline FwdItem fwd_item(const Geo& g, long long it) {
    FwdItem I;
    if (g.N >= 2 * kTile) {
        const int pairs = g.tpw / 2;
        const long long per_win = static_cast<long long>(g.heads) * pairs;
        const long long gw = it / per_win;
        const int rem = static_cast<int>(it - gw * per_win);
        I.h = rem / pairs;
        const int pr = rem - I.h * pairs;
        I.kv0 = gw * g.tpw;
        I.tA = I.kv0 + 2 * pr;
        I.tB = I.tA + 1;
        I.nkv = g.tpw;
        I.paired = false;
    } else {
        const long long x = it / g.heads;
        I.h = static_cast<int>(it - x * g.heads);
        I.tA = 2 * x;
        I.tB = 2 * x + 1 < g.tiles ? 2 * x + 1 : -1;
        I.kv0 = I.tA;
        I.nkv = I.tB >= 0 ? 2 : 1;
        I.paired = true;
    }
    return I;
}

// Is key/value list entry u used by query tile T (0 = A, 1 = B)?
__host__ __device__ inline bool fwd_active(const Geo& g, const FwdItem& I, int T, int u) {
    if (T == 1 && I.tB < 0) return false;
    if (I.paired) return u == T;
    if (g.s == 0) return true;
    const long long qt = T ? I.tB : I.tA;
    return (tile_labels(g, qt) & tile_labels(g, I.kv0 + u)) != 0;
}

// Backward: one 128-key tile u and the query tiles of its group.
struct BwdItem {
    int h;
    long long u;   // key/value tile
    long long q0;  // first candidate query tile
    int nq;        // candidate query tiles
    bool paired;   // small windows: the only query tile is u
};

__host__ __device__ inline long long bwd_item_count(const Geo& g) {
    if (g.N >= 2 * kTile) return g.wins * g.heads * g.tpw;
    return g.tiles * g.heads;
}

__host__ __device__ inline BwdItem bwd_item(const Geo& g, long long it) {
    BwdItem I;
    if (g.N >= 2 * kTile) {
        const long long per_win = static_cast<long long>(g.heads) * g.tpw;
        const long long gw = it / per_win;
        const int rem = static_cast<int>(it - gw * per_win);
        I.h = rem / g.tpw;
        I.q0 = gw * g.tpw;
        I.u = I.q0 + (rem - I.h * g.tpw);
        I.nq = g.tpw;
        I.paired = false;
    } else {
        const long long T = it / g.heads;
        I.h = static_cast<int>(it - T * g.heads);
        I.u = T;
        I.q0 = T;
        I.nq = 1;
        I.paired = true;
    }
    return I;
}

__host__ __device__ inline bool bwd_active(const Geo& g, const BwdItem& I, int n) {
    if (I.paired || g.s == 0) return true;
    return (tile_labels(g, I.q0 + n) & tile_labels(g, I.u)) != 0;
}

}  // namespace fswin
