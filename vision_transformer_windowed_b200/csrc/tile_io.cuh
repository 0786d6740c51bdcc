// TMA traffic of whole 128-token tiles: one tiled copy per geometry box.
#pragma once

#include <cuda.h>

#include "geometry.cuh"
#include "ptx.cuh"

namespace fswin {

// TMA loads (or, when `store`, stores of the boxes of real windows) of every
// box of a tile; the smem tile holds the boxes back to back, 64-byte swizzled.
// The tensor maps span the H x W tokens in memory: a load reads zeros at the
// padded positions of a box, a store leaves them out, and boxes wholly in the
// padding are not stored at all.
static __device__ __noinline__ void tile_tma(const Geo& g, const CUtensorMap* map, uint8_t* smem_tile, uint64_t* bar,
                                      long long tile, int h, bool store) {
    Win w = tile_win(g, tile);
    for (int x = 0; x < g.bpt; ++x) {
        long long gw;
        int k;
        tile_box(g, tile, x, &gw, &k);
        if (gw != w.gw) w = win_of(g, gw);
        int r0, c0;
        box_origin(g, w, k, &r0, &c0);
        uint8_t* p = smem_tile + x * g.BT * kRowBytes;
        if (!store)
            tma_load_5d(p, map, bar, 0, h, c0, r0, w.b);
        else if (w.valid && r0 < g.H && c0 < g.W)
            tma_store_5d(map, p, 0, h, c0, r0, w.b);
    }
}

}  // namespace fswin
