// Out-of-line device versions of the geometry and scheduling helpers.
//
// The helpers do integer division once per window or work item; inlined at
// every call site of a warp-specialised kernel they would multiply its code
// size far beyond the instruction cache.  The kernels call these wrappers
// (the geometry lives in a __grid_constant__ kernel parameter, so it is passed
// by reference without a copy).
#pragma once

#include "geometry.cuh"
#include "schedule.cuh"

namespace fswin {

static __device__ __noinline__ FwdItem d_fwd_item(const Geo& g, long long it) { return fwd_item(g, it); }
static __device__ __noinline__ BwdItem d_bwd_item(const Geo& g, long long it) { return bwd_item(g, it); }
static __device__ __noinline__ Win d_tile_win(const Geo& g, long long tile) { return tile_win(g, tile); }
static __device__ __noinline__ uint64_t d_tile_segs(const Geo& g, long long tile, const Win& w) {
    return tile_segs(g, tile, w);
}
static __device__ __noinline__ uint32_t d_allow16(const Geo& g, uint32_t my, long long tile, const Win& w) {
    return allow16(g, my, tile_segs(g, tile, w));
}

}  // namespace fswin
