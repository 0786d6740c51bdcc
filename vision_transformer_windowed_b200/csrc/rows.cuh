// Per-row helpers shared by the kernels: 64-byte-swizzled 16-bit token rows in
// shared memory (the layout a TMA SWIZZLE_64B copy produces), packing, the
// compact RoPE table of windows of at most 8 x 8 tokens, and the grid token of
// a tile slot.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "geometry.cuh"
#include "ptx.cuh"

namespace fswin {

__device__ __forceinline__ uint32_t pack2(float lo, float hi, bool fp16) {
    return fp16 ? pack_f16x2(lo, hi) : pack_bf16x2(lo, hi);
}

__device__ __forceinline__ uint4 pack_chunk(const float (&x)[32], int c, bool fp16 = false) {
    return make_uint4(pack2(x[8 * c], x[8 * c + 1], fp16), pack2(x[8 * c + 2], x[8 * c + 3], fp16),
                      pack2(x[8 * c + 4], x[8 * c + 5], fp16), pack2(x[8 * c + 6], x[8 * c + 7], fp16));
}

// Row r of a 64-byte-swizzled 16-bit tile image (bf16, or fp16 for the
// rotated Q' and K', see the forward kernel).
__device__ __forceinline__ void store_row_swz(uint8_t* tile, int r, const float (&x)[32], bool fp16 = false) {
    uint8_t* row = tile + r * kRowBytes;
    const int sw = (r >> 1) & 3;
#pragma unroll
    for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4*>(row + ((c ^ sw) << 4)) = pack_chunk(x, c, fp16);
}

// Row r of a 64-byte-swizzled 16-bit tile (bf16, or fp16) as 32 floats.
__device__ __forceinline__ void load_row_swz(const uint8_t* tile, int r, float (&x)[32], bool fp16) {
    const uint8_t* row = tile + r * kRowBytes;
    const int sw = (r >> 1) & 3;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint4 v = *reinterpret_cast<const uint4*>(row + ((c ^ sw) << 4));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (fp16) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[e]));
                x[8 * c + 2 * e] = f.x;
                x[8 * c + 2 * e + 1] = f.y;
            } else {
                x[8 * c + 2 * e] = bf16lo_to_f32(w[e]);
                x[8 * c + 2 * e + 1] = bf16hi_to_f32(w[e]);
            }
        }
    }
}

// Rotation by the compact table of one head ([axis][pair][position], M <= 8).
__device__ __forceinline__ void rope32_small(float (&x)[32], int i, int j, const float2* tab, bool inv) {
#pragma unroll
    for (int ax = 0; ax < 2; ++ax) {
        const int pos = ax ? i : j;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const float2 cs = tab[(ax * 8 + k) * 8 + pos];
            const float sn = inv ? -cs.y : cs.y;
            const float a = x[ax * 16 + 2 * k], b = x[ax * 16 + 2 * k + 1];
            float t0, t1;
            fmul2(t0, t1, a, b, cs.x, cs.x);  // (a cos, b cos), then + (-b sin, a sin)
            ffma2(x[ax * 16 + 2 * k], x[ax * 16 + 2 * k + 1], -b, a, sn, sn, t0, t1);
        }
    }
}

__device__ __forceinline__ void build_small_table(float2* tab, const float* theta_h, int M, int tid, int nthreads) {
    for (int e = tid; e < 16 * M; e += nthreads) {
        const int ap = e / M, pos = e - ap * M;  // ap = axis * 8 + pair
        float sn, cs;
        sincosf(static_cast<float>(pos) * theta_h[ap], &sn, &cs);
        tab[ap * 8 + pos] = make_float2(cs, sn);
    }
}

// Token of slot r of tile X: in-window position and flat index of the
// [B, H, W, heads] tokens at head h.  False (and *tok meaningless) for the
// slots of padding windows and for padded positions of the grid.
__device__ __forceinline__ bool slot_token(const Geo& g, long long X, int r, int h, int* pi, int* pj,
                                           long long* tok) {
    Win w = tile_win(g, X);
    const int widx = r >> (g.lnbw + g.lBT);  // window of the slot inside the tile
    if (widx) w = win_of(g, w.gw + widx);
    tile_row_pos(g, X, r, pi, pj);
    int row = w.wr * g.M + *pi + g.s, col = w.wc * g.M + *pj + g.s;
    if (row >= g.Hp) row -= g.Hp;
    if (col >= g.Wp) col -= g.Wp;
    *tok = ((static_cast<long long>(w.b) * g.H + row) * g.W + col) * g.heads + h;
    return w.valid && row < g.H && col < g.W;
}

}  // namespace fswin
