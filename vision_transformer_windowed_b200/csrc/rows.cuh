// Per-row helpers shared by the kernels: 64-byte-swizzled 16-bit token rows in
// shared memory (the layout a TMA SWIZZLE_64B copy produces), packing, the
// compact RoPE table of windows of at most 8 x 8 tokens, and the grid token of
// a tile slot.
#pragma once

#include <cuda_fp16.h>
#include <cstring>
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

// Squared norm of row r of a 16-bit bf16 tile (the swizzle only permutes the
// row's 16-byte chunks, which leaves the norm unchanged).
__device__ __forceinline__ float row_norm2(const uint8_t* tile, int r) {
    const uint4* row = reinterpret_cast<const uint4*>(tile + r * kRowBytes);
    float n[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint4 v = row[c];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; e += 2) {
            const float a0 = bf16lo_to_f32(w[e]), a1 = bf16hi_to_f32(w[e]);
            const float b0 = bf16lo_to_f32(w[e + 1]), b1 = bf16hi_to_f32(w[e + 1]);
            ffma2(n[0], n[1], a0, a1, a0, a1, n[0], n[1]);
            ffma2(n[2], n[3], b0, b1, b0, b1, n[2], n[3]);
        }
    }
    return (n[0] + n[1]) + (n[2] + n[3]);
}

// Power-of-two scaling of the gradient products.  dS = P o (dP - D) is rounded
// to fp16 for the dQ' and dK' products; unscaled, the tiny upstream gradients
// of bf16 training (1e-9 .. 1e-5, no loss scaling) would leave it in fp16's
// subnormal range or flush it to zero, and large ones would overflow.  The
// backward therefore works with P' = 2^e P = exp2(S c - (lse2 - e)): then
// dS' = P' o (dP - D) = 2^e dS and dV' = P'^T dO = 2^e dV, with no extra
// arithmetic per score (only lse2 is shifted), and the fp32 epilogue multiplies
// dQ', dK' and dV by 2^-e.  G = 4 max|dO_t| max|v_u| over the rows a product
// reaches bounds |dP_tu - D_t| (|dO_t . v_u| <= |dO_t| |v_u|, and O_t is a
// convex combination of v rows, so |D_t| <= |dO_t| max|v_u|; the factor 4
// leaves room for O's rounding), and e with G 2^e <= 2^14 keeps every scaled dS
// below fp16's largest value 65504 while values 2^28 times below G are still
// normal.  P' = 2^e P <= 2^e stays inside bf16's range (that of fp32).  The
// scaling is exact (a power of two).
//
// e from the largest squared norms a = max|dO_t|^2, b = max|v_u|^2 (integer
// arithmetic on the exponent fields; no square root, no overflow):
// a < 2^(Ea+1), b < 2^(Eb+1) give G^2 = 16 a b < 2^(Ea+Eb+6), so
// G < 2^ceil((Ea+Eb+6)/2), and e = 14 - ceil((Ea+Eb+6)/2).
__host__ __device__ inline int grad_scale_exp(float max_do2, float max_v2) {
#ifdef __CUDA_ARCH__
    const uint32_t ua = __float_as_uint(max_do2), ub = __float_as_uint(max_v2);
#else
    uint32_t ua, ub;
    memcpy(&ua, &max_do2, 4);
    memcpy(&ub, &max_v2, 4);
#endif
    const int ea = static_cast<int>((ua >> 23) & 0xFFu) - 127, eb = static_cast<int>((ub >> 23) & 0xFFu) - 127;
    const int sum = ea + eb + 6;
    const int up = sum >= 0 ? (sum + 1) / 2 : -((-sum) / 2);  // ceil(sum / 2)
    int e = 14 - up;
    return e < -125 ? -125 : (e > 125 ? 125 : e);  // zero norms give e = 125: the products are zero then
}

// 2^e as a float, for -126 < e < 127.
__device__ __forceinline__ float exp2i(int e) { return __uint_as_float(static_cast<uint32_t>(e + 127) << 23); }

// The exponent of a tile from its row warps' largest |dO row|^2 and |v row|^2.
__device__ __forceinline__ int grad_scale_exp4(const float2 (&nrm)[4]) {
    float a = nrm[0].x, b = nrm[0].y;
#pragma unroll
    for (int w = 1; w < 4; ++w) {
        a = fmaxf(a, nrm[w].x);
        b = fmaxf(b, nrm[w].y);
    }
    return grad_scale_exp(a, b);
}

// Largest value over the warp of a non-negative float (its bits order like
// unsigned integers): one warp-wide unsigned max reduction.
__device__ __forceinline__ float warp_max_nonneg(float x) {
    return __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(x)));
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
