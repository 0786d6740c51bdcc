"""Seeded synthetic inputs shared by the CUDA path's tests, the oracle tests and
the benchmark.  This module holds no arithmetic of the method itself: it only
draws tensors.

Recipe (the Swin-shaped synthetic workloads of the FlashSwin evaluation,
thelatestinai.com/papers/2610.04664, Table S1 and Figure S1 shapes):
  * Q, K, V, dO: bf16 draws of N(0, 1) on a [B, H, W, heads, d] grid from
    torch generators seeded 0, 1, 2, 3; optionally Q and K scaled by a constant
    (the high-resolution stress case sharpens the softmax with a factor 3);
  * theta: fp32 [heads, 2, d/4], the geometric RoPE schedule
    100 ** (-2 i / (d / 2)), i = 0 .. d/4 - 1, repeated for both axes and every
    head (the initialisation the pages call "the standard geometric RoPE
    schedule", Figure S4), plus N(0, 0.01) noise from a generator seeded 4.

For the attention block with its projections (Figure 1B): x bf16 N(0, 1) on a
[B, H, W, C] grid (seed 5), C = heads * d; W_qkv [3C, C] and W_o [C, C] bf16
N(0, 1/C), the variance of a linear layer's initialisation, so that q, k, v
are near N(0, 1) like the attention workloads' (seeds 6 and 8); b_qkv and b_o
fp32 N(0, 0.02^2) (seeds 7 and 9); theta as above.

For the low-rank additive bias (the FlashBias-T variant, Table 2 and Table S1:
a trainable rank-16 bias factorization): factors U, W fp32 [heads, M*M, rank]
drawn N(0, 0.5^2) (seeds 10 and 11), so that every bias entry U_t.W_u of rank
16 has unit variance, the spread of the scores themselves.
"""
from __future__ import annotations

import torch

SEED_Q, SEED_K, SEED_V, SEED_DO, SEED_THETA = 0, 1, 2, 3, 4
SEED_X, SEED_WQKV, SEED_BQKV, SEED_WO, SEED_BO = 5, 6, 7, 8, 9
SEED_U, SEED_W = 10, 11


def _normal(shape, seed: int, device, scale: float = 1.0) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if scale != 1.0:
        x.mul_(scale)
    return x.to(torch.bfloat16)


def theta_init(heads: int, d: int, device="cpu", noise: float = 0.01, seed: int = SEED_THETA) -> torch.Tensor:
    q = d // 4
    i = torch.arange(q, dtype=torch.float64)
    base = (100.0 ** (-2.0 * i / (d / 2))).to(torch.float32)
    th = base.repeat(heads, 2, 1).contiguous()
    if noise:
        g = torch.Generator(device="cpu")
        g.manual_seed(seed)
        th = th + noise * torch.randn(th.shape, generator=g, dtype=torch.float32)
    return th.to(device)


def make_inputs(B: int, H: int, W: int, heads: int, d: int, device="cpu", qk_scale: float = 1.0,
                with_dout: bool = True, shard: int = 0) -> dict:
    """`shard` > 0 draws other images (seeds offset by 16 * shard) with the same
    theta: the per-process batch of a data-parallel run."""
    shape = (B, H, W, heads, d)
    off = 16 * shard
    out = {
        "q": _normal(shape, SEED_Q + off, device, qk_scale),
        "k": _normal(shape, SEED_K + off, device, qk_scale),
        "v": _normal(shape, SEED_V + off, device),
        "theta": theta_init(heads, d, device),
    }
    if with_dout:
        out["dout"] = _normal(shape, SEED_DO + off, device)
    return out


def make_block_inputs(B: int, H: int, W: int, heads: int, d: int, device="cpu") -> dict:
    """Inputs of the attention block: x, w_qkv, b_qkv, w_o, b_o, theta."""
    C = heads * d

    def draw(shape, seed, std, dtype):
        g = torch.Generator(device=device)
        g.manual_seed(seed)
        return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(dtype)

    return {
        "x": draw((B, H, W, C), SEED_X, 1.0, torch.bfloat16),
        "w_qkv": draw((3 * C, C), SEED_WQKV, C ** -0.5, torch.bfloat16),
        "b_qkv": draw((3 * C,), SEED_BQKV, 0.02, torch.float32),
        "w_o": draw((C, C), SEED_WO, C ** -0.5, torch.bfloat16),
        "b_o": draw((C,), SEED_BO, 0.02, torch.float32),
        "theta": theta_init(heads, d, device),
    }


def make_bias(heads: int, M: int, rank: int = 16, device="cpu", std: float = 0.5) -> dict:
    """Low-rank bias factors u, w: fp32 [heads, M*M, rank]."""

    def draw(seed):
        g = torch.Generator(device="cpu")
        g.manual_seed(seed)
        return (torch.randn((heads, M * M, rank), generator=g, dtype=torch.float32) * std).to(device)

    return {"u": draw(SEED_U), "w": draw(SEED_W)}
