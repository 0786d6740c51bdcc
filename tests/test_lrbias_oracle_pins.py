"""Pins of the oracle's low-rank additive bias against facts outside the oracle.

The bias is the FlashBias-T variant of the pages (thelatestinai.com/papers/
2610.04664, Table 2 and Table S1 captions: a trainable rank-16 factorization
of an additive attention bias).  Reading: per head, U W^T over window-local
positions t = i*M + j, shared by every window, added to the scaled scores
before the shift mask.  Each pin below fails for a plausible slip: a bias
added after the mask or before the 1/sqrt(d) scale, U and W swapped, a
transposed position index, a gradient not summed over windows.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import oracle.literal as lit
from vision_transformer_windowed_b200.inputs import make_bias, make_inputs


def _rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-300))


SHAPES = [  # (B, H, W, heads, d, M, s, rank)
    (2, 8, 8, 2, 8, 4, 2, 16),
    (1, 8, 12, 2, 16, 4, 0, 4),
    (1, 16, 16, 2, 32, 8, 4, 16),
    (1, 10, 7, 1, 32, 4, 2, 16),    # padded grid
    (1, 8, 8, 1, 8, 2, 1, 3),
]


@pytest.mark.parametrize("shape", SHAPES)
def test_c_oracle_matches_tensor_level_restatement_with_bias(shape):
    """C loops vs the torch restatement (bias as U @ W^T broadcast, autograd)."""
    B, H, W, h, d, M, s, rank = shape
    inp = make_inputs(B, H, W, h, d)
    bias = make_bias(h, M, rank)
    r = oracle.full(inp["q"], inp["k"], inp["v"], inp["theta"], M, s, dout=inp["dout"],
                    bias=(bias["u"], bias["w"]))
    f = {k: v.to(torch.float64) for k, v in inp.items()}
    ref = lit.forward_backward(f["q"], f["k"], f["v"], f["theta"], M, s, f["dout"],
                               bias=(bias["u"].double(), bias["w"].double()))
    for key in ("o", "lse", "dq", "dk", "dv", "dtheta", "du", "dw"):
        assert _rel(r[key], ref[key].numpy()) < 1e-12, key


def test_full_rank_bias_is_sdpa_with_an_additive_mask():
    """rank = N with U = I and W = B^T makes U W^T = B, any N x N bias matrix:
    with theta = 0 and s = 0 every window is torch's scaled_dot_product_attention
    with the float attn_mask B (added to the scaled scores by that routine)."""
    B_, H, W, h, d, M = 2, 8, 8, 2, 16, 4
    N = M * M
    inp = make_inputs(B_, H, W, h, d)
    g = torch.Generator().manual_seed(5)
    bmat = torch.randn(h, N, N, generator=g, dtype=torch.float64) * 2.0
    u = torch.eye(N, dtype=torch.float64).expand(h, N, N).contiguous()
    w = bmat.transpose(1, 2).contiguous()
    zero = torch.zeros_like(inp["theta"])
    r = oracle.full(inp["q"], inp["k"], inp["v"], zero, M, 0, bias=(u, w))
    q, k, v = (inp[x].double() for x in ("q", "k", "v"))
    for b in range(B_):
        for wr in range(H // M):
            for wc in range(W // M):
                sl = (b, slice(wr * M, wr * M + M), slice(wc * M, wc * M + M))
                qq, kk, vv = (t[sl].reshape(N, h, d).transpose(0, 1) for t in (q, k, v))
                ref = F.scaled_dot_product_attention(qq, kk, vv, attn_mask=bmat)
                ref = ref.transpose(0, 1).reshape(M, M, h, d)
                assert _rel(r["o"][sl], ref.numpy()) < 1e-12


def test_row_constant_bias_leaves_o_and_shifts_lse():
    """A bias constant along the keys (W_u = e_0 for every u) adds U_t[0] to every
    score of row t: O is unchanged (softmax is shift invariant), LSE grows by
    U_t[0], and the row's gradient sum dU_t[0] = sum_u dS_tu vanishes."""
    B_, H, W, h, d, M, s = 1, 8, 8, 2, 8, 4, 2
    N, rank = M * M, 4
    inp = make_inputs(B_, H, W, h, d)
    g = torch.Generator().manual_seed(9)
    u = torch.randn(h, N, rank, generator=g, dtype=torch.float64) * 3.0
    w = torch.zeros(h, N, rank, dtype=torch.float64)
    w[:, :, 0] = 1.0
    r0 = oracle.full(inp["q"], inp["k"], inp["v"], inp["theta"], M, s, dout=inp["dout"])
    r = oracle.full(inp["q"], inp["k"], inp["v"], inp["theta"], M, s, dout=inp["dout"], bias=(u, w))
    assert _rel(r["o"], r0["o"]) < 1e-13
    for key in ("dq", "dk", "dv", "dtheta"):
        assert _rel(r[key], r0[key]) < 1e-12, key
    # lse at original positions: rolled token (rr, cc) sits at ((rr+s)%H, (cc+s)%W),
    # window-local position t = (rr % M) * M + cc % M
    for rr in range(H):
        for cc in range(W):
            t = (rr % M) * M + cc % M
            ro, co = (rr + s) % H, (cc + s) % W
            assert np.allclose(r["lse"][0, ro, co] - r0["lse"][0, ro, co], u[:, t, 0].numpy(), rtol=0, atol=1e-12)
    assert np.abs(r["du"][:, :, 0]).max() < 1e-12 * max(1.0, np.abs(r["du"]).max())


def test_bias_gradients_are_sums_over_windows():
    """The full-tensor du, dw equal the sum of the per-unit shares of every
    (image, window) unit of the head (the units API), and differ from any single
    window's share."""
    B_, H, W, h, d, M, s = 2, 8, 8, 2, 8, 4, 2
    inp = make_inputs(B_, H, W, h, d)
    bias = make_bias(h, M, 16)
    bt = (bias["u"], bias["w"])
    r = oracle.full(inp["q"], inp["k"], inp["v"], inp["theta"], M, s, dout=inp["dout"], bias=bt)
    nW = (H // M) * (W // M)
    ids = list(range(B_ * nW * h))
    per = oracle.units(inp["q"], inp["k"], inp["v"], inp["theta"], M, s, ids, dout=inp["dout"], bias=bt)
    for hh in range(h):
        mine = [n for n in ids if n % h == hh]
        assert _rel(r["du"][hh], per["du"][mine].sum(0)) < 1e-13
        assert _rel(r["dw"][hh], per["dw"][mine].sum(0)) < 1e-13
        assert _rel(r["du"][hh], per["du"][mine[0]]) > 1e-3


@pytest.mark.parametrize("s", [0, 2])
def test_finite_difference_bias_gradients(s):
    """Central differences of L = sum(O * dO) w.r.t. U and W (rel. err <= 1e-6)."""
    B_, H, W, h, d, M, rank = 1, 8, 8, 2, 8, 4, 16
    inp = {k: v.to(torch.float64) for k, v in make_inputs(B_, H, W, h, d).items()}
    bias = {k: v.double().numpy() for k, v in make_bias(h, M, rank).items()}
    r = oracle.full(inp["q"], inp["k"], inp["v"], inp["theta"], M, s, dout=inp["dout"],
                    bias=(bias["u"], bias["w"]))
    do = inp["dout"].numpy()

    def loss(u, w):
        o = oracle.full(inp["q"], inp["k"], inp["v"], inp["theta"], M, s, bias=(u, w))["o"]
        return float((o * do).sum())

    eps = 1e-5
    rng = np.random.default_rng(1)
    for name, grad in (("u", "du"), ("w", "dw")):
        base = bias[name]
        for fid in rng.choice(base.size, size=12, replace=False):
            idx = np.unravel_index(fid, base.shape)
            plus, minus = base.copy(), base.copy()
            plus[idx] += eps
            minus[idx] -= eps
            args_p = (plus, bias["w"]) if name == "u" else (bias["u"], plus)
            args_m = (minus, bias["w"]) if name == "u" else (bias["u"], minus)
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            an = r[grad][idx]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, idx, fd, an)


def test_bias_never_unmasks_a_shift_region_pair():
    """The shift mask wins over any bias: a huge bias toward one key per row
    changes nothing for queries whose window does not hold that key's region, and
    each masked pair keeps probability zero (checked by o staying a convex
    combination of the query's own region's v rows: v = region indicator)."""
    B_, H, W, h, d, M, s = 1, 8, 8, 1, 8, 4, 2
    N = M * M
    inp = make_inputs(B_, H, W, h, d)
    lab = oracle.labels(H, W, M, s)  # rolled frame
    # v = one-hot of the token's region label (9 labels, d = 8 channels: label 8 -> zeros)
    v = torch.zeros(B_, H, W, h, d, dtype=torch.float64)
    for rr in range(H):
        for cc in range(W):
            L = lab[rr, cc]
            if L < d:
                v[0, (rr + s) % H, (cc + s) % W, 0, L] = 1.0
    u = torch.zeros(h, N, 1, dtype=torch.float64)
    w = torch.zeros(h, N, 1, dtype=torch.float64)
    u[:, :, 0] = 40.0
    w[:, 0, 0] = 1.0  # every query strongly prefers window position 0
    r = oracle.full(inp["q"], inp["k"], v, inp["theta"], M, s, bias=(u, w))
    for rr in range(H):
        for cc in range(W):
            L = lab[rr, cc]
            o = r["o"][0, (rr + s) % H, (cc + s) % W, 0]
            expect = np.zeros(d)
            if L < d:
                expect[L] = 1.0
            assert np.allclose(o, expect, rtol=0, atol=1e-12), (rr, cc, o)


def test_units_api_matches_full_with_bias():
    B_, H, W, h, d, M, s = 2, 8, 8, 2, 8, 4, 2
    inp = make_inputs(B_, H, W, h, d)
    bias = make_bias(h, M, 16)
    bt = (bias["u"], bias["w"])
    r = oracle.full(inp["q"], inp["k"], inp["v"], inp["theta"], M, s, dout=inp["dout"], bias=bt)
    u = oracle.units(inp["q"], inp["k"], inp["v"], inp["theta"], M, s, [0, 5, 13], dout=inp["dout"], bias=bt)
    for i, n in enumerate([0, 5, 13]):
        b, rows, cols, hh = oracle.unit_token_positions(H, W, M, s, n, h)
        assert _rel(u["o"][i], r["o"][b, rows, cols, hh]) < 1e-13
        assert _rel(u["dq"][i], r["dq"][b, rows, cols, hh]) < 1e-13
