"""Pins of the oracle on grids whose H or W is not a multiple of the window.

A Swin layer pads such a grid at the bottom and right with zero tokens up to
the next multiple of M, shifts and masks on the padded grid, and crops the
result (Swin Transformer, the shifted-window block; the FlashSwin pages use
the Swin layer unchanged around the attention, thelatestinai.com/papers/
2610.04664, Figure 1B).  Each test below fixes that reading from outside the
C oracle: an independent tensor-level restatement, a closed form, the
unpadded oracle on explicitly padded inputs, and finite differences.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import oracle.block as ob
import oracle.literal as lit
from vision_transformer_windowed_b200.inputs import make_inputs


def _rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-300))


def _pad(t, Hp, Wp):
    B, H, W = t.shape[:3]
    out = torch.zeros((B, Hp, Wp) + tuple(t.shape[3:]), dtype=t.dtype)
    out[:, :H, :W] = t
    return out


PADDED = [  # (B, H, W, heads, d, M, s)
    (1, 6, 10, 2, 8, 4, 2),
    (2, 5, 7, 1, 8, 2, 1),
    (1, 10, 9, 2, 16, 4, 0),
    (1, 13, 11, 1, 32, 8, 4),
    (1, 9, 12, 2, 8, 3, 1),
]


@pytest.mark.parametrize("shape", PADDED)
def test_padded_matches_tensor_level_restatement(shape):
    """C loops vs F.pad + torch.roll + reshape + autograd (independent code)."""
    B, H, W, h, d, M, s = shape
    inp = make_inputs(B, H, W, h, d)
    r = oracle.full(inp["q"], inp["k"], inp["v"], inp["theta"], M, s, dout=inp["dout"])
    f = {k: v.to(torch.float64) for k, v in inp.items()}
    ref = lit.forward_backward(f["q"], f["k"], f["v"], f["theta"], M, s, f["dout"])
    for key in ("o", "lse", "dq", "dk", "dv", "dtheta"):
        assert r[key].shape == tuple(ref[key].shape), key
        assert _rel(r[key], ref[key].numpy()) < 1e-12, key


@pytest.mark.parametrize("shape", PADDED)
def test_padded_equals_unpadded_oracle_on_zero_padded_grid(shape):
    """Padding inside the oracle == the multiple-of-M oracle (pinned elsewhere)
    run on inputs padded with zeros by hand, cropped; gradients included."""
    B, H, W, h, d, M, s = shape
    Hp, Wp = -(-H // M) * M, -(-W // M) * M
    inp = make_inputs(B, H, W, h, d)
    r = oracle.full(inp["q"], inp["k"], inp["v"], inp["theta"], M, s, dout=inp["dout"])
    pq, pk, pv, pdo = (_pad(inp[x].double(), Hp, Wp) for x in ("q", "k", "v", "dout"))
    rp = oracle.full(pq, pk, pv, inp["theta"], M, s, dout=pdo)
    for key in ("o", "lse", "dq", "dk", "dv"):
        assert np.array_equal(r[key], rp[key][:, :H, :W]), key
    assert _rel(r["dtheta"], rp["dtheta"]) < 1e-13


@pytest.mark.parametrize("s", [0, 2])
def test_padded_tokens_count_in_the_softmax(s):
    """q = k = 0: every allowed score is 0, so a token averages v over the
    tokens of its window with its label, padded ones (v = 0) included:
    o = (sum of real v) / n and lse = ln n, n counted on the padded grid."""
    B, H, W, h, d, M = 1, 6, 7, 1, 8, 4
    Hp, Wp = 8, 8
    inp = make_inputs(B, H, W, h, d)
    zero = torch.zeros_like(inp["q"], dtype=torch.float64)
    v = inp["v"].double().numpy()
    r = oracle.full(zero, zero, inp["v"], inp["theta"], M, s)
    lab = oracle.labels(Hp, Wp, M, s)
    for rr in range(Hp):
        for cc in range(Wp):
            ro, co = (rr + s) % Hp, (cc + s) % Wp
            if ro >= H or co >= W:
                continue
            n, acc = 0, np.zeros(d)
            for r2 in range(rr // M * M, rr // M * M + M):
                for c2 in range(cc // M * M, cc // M * M + M):
                    if lab[r2, c2] != lab[rr, cc]:
                        continue
                    n += 1
                    o2, p2 = (r2 + s) % Hp, (c2 + s) % Wp
                    if o2 < H and p2 < W:
                        acc += v[0, o2, p2, 0]
            assert abs(r["lse"][0, ro, co, 0] - math.log(n)) < 1e-13
            assert np.allclose(r["o"][0, ro, co, 0], acc / n, rtol=0, atol=1e-13)


def test_padded_finite_difference_gradients():
    """Central differences of L = sum(O * dO) on a padded, shifted grid."""
    B, H, W, h, d, M, s = 1, 6, 5, 2, 8, 4, 2
    inp = {k: v.to(torch.float64) for k, v in make_inputs(B, H, W, h, d).items()}
    inp["theta"] = inp["theta"] * 3.0
    r = oracle.full(inp["q"], inp["k"], inp["v"], inp["theta"], M, s, dout=inp["dout"])
    do = inp["dout"].numpy()

    def loss(**kw):
        args = {x: inp[x] for x in ("q", "k", "v", "theta")}
        args.update(kw)
        return float((oracle.full(args["q"], args["k"], args["v"], args["theta"], M, s)["o"] * do).sum())

    eps = 1e-5
    rng = np.random.default_rng(1)
    for name, grad in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("theta", "dtheta")):
        base = inp[name].numpy()
        for fid in rng.choice(base.size, size=min(base.size, 12), replace=False):
            idx = np.unravel_index(fid, base.shape)
            plus, minus = base.copy(), base.copy()
            plus[idx] += eps
            minus[idx] -= eps
            fd = (loss(**{name: plus}) - loss(**{name: minus})) / (2 * eps)
            assert abs(fd - r[grad][idx]) <= 1e-6 * max(1.0, abs(r[grad][idx])), (name, idx)


def test_padded_units_match_full():
    B, H, W, h, d, M, s = 1, 10, 6, 2, 8, 4, 2
    inp = make_inputs(B, H, W, h, d)
    r = oracle.full(inp["q"], inp["k"], inp["v"], inp["theta"], M, s, dout=inp["dout"])
    nunits = B * 3 * 2 * h
    u = oracle.units(inp["q"], inp["k"], inp["v"], inp["theta"], M, s, list(range(nunits)), dout=inp["dout"])
    dth = np.zeros_like(r["dtheta"])
    seen = 0
    for uid in range(nunits):
        b, rows, cols, hh = oracle.unit_token_positions(H, W, M, s, uid, h)
        real = (rows < H) & (cols < W)
        seen += int(real.sum())
        for key in ("o", "dq", "dk", "dv"):
            assert np.array_equal(u[key][uid][real], r[key][b, rows[real], cols[real], hh])
        dth[hh] += u["dtheta"][uid]
    assert seen == B * H * W * h
    assert _rel(dth, r["dtheta"]) < 1e-13


def test_block_pads_x_before_the_projection():
    """W_qkv = 0: q = k = 0 and v = b_v at every token, padded ones included
    (a Swin layer pads x, not q, k, v), so o = b_v and y = b_v W_o^T + b_o
    everywhere; padding q, k, v with zeros instead would give |o| < |b_v| at
    tokens whose window holds padding."""
    B, H, W, heads, d, M, s = 1, 6, 7, 2, 8, 4, 2
    C = heads * d
    g = torch.Generator().manual_seed(3)
    x = torch.randn(B, H, W, C, generator=g, dtype=torch.float64)
    w_qkv = torch.zeros(3 * C, C, dtype=torch.float64)
    b_qkv = torch.randn(3 * C, generator=g, dtype=torch.float64)
    w_o = torch.randn(C, C, generator=g, dtype=torch.float64)
    b_o = torch.randn(C, generator=g, dtype=torch.float64)
    theta = torch.rand(heads, 2, d // 4, generator=g, dtype=torch.float64)
    y, o = ob.block_forward(x, w_qkv, b_qkv, w_o, b_o, theta, M, s, heads)
    bv = b_qkv[2 * C:].numpy()
    assert np.abs(o.reshape(B, H, W, C) - bv).max() < 1e-13
    assert np.abs(y - (bv @ w_o.numpy().T + b_o.numpy())).max() < 1e-12
