"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

The pages print no worked example for the attention operator, so every pin is
a closed form, an invariant, a library routine it must reduce to, an
independent restatement, or finite differences.  Each is chosen so that a
plausible slip in the oracle (a dropped term, a wrong sign or index, a
transposed operand, a wrong axis or shift direction) fails at least one test.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import oracle.literal as lit
from vision_transformer_windowed_b200.inputs import make_inputs, theta_init

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-300))


def _f64(inp):
    return {k: v.to(torch.float64) for k, v in inp.items()}


SHAPES = [  # (B, H, W, heads, d, M, s)
    (2, 8, 8, 2, 8, 4, 2),
    (1, 4, 4, 1, 8, 2, 1),
    (1, 8, 12, 2, 16, 4, 3),
    (1, 6, 6, 1, 4, 3, 1),
    (1, 16, 16, 2, 32, 8, 4),
    (1, 16, 8, 3, 32, 8, 0),
    (1, 8, 8, 1, 64, 4, 2),      # 64-channel heads (16 RoPE pairs per axis)
    (1, 16, 16, 2, 64, 8, 4),
]


@pytest.mark.parametrize("shape", SHAPES)
def test_c_oracle_matches_tensor_level_restatement(shape):
    """C loops vs torch.roll / reshape / complex RoPE / autograd (independent code)."""
    B, H, W, h, d, M, s = shape
    inp = make_inputs(B, H, W, h, d)
    r = oracle.full(inp["q"], inp["k"], inp["v"], inp["theta"], M, s, dout=inp["dout"])
    f = _f64(inp)
    ref = lit.forward_backward(f["q"], f["k"], f["v"], f["theta"], M, s, f["dout"])
    for key in ("o", "lse", "dq", "dk", "dv", "dtheta"):
        assert _rel(r[key], ref[key].numpy()) < 1e-12, key


def test_labels_match_hand_enumeration():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "labels_H4_W4_M2_s1.txt")) if not l.startswith("#")]
    golden = np.array(rows, dtype=np.int32)
    assert (oracle.labels(4, 4, 2, 1) == golden).all()
    assert (lit.region_labels(4, 4, 2, 1).numpy() == golden).all()
    assert (oracle.labels(8, 8, 4, 0) == 0).all()


def test_self_only_window_closed_form():
    """Window (1,1) of the 4x4, M=2, s=1 grid has four distinct labels: each token
    attends only to itself, so o = v and lse = q.k / sqrt(d) whatever theta is
    (the rotation is orthogonal and both vectors sit at the same position)."""
    B, H, W, h, d, M, s = 1, 4, 4, 2, 8, 2, 1
    inp = make_inputs(B, H, W, h, d)
    inp["theta"] = inp["theta"] * 7.3  # large angles: the result must not depend on theta
    r = oracle.full(inp["q"], inp["k"], inp["v"], inp["theta"], M, s)
    q, k, v = (inp[x].double().numpy() for x in ("q", "k", "v"))
    for rr in (2, 3):
        for cc in (2, 3):
            ro, co = (rr + s) % H, (cc + s) % W
            assert np.allclose(r["o"][0, ro, co], v[0, ro, co], rtol=0, atol=1e-14)
            exp_lse = (q[0, ro, co] * k[0, ro, co]).sum(-1) / math.sqrt(d)
            assert np.allclose(r["lse"][0, ro, co], exp_lse, rtol=0, atol=1e-13)


def test_theta_zero_is_plain_windowed_attention():
    """theta = 0: windowed softmax attention, checked window by window against
    torch's scaled_dot_product_attention (a library routine)."""
    B, H, W, h, d, M = 2, 8, 8, 2, 16, 4
    inp = make_inputs(B, H, W, h, d)
    zero = torch.zeros_like(inp["theta"])
    r = oracle.full(inp["q"], inp["k"], inp["v"], zero, M, 0)
    q, k, v = (inp[x].double() for x in ("q", "k", "v"))
    for b in range(B):
        for wr in range(H // M):
            for wc in range(W // M):
                sl = (b, slice(wr * M, wr * M + M), slice(wc * M, wc * M + M))
                qq, kk, vv = (t[sl].reshape(M * M, h, d).transpose(0, 1) for t in (q, k, v))
                ref = F.scaled_dot_product_attention(qq, kk, vv).transpose(0, 1).reshape(M, M, h, d)
                assert _rel(r["o"][sl], ref.numpy()) < 1e-12


def _rotate_complex(x, theta, pi, pj):
    """x [N, h, d]; rotate pairs by positions (pi rows, pj cols) as complex numbers."""
    N, h, d = x.shape
    out = x.clone()
    for ax, pos in ((0, pj), (1, pi)):
        half = x[..., ax * d // 2:(ax + 1) * d // 2].reshape(N, h, d // 4, 2)
        z = torch.complex(half[..., 0], half[..., 1])
        ang = pos[:, None, None] * theta[None, :, ax, :]
        z = z * torch.exp(1j * ang)
        out[..., ax * d // 2:(ax + 1) * d // 2] = torch.stack([z.real, z.imag], -1).reshape(N, h, d // 2)
    return out


@pytest.mark.parametrize("offset", [(0, 0), (3, -5), (11, 2)])
def test_single_window_is_global_rope_attention(offset):
    """H = W = M, s = 0: global attention over the grid with 2D RoPE at positions
    (row, col) + any constant offset (RoPE scores depend only on relative
    offsets), via torch's scaled_dot_product_attention."""
    B, H, W, h, d, M = 1, 6, 6, 2, 16, 6
    inp = make_inputs(B, H, W, h, d)
    th = inp["theta"].double() * 3.0
    r = oracle.full(inp["q"], inp["k"], inp["v"], th, M, 0)
    t = torch.arange(M * M, dtype=torch.float64)
    pi, pj = t // M + offset[0], t % M + offset[1]
    q, k, v = (inp[x].double()[0].reshape(M * M, h, d) for x in ("q", "k", "v"))
    qr, kr = _rotate_complex(q, th, pi, pj), _rotate_complex(k, th, pi, pj)
    ref = F.scaled_dot_product_attention(qr.transpose(0, 1), kr.transpose(0, 1), v.transpose(0, 1))
    assert _rel(r["o"][0].reshape(M * M, h, d), ref.transpose(0, 1).numpy()) < 1e-12


def test_rope_scores_depend_on_relative_offset_only():
    """With the same vector for every query and key, score(t, u) = f(p_u - p_t)
    with f even, so lse is symmetric under the point reflection of the window."""
    B, H, W, h, d, M = 1, 8, 8, 1, 16, 8
    g = torch.Generator().manual_seed(7)
    vec = torch.randn(d, generator=g, dtype=torch.float64) * 2
    q = vec.expand(B, H, W, h, d).contiguous()
    v = torch.randn(B, H, W, h, d, generator=g, dtype=torch.float64)
    th = theta_init(h, d).double() * 2.5
    r = oracle.full(q, q, v, th, M, 0)
    lse = r["lse"][0, :, :, 0]
    assert np.allclose(lse, lse[::-1, ::-1], rtol=0, atol=1e-12)
    assert not np.allclose(lse, lse.T, rtol=0, atol=1e-6)  # x and y frequencies differ


@pytest.mark.parametrize("s", [0, 2])
def test_softmax_rows_sum_to_one(s):
    """V constant => O equals that constant, with and without the shift mask."""
    B, H, W, h, d, M = 1, 8, 8, 2, 8, 4
    inp = make_inputs(B, H, W, h, d)
    c = torch.linspace(-2, 3, d, dtype=torch.float64)
    v = c.expand(B, H, W, h, d).contiguous()
    r = oracle.full(inp["q"], inp["k"], v, inp["theta"], M, s)
    assert np.abs(r["o"] - c.numpy()).max() < 1e-13


def test_shift_consistency_interior_windows():
    """Windows outside the last window row/column are unmasked: with shift s they
    equal the s = 0 result on the grid rolled by -s (torch.roll)."""
    B, H, W, h, d, M, s = 1, 12, 8, 2, 8, 4, 2
    inp = make_inputs(B, H, W, h, d)
    r = oracle.full(inp["q"], inp["k"], inp["v"], inp["theta"], M, s)
    rolled = [torch.roll(inp[x], (-s, -s), (1, 2)) for x in ("q", "k", "v")]
    r0 = oracle.full(*rolled, inp["theta"], M, 0)
    o_back = np.roll(r0["o"], (s, s), (1, 2))
    lse_back = np.roll(r0["lse"], (s, s), (1, 2))
    for rr in range(H - M):
        for cc in range(W - M):
            ro, co = (rr + s) % H, (cc + s) % W
            assert np.allclose(r["o"][0, ro, co], o_back[0, ro, co], rtol=0, atol=1e-13)
            assert np.allclose(r["lse"][0, ro, co], lse_back[0, ro, co], rtol=0, atol=1e-13)
    # and the last window row does differ (the mask is active there)
    assert not np.allclose(r["o"][0, (H - 1 + s) % H], o_back[0, (H - 1 + s) % H], atol=1e-6)


@pytest.mark.parametrize("s,d", [(0, 8), (2, 8), (2, 64)])
def test_finite_difference_gradients(s, d):
    """Central differences of L = sum(O * dO) in fp64 (rel. err <= 1e-6)."""
    B, H, W, h, M = 1, 8, 8, 2, 4
    inp = _f64(make_inputs(B, H, W, h, d))
    inp["theta"] = inp["theta"] * 3.0
    r = oracle.full(inp["q"], inp["k"], inp["v"], inp["theta"], M, s, dout=inp["dout"])
    do = inp["dout"].numpy()

    def loss(**kw):
        args = {x: inp[x] for x in ("q", "k", "v", "theta")}
        args.update(kw)
        o = oracle.full(args["q"], args["k"], args["v"], args["theta"], M, s)["o"]
        return float((o * do).sum())

    eps = 1e-5
    rng = np.random.default_rng(0)
    for name, grad in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("theta", "dtheta")):
        base = inp[name].numpy()
        flat_ids = rng.choice(base.size, size=min(base.size, 12), replace=False)
        for fid in flat_ids:
            idx = np.unravel_index(fid, base.shape)
            plus, minus = base.copy(), base.copy()
            plus[idx] += eps
            minus[idx] -= eps
            fd = (loss(**{name: plus}) - loss(**{name: minus})) / (2 * eps)
            an = r[grad][idx]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, idx, fd, an)


def test_units_api_matches_full():
    B, H, W, h, d, M, s = 2, 8, 8, 2, 8, 4, 2
    inp = make_inputs(B, H, W, h, d)
    r = oracle.full(inp["q"], inp["k"], inp["v"], inp["theta"], M, s, dout=inp["dout"])
    ids = [0, 5, 13, 15]
    u = oracle.units(inp["q"], inp["k"], inp["v"], inp["theta"], M, s, ids, dout=inp["dout"])
    for n, uid in enumerate(ids):
        b, rows, cols, hh = oracle.unit_token_positions(H, W, M, s, uid, h)
        for key in ("o", "dq", "dk", "dv"):
            assert np.array_equal(u[key][n], r[key][b, rows, cols, hh])
        assert np.array_equal(u["lse"][n], r["lse"][b, rows, cols, hh])
    all_ids = list(range(B * (H // M) * (W // M) * h))
    ua = oracle.units(inp["q"], inp["k"], inp["v"], inp["theta"], M, s, all_ids, dout=inp["dout"])
    dth = np.zeros_like(r["dtheta"])
    for uid in all_ids:
        dth[uid % h] += ua["dtheta"][uid]
    assert _rel(dth, r["dtheta"]) < 1e-13
