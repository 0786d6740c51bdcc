"""Pins of the attention block's backward oracle (oracle.block.block_backward)
to things other than itself:

* torch float64 autograd through an independent restatement of the block
  (einsum projections around the tensor-level attention of oracle/literal.py),
  on grids that are multiples of the window;
* central finite differences of the C-oracle block forward at sampled
  coordinates of every gradient, on a grid that is not a multiple of the window
  (so the padding tokens' share of db_qkv is checked too).
A dropped term of the chain rule, a transposed weight gradient, q, k, v stacked
in the wrong channel order or the padding tokens' gradient kept in dx fails one
of them.
"""
import numpy as np
import pytest
import torch

import oracle.literal as lit
from oracle.block import block_backward, block_forward
from vision_transformer_windowed_b200.inputs import make_block_inputs

GRADS = ("dx", "dw_qkv", "db_qkv", "dw_o", "db_o", "dtheta")


def _inputs(B, H, W, heads, seed=0):
    inp = {k: v.to(torch.float64) for k, v in make_block_inputs(B, H, W, heads, 32).items()}
    g = torch.Generator().manual_seed(100 + seed)
    inp["dy"] = torch.randn(inp["x"].shape, generator=g, dtype=torch.float64)
    return inp


def _autograd(inp, heads, M, s):
    leaves = {k: inp[k].clone().requires_grad_(True) for k in ("x", "w_qkv", "b_qkv", "w_o", "b_o", "theta")}
    x = leaves["x"]
    B, H, W, C = x.shape
    qkv = torch.einsum("bhwc,nc->bhwn", x, leaves["w_qkv"]) + leaves["b_qkv"]
    q, k, v = qkv.reshape(B, H, W, 3, heads, C // heads).unbind(3)
    o, _ = lit.forward(q, k, v, leaves["theta"], M, s)
    y = torch.einsum("bhwc,nc->bhwn", o.reshape(B, H, W, C), leaves["w_o"]) + leaves["b_o"]
    (y * inp["dy"]).sum().backward()
    return {"d" + k: leaves[k].grad.numpy() for k in leaves}


@pytest.mark.parametrize("shape", [(1, 8, 8, 2, 4, 0), (2, 8, 8, 1, 8, 4), (1, 16, 16, 2, 8, 4)])
def test_block_backward_matches_autograd_of_a_restatement(shape):
    B, H, W, heads, M, s = shape
    inp = _inputs(B, H, W, heads)
    got = block_backward(inp["x"], inp["w_qkv"], inp["b_qkv"], inp["w_o"], inp["b_o"], inp["theta"], M, s, heads,
                         inp["dy"], nthreads=2)
    ref = _autograd(inp, heads, M, s)
    for name in GRADS:
        np.testing.assert_allclose(got[name], ref[name], rtol=1e-9, atol=1e-10, err_msg=name)


def test_block_backward_matches_finite_differences_on_a_padded_grid():
    B, H, W, heads, M, s = 1, 10, 7, 2, 4, 0  # padded to 12 x 8
    inp = _inputs(B, H, W, heads, seed=1)
    names = {"dx": "x", "dw_qkv": "w_qkv", "db_qkv": "b_qkv", "dw_o": "w_o", "db_o": "b_o", "dtheta": "theta"}
    got = block_backward(inp["x"], inp["w_qkv"], inp["b_qkv"], inp["w_o"], inp["b_o"], inp["theta"], M, s, heads,
                         inp["dy"], nthreads=2)
    dy = inp["dy"].numpy()

    def loss(args):
        y, _ = block_forward(args["x"], args["w_qkv"], args["b_qkv"], args["w_o"], args["b_o"], args["theta"], M, s,
                             heads, nthreads=2)
        return float((y * dy).sum())

    rng = np.random.default_rng(7)
    eps = 1e-5
    for gname, pname in names.items():
        base = {k: inp[k].numpy().copy() for k in names.values()}
        flat = base[pname].reshape(-1)
        for idx in rng.choice(flat.size, size=6, replace=False):
            keep = flat[idx]
            flat[idx] = keep + eps
            up = loss(base)
            flat[idx] = keep - eps
            down = loss(base)
            flat[idx] = keep
            fd = (up - down) / (2 * eps)
            an = got[gname].reshape(-1)[idx]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (gname, idx, fd, an)
