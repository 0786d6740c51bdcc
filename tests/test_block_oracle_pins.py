"""Pins of the attention-block oracle (oracle/block.py) to things other than itself.

* an independent restatement: torch float64 projections (einsum) around the
  tensor-level attention of oracle/literal.py, on tiny grids;
* a closed form: with W_v = 0 every value row is b_v, so every attention output
  row is b_v (softmax rows sum to one) and y = b_v W_o^T + b_o whatever q and k;
* exact affinity of y in (W_o, b_o), and head separation: zeroing the W_o
  columns of one head removes exactly that head's share.
"""
import numpy as np
import pytest
import torch

import oracle.literal as lit
from oracle.block import block_forward, project_qkv
from vision_transformer_windowed_b200.inputs import make_block_inputs

SHAPES = [(1, 8, 8, 2, 4, 0), (2, 8, 8, 1, 4, 2), (1, 16, 16, 3, 8, 4)]  # B, H, W, heads, M, s


def _restated(inp, heads, M, s):
    x = inp["x"].to(torch.float64)
    B, H, W, C = x.shape
    d = C // heads
    qkv = torch.einsum("bhwc,nc->bhwn", x, inp["w_qkv"].to(torch.float64)) + inp["b_qkv"].to(torch.float64)
    q, k, v = qkv.reshape(B, H, W, 3, heads, d).unbind(3)
    o, _ = lit.forward(q, k, v, inp["theta"].to(torch.float64), M, s)
    y = torch.einsum("bhwc,nc->bhwn", o.reshape(B, H, W, C), inp["w_o"].to(torch.float64))
    return (y + inp["b_o"].to(torch.float64)).numpy()


@pytest.mark.parametrize("shape", SHAPES)
def test_block_oracle_matches_tensor_level_restatement(shape):
    B, H, W, heads, M, s = shape
    inp = make_block_inputs(B, H, W, heads, 32)
    y, _ = block_forward(inp["x"], inp["w_qkv"], inp["b_qkv"], inp["w_o"], inp["b_o"], inp["theta"], M, s, heads,
                         nthreads=2)
    np.testing.assert_allclose(y, _restated(inp, heads, M, s), rtol=1e-10, atol=1e-10)


def test_zero_value_weights_give_the_value_bias_everywhere():
    B, H, W, heads, M, s = 1, 16, 16, 2, 8, 4
    inp = make_block_inputs(B, H, W, heads, 32)
    C = heads * 32
    w = inp["w_qkv"].clone()
    w[2 * C:] = 0
    y, o = block_forward(inp["x"], w, inp["b_qkv"], inp["w_o"], inp["b_o"], inp["theta"], M, s, heads, nthreads=2)
    bv = inp["b_qkv"][2 * C:].to(torch.float64).numpy()
    np.testing.assert_allclose(o.reshape(B, H, W, C), np.broadcast_to(bv, (B, H, W, C)), rtol=0, atol=1e-12)
    expect = bv @ inp["w_o"].to(torch.float64).numpy().T + inp["b_o"].to(torch.float64).numpy()
    np.testing.assert_allclose(y, np.broadcast_to(expect, y.shape), rtol=0, atol=1e-12)


def test_output_is_affine_in_the_output_map_and_separates_heads():
    B, H, W, heads, M, s = 1, 16, 16, 3, 8, 0
    inp = make_block_inputs(B, H, W, heads, 32)
    args = (inp["x"], inp["w_qkv"], inp["b_qkv"])
    y1, o = block_forward(*args, inp["w_o"], inp["b_o"], inp["theta"], M, s, heads, nthreads=2)
    y2, _ = block_forward(*args, 2 * inp["w_o"].double(), 2 * inp["b_o"], inp["theta"], M, s, heads, nthreads=2)
    np.testing.assert_allclose(y2, 2 * y1, rtol=1e-12, atol=1e-12)
    wo = inp["w_o"].double().clone()
    wo[:, 32:64] = 0  # drop head 1
    y3, _ = block_forward(*args, wo, inp["b_o"], inp["theta"], M, s, heads, nthreads=2)
    head1 = o[..., 1, :] @ inp["w_o"].double()[:, 32:64].numpy().T
    np.testing.assert_allclose(y1 - y3, head1, rtol=1e-10, atol=1e-10)


def test_projection_splits_channels_as_q_k_v_then_heads():
    """Output channel n of the qkv map is (part, head, e) = divmod order (3, heads, d)."""
    inp = make_block_inputs(1, 8, 8, 2, 32)
    q, k, v = project_qkv(inp["x"], inp["w_qkv"], inp["b_qkv"], 2)
    x = inp["x"].double().numpy()[0, 3, 5]
    w = inp["w_qkv"].double().numpy()
    b = inp["b_qkv"].double().numpy()
    for part, t in enumerate((q, k, v)):
        for h in range(2):
            for e in (0, 17, 31):
                n = part * 64 + h * 32 + e
                assert abs(t[0, 3, 5, h, e] - (x @ w[n] + b[n])) < 1e-12
