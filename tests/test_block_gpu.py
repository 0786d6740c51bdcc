"""GPU parity of the attention block with its projections (fs_winattn_block_fwd)
against the fp64 block oracle (oracle/block.py): y within the forward
tolerance, max|err| <= 1e-2 * max|ref| + 2e-3."""
import numpy as np
import pytest
import torch

from oracle.block import block_forward
from vision_transformer_windowed_b200 import _lib, ops
from vision_transformer_windowed_b200.inputs import make_block_inputs

pytestmark = pytest.mark.gpu

CASES = [  # (B, H, W, heads, M, s)
    (1, 16, 16, 3, 8, 0),   # 4 windows of 64 tokens: 2 tiles
    (2, 16, 16, 3, 8, 4),   # shifted, 4 x 4 boxes
    (1, 8, 24, 2, 8, 4),    # 3 windows: a ragged last tile
    (1, 8, 12, 1, 4, 0),    # 16-token windows, one head
    (3, 32, 32, 3, 8, 4),   # more tiles than one CTA's first item
    (1, 16, 16, 2, 4, 0),
    (1, 20, 13, 3, 8, 4),   # grid padded to 24 x 16: padded tokens carry the bias
    (2, 10, 6, 2, 4, 0),
]


@pytest.fixture(autouse=True)
def _device_status_clean():
    _lib.fs_set_wait_limit_ns(4_000_000_000)
    _lib.fs_device_status()
    yield
    torch.cuda.synchronize()
    assert _lib.fs_device_status() == 0


@pytest.mark.parametrize("B,H,W,heads,M,s", CASES)
def test_block_forward_matches_oracle(B, H, W, heads, M, s):
    inp = make_block_inputs(B, H, W, heads, 32)
    dev = {k: v.cuda() for k, v in inp.items()}
    y = ops.winattn_block_fwd(dev["x"], dev["w_qkv"], dev["b_qkv"], dev["w_o"], dev["b_o"], dev["theta"], M, s, heads)
    torch.cuda.synchronize()
    ref, _ = block_forward(inp["x"], inp["w_qkv"], inp["b_qkv"], inp["w_o"], inp["b_o"], inp["theta"], M, s, heads)
    got = y.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    err = np.abs(got - ref).max()
    assert err <= 1e-2 * np.abs(ref).max() + 2e-3, f"max|err| {err:.4g}, max|ref| {np.abs(ref).max():.4g}"


def test_block_forward_is_deterministic_and_matches_the_unfused_path():
    """Twice bit for bit; and against our attention kernel between torch projections
    (same arithmetic up to where q, k, v and o are rounded)."""
    B, H, W, heads, M, s = 2, 32, 32, 3, 8, 4
    inp = make_block_inputs(B, H, W, heads, 32, device="cuda")
    args = (inp["x"], inp["w_qkv"], inp["b_qkv"], inp["w_o"], inp["b_o"], inp["theta"], M, s, heads)
    y1 = ops.winattn_block_fwd(*args)
    y2 = ops.winattn_block_fwd(*args)
    C = heads * 32
    qkv = (inp["x"].float() @ inp["w_qkv"].float().T + inp["b_qkv"]).reshape(B, H, W, 3, heads, 32)
    q, k, v = (qkv[..., i, :, :].to(torch.bfloat16).contiguous() for i in range(3))
    o, _ = ops.winattn_fwd(q, k, v, inp["theta"], M, s, need_lse=False)
    y3 = o.float().reshape(B, H, W, C) @ inp["w_o"].float().T + inp["b_o"]
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    err = (y1.float() - y3).abs().max().item()
    assert err <= 1e-2 * y3.abs().max().item() + 2e-3, err
