"""Inference forward: fs_winattn_fwd with no log-sum-exp buffer (the workload of
FlashSwin's inference-throughput figure, thelatestinai.com Fig. S1).

It must write the same O as the training forward, bit for bit (the same
kernels; only the LSE store is skipped), and so match the fp64 oracle within
the forward tolerance; the LSE buffer of a training call is left as it was.
"""
import numpy as np
import pytest
import torch

import oracle
from vision_transformer_windowed_b200 import _lib, ops
from vision_transformer_windowed_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu

CASES = [  # (B, H, W, heads, M, s): both kernel families, shifted and not, ragged tiles
    (1, 16, 16, 2, 8, 0),
    (2, 16, 16, 3, 8, 4),
    (1, 8, 12, 2, 4, 0),
    (1, 32, 48, 1, 16, 4),
    (1, 64, 64, 1, 32, 16),
    (1, 64, 64, 1, 64, 32),
    (1, 20, 13, 2, 8, 4),     # padded grids
    (1, 33, 20, 1, 16, 4),
]


@pytest.fixture(autouse=True)
def _device_status_clean():
    _lib.fs_set_wait_limit_ns(4_000_000_000)
    _lib.fs_device_status()  # clear
    yield
    torch.cuda.synchronize()
    assert _lib.fs_device_status() == 0


@pytest.mark.parametrize("B,H,W,heads,M,s", CASES)
def test_inference_forward_equals_training_forward_and_oracle(B, H, W, heads, M, s):
    inp = make_inputs(B, H, W, heads, 32, with_dout=False)
    dev = {k: v.cuda() for k, v in inp.items()}
    o_train, lse = ops.winattn_fwd(dev["q"], dev["k"], dev["v"], dev["theta"], M, s)
    o_inf, none = ops.winattn_fwd(dev["q"], dev["k"], dev["v"], dev["theta"], M, s, need_lse=False)
    torch.cuda.synchronize()
    assert none is None
    assert torch.equal(o_inf, o_train)
    ref = oracle.full(inp["q"], inp["k"], inp["v"], inp["theta"], M, s)
    got = o_inf.float().cpu().numpy().astype(np.float64)
    err = np.abs(got - ref["o"]).max()
    assert err <= 1e-2 * np.abs(ref["o"]).max() + 2e-3


def test_inference_forward_leaves_an_lse_buffer_untouched():
    B, H, W, heads, M, s = 2, 32, 32, 3, 8, 4
    t = make_inputs(B, H, W, heads, 32, device="cuda", with_dout=False)
    sentinel = torch.full((B, H, W, heads), 12345.0, device="cuda")
    o, lse = ops.winattn_fwd(t["q"], t["k"], t["v"], t["theta"], M, s, need_lse=False)
    torch.cuda.synchronize()
    assert lse is None and torch.all(sentinel == 12345.0)
    _, lse_train = ops.winattn_fwd(t["q"], t["k"], t["v"], t["theta"], M, s, lse=sentinel)
    torch.cuda.synchronize()
    assert lse_train.data_ptr() == sentinel.data_ptr() and not torch.any(sentinel == 12345.0)
