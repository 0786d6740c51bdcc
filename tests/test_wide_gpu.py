"""GPU parity for heads of 64 channels (the wide kernels) against the fp64 oracle.

The same shape lists as the 32-channel parity tests (every window size, shifted
and not, ragged tiles, padded grids), element by element, with the same
tolerances; plus upstream gradients at training magnitudes compared at their unit
scale, and a sharpened softmax.
"""
import numpy as np
import pytest
import torch

import oracle
from vision_transformer_windowed_b200 import _lib, ops
from vision_transformer_windowed_b200.inputs import make_inputs

FWD_TOL = (1e-2, 2e-3)
GRAD_TOL = (3e-2, 5e-3)
D = 64


def check(name, got, ref, tol):
    got = got.detach().double().cpu().numpy() if isinstance(got, torch.Tensor) else np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, name
    assert np.isfinite(got).all(), f"{name}: non-finite values"
    err = np.abs(got - ref).max() if got.size else 0.0
    bound = tol[0] * (np.abs(ref).max() if ref.size else 0.0) + tol[1]
    assert err <= bound, f"{name}: max|err| {err:.4g} > {bound:.4g}"


@pytest.fixture(autouse=True)
def _device_status_clean():
    _lib.fs_set_wait_limit_ns(4_000_000_000)
    _lib.fs_device_status()  # clear
    yield
    torch.cuda.synchronize()
    assert _lib.fs_device_status() == 0


def run_both(B, H, W, h, M, s, qk_scale=1.0, dout_scale=1.0):
    inp = make_inputs(B, H, W, h, D, qk_scale=qk_scale)
    dev = {k: v.cuda() for k, v in inp.items()}
    o, lse = ops.winattn_fwd(dev["q"], dev["k"], dev["v"], dev["theta"], M, s)
    dout = dev["dout"] * dout_scale if dout_scale != 1.0 else dev["dout"]
    dq, dk, dv, dth = ops.winattn_bwd(dev["q"], dev["k"], dev["v"], o, dout, lse, dev["theta"], M, s)
    torch.cuda.synchronize()
    if dout_scale != 1.0:
        dq, dk, dv, dth = (t.double() / dout_scale for t in (dq, dk, dv, dth))
    ref = oracle.full(inp["q"], inp["k"], inp["v"], inp["theta"], M, s, dout=inp["dout"])
    return {"o": o, "lse": lse, "dq": dq, "dk": dk, "dv": dv, "dtheta": dth}, ref


SMALL = [  # (B, H, W, heads, M, s)
    (1, 16, 16, 2, 8, 0),
    (2, 16, 16, 3, 8, 4),
    (1, 8, 24, 1, 8, 4),      # ragged last tile
    (1, 8, 12, 2, 4, 0),      # 16-token windows, ragged
    (1, 32, 32, 2, 16, 8),
    (1, 32, 48, 1, 16, 4),
    (1, 64, 64, 1, 32, 16),
    (2, 32, 32, 2, 32, 0),
    (1, 64, 64, 1, 64, 32),   # 4096-token window
    (1, 64, 96, 1, 32, 12),
    (1, 16, 16, 6, 8, 4),
    (1, 32, 32, 12, 32, 16),
    (1, 16, 16, 24, 16, 0),
]

PADDED = [  # H or W not a multiple of M: padded with zero tokens
    (1, 20, 13, 2, 8, 4),
    (2, 12, 18, 3, 8, 0),
    (1, 10, 6, 1, 4, 0),
    (1, 50, 83, 3, 8, 4),
    (1, 40, 36, 2, 16, 8),
    (1, 33, 20, 1, 16, 4),
    (1, 70, 50, 1, 32, 16),
    (1, 100, 70, 1, 64, 32),
]


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", SMALL + PADDED)
def test_d64_fwd_bwd_parity(cfg):
    got, ref = run_both(*cfg)
    check("o", got["o"], ref["o"], FWD_TOL)
    check("lse", got["lse"], ref["lse"], FWD_TOL)
    for key in ("dq", "dk", "dv", "dtheta"):
        check(key, got[key], ref[key], GRAD_TOL)


@pytest.mark.gpu
@pytest.mark.parametrize("dout_scale", [2.0 ** -20, 2.0 ** 12], ids=["2^-20", "2^12"])
@pytest.mark.parametrize("cfg", [(2, 16, 16, 3, 8, 4), (1, 20, 13, 2, 8, 4), (1, 64, 64, 1, 32, 16),
                                 (1, 70, 50, 1, 32, 16)])
def test_d64_gradient_magnitude_parity(cfg, dout_scale):
    got, ref = run_both(*cfg, dout_scale=dout_scale)
    for key in ("dq", "dk", "dv", "dtheta"):
        check(key, got[key], ref[key], GRAD_TOL)


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", [(2, 16, 16, 3, 8, 4), (1, 64, 64, 1, 32, 16)])
def test_d64_sharp_softmax_parity(cfg):
    got, ref = run_both(*cfg, qk_scale=3.0)
    check("o", got["o"], ref["o"], FWD_TOL)
    check("lse", got["lse"], ref["lse"], FWD_TOL)
    for key in ("dq", "dk", "dv", "dtheta"):
        check(key, got[key], ref[key], GRAD_TOL)


@pytest.mark.gpu
def test_d64_inference_forward_writes_o_only():
    inp = make_inputs(1, 16, 16, 2, D)
    dev = {k: v.cuda() for k, v in inp.items()}
    o_train, _ = ops.winattn_fwd(dev["q"], dev["k"], dev["v"], dev["theta"], 8, 4)
    o_inf, _ = ops.winattn_fwd(dev["q"], dev["k"], dev["v"], dev["theta"], 8, 4, need_lse=False)
    torch.cuda.synchronize()
    assert torch.equal(o_train, o_inf)


@pytest.mark.gpu
def test_d64_empty_batch_zeroes_dtheta():
    inp = make_inputs(0, 16, 16, 2, D)
    dev = {k: v.cuda() for k, v in inp.items()}
    o, lse = ops.winattn_fwd(dev["q"], dev["k"], dev["v"], dev["theta"], 8, 0)
    dth = torch.full_like(dev["theta"], 7.0)
    ops.winattn_bwd(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, dev["theta"], 8, 0, dtheta=dth)
    torch.cuda.synchronize()
    assert o.numel() == 0 and (dth == 0).all()
