"""GPU parity of the training pair (fs_winattn_fwd_train / fs_winattn_bwd_train)
against the fp64 oracle.

The training forward leaves the rotated q', k' tiles in the backward's
workspace and, for windows of >= 128 tokens, reads its own Q', K' tiles from
them; the backward then reuses them.  Same shape lists and tolerances as the
stand-alone calls, plus a check that the backward's results equal those of the
stand-alone backward bit for bit where that one is deterministic (dk, dv), and
the autograd wrapper with reuse_rotated=True (which uses the pair).
"""
import numpy as np
import pytest
import torch

import oracle
from vision_transformer_windowed_b200 import _lib, ops
from vision_transformer_windowed_b200.inputs import make_inputs

from test_parity_gpu import FWD_TOL, GRAD_TOL, PADDED, SMALL, check


@pytest.fixture(autouse=True)
def _device_status_clean():
    _lib.fs_set_wait_limit_ns(4_000_000_000)
    _lib.fs_device_status()  # clear
    yield
    torch.cuda.synchronize()
    assert _lib.fs_device_status() == 0


def run_pair(B, H, W, h, M, s, d=32, qk_scale=1.0, dout_scale=1.0):
    inp = make_inputs(B, H, W, h, d, qk_scale=qk_scale)
    dev = {k: v.cuda() for k, v in inp.items()}
    ws = ops.alloc_workspace(dev["q"], M, s)
    ws.fill_(0xFF)  # the pair must not depend on what the workspace held before
    o, lse = ops.winattn_fwd(dev["q"], dev["k"], dev["v"], dev["theta"], M, s, workspace=ws)
    dout = dev["dout"] * dout_scale if dout_scale != 1.0 else dev["dout"]
    dq, dk, dv, dth = ops.winattn_bwd(dev["q"], dev["k"], dev["v"], o, dout, lse, dev["theta"], M, s,
                                      workspace=ws, after_train_fwd=True)
    torch.cuda.synchronize()
    if dout_scale != 1.0:
        dq, dk, dv, dth = (t.double() / dout_scale for t in (dq, dk, dv, dth))
    ref = oracle.full(inp["q"], inp["k"], inp["v"], inp["theta"], M, s, dout=inp["dout"])
    return {"o": o, "lse": lse, "dq": dq, "dk": dk, "dv": dv, "dtheta": dth}, ref, dev


def _compare(got, ref):
    check("o", got["o"], ref["o"], FWD_TOL)
    check("lse", got["lse"], ref["lse"], FWD_TOL)
    for key in ("dq", "dk", "dv", "dtheta"):
        check(key, got[key], ref[key], GRAD_TOL)


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", SMALL + PADDED)
def test_train_pair_parity(cfg):
    got, ref, _ = run_pair(*cfg)
    _compare(got, ref)


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", [(1, 16, 16, 2, 8, 4), (1, 64, 64, 1, 32, 16), (1, 70, 50, 1, 32, 16)])
def test_train_pair_parity_d64(cfg):
    got, ref, _ = run_pair(*cfg, d=64)
    _compare(got, ref)


@pytest.mark.gpu
@pytest.mark.parametrize("dout_scale", [2.0 ** -20, 2.0 ** 12], ids=["2^-20", "2^12"])
@pytest.mark.parametrize("cfg", [(1, 64, 64, 1, 32, 16), (1, 32, 48, 1, 16, 4), (1, 64, 64, 1, 64, 32)])
def test_train_pair_gradient_magnitude(cfg, dout_scale):
    got, ref, _ = run_pair(*cfg, dout_scale=dout_scale)
    for key in ("dq", "dk", "dv", "dtheta"):
        check(key, got[key], ref[key], GRAD_TOL)


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", [(1, 64, 64, 1, 32, 16), (2, 32, 32, 2, 16, 0)])
def test_train_pair_sharp_softmax(cfg):
    got, ref, _ = run_pair(*cfg, qk_scale=3.0)
    _compare(got, ref)


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", [(2, 64, 64, 3, 32, 16), (1, 100, 70, 1, 64, 32)])
def test_train_backward_matches_standalone_backward(cfg):
    """The reused images are those the stand-alone backward computes itself:
    dk and dv (no reductions in any order) are bit-identical."""
    got, _, dev = run_pair(*cfg)
    B, H, W, h, M, s = cfg
    dq, dk, dv, dth = ops.winattn_bwd(dev["q"], dev["k"], dev["v"], got["o"], dev["dout"], got["lse"],
                                      dev["theta"], M, s)
    torch.cuda.synchronize()
    assert torch.equal(dk, got["dk"]) and torch.equal(dv, got["dv"])


@pytest.mark.gpu
def test_autograd_with_the_pair():
    inp = make_inputs(1, 64, 64, 2, 32)
    leaves = {k: v.cuda().requires_grad_(k != "dout") for k, v in inp.items()}
    o = ops.window_attention(leaves["q"], leaves["k"], leaves["v"], leaves["theta"], 32, 16, reuse_rotated=True)
    (o.float() * leaves["dout"].float()).sum().backward()
    ref = oracle.full(inp["q"], inp["k"], inp["v"], inp["theta"], 32, 16, dout=inp["dout"])
    check("o", o, ref["o"], FWD_TOL)
    for key, t in (("dq", leaves["q"]), ("dk", leaves["k"]), ("dv", leaves["v"]), ("dtheta", leaves["theta"])):
        check(key, t.grad, ref[key], GRAD_TOL)
