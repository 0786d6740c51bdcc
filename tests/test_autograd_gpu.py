"""The torch.autograd wrapper (ops.window_attention) against the fp64 oracle.

The pages learn the RoPE frequencies in log form, theta = exp(omega)
(thelatestinai.com/papers/2610.04664, Figure S4); the library takes theta and
returns d theta, and autograd through torch.exp then gives d omega =
theta * d theta.  Both kernels run through the C ABI.
"""
import numpy as np
import pytest
import torch

import oracle
from vision_transformer_windowed_b200 import _lib, ops
from vision_transformer_windowed_b200.inputs import make_inputs

FWD_TOL = (1e-2, 2e-3)
GRAD_TOL = (3e-2, 5e-3)


def _check(name, got, ref, tol):
    got = got.detach().float().cpu().numpy().astype(np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, name
    err = np.abs(got - ref).max()
    bound = tol[0] * np.abs(ref).max() + tol[1]
    assert err <= bound, f"{name}: max|err| {err:.4g} > {bound:.4g}"


@pytest.fixture(autouse=True)
def _device_status_clean():
    _lib.fs_set_wait_limit_ns(4_000_000_000)
    _lib.fs_device_status()
    yield
    torch.cuda.synchronize()
    assert _lib.fs_device_status() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", [(2, 16, 16, 3, 8, 4), (1, 64, 64, 1, 32, 16), (1, 20, 13, 2, 8, 4)])
def test_autograd_with_log_frequencies(cfg):
    B, H, W, heads, M, s = cfg
    inp = make_inputs(B, H, W, heads, 32)
    dev = {k: v.cuda() for k, v in inp.items()}
    q, k, v = (dev[x].clone().requires_grad_(True) for x in ("q", "k", "v"))
    # log frequencies (the seeded theta, whose noise can make a small one negative, by magnitude)
    omega0 = torch.log(inp["theta"].abs() + 1e-3)
    omega = omega0.cuda().requires_grad_(True)
    o = ops.window_attention(q, k, v, torch.exp(omega), M, s)
    (o.float() * dev["dout"].float()).sum().backward()
    torch.cuda.synchronize()
    theta = torch.exp(omega0.double())  # the theta the kernels saw, up to fp32 rounding
    ref = oracle.full(inp["q"], inp["k"], inp["v"], theta, M, s, dout=inp["dout"])
    _check("o", o, ref["o"], FWD_TOL)
    _check("dq", q.grad, ref["dq"], GRAD_TOL)
    _check("dk", k.grad, ref["dk"], GRAD_TOL)
    _check("dv", v.grad, ref["dv"], GRAD_TOL)
    _check("domega", omega.grad, theta.numpy() * ref["dtheta"], GRAD_TOL)
