"""The backward entry point that allocates nothing (fs_winattn_bwd_noalloc).

It exists for callers that cannot allocate device memory when they run the
backward (a memory pool already handed out, a runtime that forbids cudaMalloc
after start-up): instead of a caller workspace it uses one fixed scratch array
inside the library.  These tests call it through the C ABI and compare it with
the regular entry point, which gets a workspace allocated by the caller.

This file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

from vision_transformer_windowed_b200 import _lib, ops
from vision_transformer_windowed_b200.inputs import make_inputs

GRAD_TOL = (3e-2, 5e-3)  # the gradient tolerance of the parity tests


def _close(name, got, ref, tol):
    g = got.detach().float().cpu().numpy().astype(np.float64)
    r = ref.detach().float().cpu().numpy().astype(np.float64)
    err = np.abs(g - r).max()
    bound = tol[0] * np.abs(r).max() + tol[1]
    assert np.isfinite(g).all() and err <= bound, f"{name}: max|err| {err:.4g} > {bound:.4g}"


def test_oversized_problem_is_rejected_without_launch():
    big = _lib.make_shape(128, 128, 128, 3, 32, 32, 16)  # needs far more than the fixed scratch
    assert _lib.fs_winattn_bwd_workspace_bytes(big) > _lib.fs_winattn_bwd_noalloc_max_bytes()
    with pytest.raises(_lib.FswinError) as e:
        _lib.fs_winattn_bwd_noalloc(big, *([256] * 11), 0)
    assert e.value.status == _lib.FS_ERR_WORKSPACE


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", [(2, 32, 32, 2, 16, 8), (1, 16, 16, 2, 8, 4), (1, 20, 13, 2, 8, 4), (1, 33, 20, 1, 16, 4)])
def test_noalloc_matches_workspace_entry_point_twice(cfg):
    B, H, W, h, M, s = cfg
    inp = make_inputs(B, H, W, h, 32)
    d = {k: v.cuda() for k, v in inp.items()}
    o, lse = ops.winattn_fwd(d["q"], d["k"], d["v"], d["theta"], M, s)
    ref = ops.winattn_bwd(d["q"], d["k"], d["v"], o, d["dout"], lse, d["theta"], M, s)
    sh = _lib.make_shape(B, H, W, h, 32, M, s)
    assert _lib.fs_winattn_bwd_workspace_bytes(sh) <= _lib.fs_winattn_bwd_noalloc_max_bytes()
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):  # the scratch keeps the previous call's contents; results must not depend on it
        dq, dk, dv = (torch.full_like(d["q"], float("nan")) for _ in range(3))
        dth = torch.full_like(d["theta"], float("nan"))
        _lib.fs_winattn_bwd_noalloc(sh, d["q"].data_ptr(), d["k"].data_ptr(), d["v"].data_ptr(), o.data_ptr(),
                                    d["dout"].data_ptr(), lse.data_ptr(), d["theta"].data_ptr(), dq.data_ptr(),
                                    dk.data_ptr(), dv.data_ptr(), dth.data_ptr(), stream)
        torch.cuda.synchronize()
        assert _lib.fs_device_status() == 0
        for name, got, want in (("dq", dq, ref[0]), ("dk", dk, ref[1]), ("dv", dv, ref[2]), ("dtheta", dth, ref[3])):
            _close(name, got, want, GRAD_TOL)
