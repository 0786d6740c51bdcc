"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Tolerances (bf16 inputs/outputs, fp32 accumulation):
  forward outputs (o, lse):   max|err| <= 1e-2 * max|ref| + 2e-3
  gradients (dq, dk, dv, dθ): max|err| <= 3e-2 * max|ref| + 5e-3
"""
import numpy as np
import pytest
import torch

import oracle
from vision_transformer_windowed_b200 import _lib, ops
from vision_transformer_windowed_b200.inputs import make_inputs

FWD_TOL = (1e-2, 2e-3)
GRAD_TOL = (3e-2, 5e-3)


def check(name, got, ref, tol):
    got = got.detach().float().cpu().numpy() if isinstance(got, torch.Tensor) else np.asarray(got)
    got = got.astype(np.float64)
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
    """The CUDA path and the oracle on the same seeded inputs.  With dout_scale
    (a power of two) the CUDA path gets dO * dout_scale, its gradients are
    divided by dout_scale (both exact in binary floating point), and the oracle
    runs at scale 1: the comparison is then made at the gradients' unit scale,
    so the absolute term of the tolerance cannot hide an underflow."""
    inp = make_inputs(B, H, W, h, 32, qk_scale=qk_scale)
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
    (1, 16, 16, 2, 8, 0),     # the tiny configuration: 4 windows of 64 tokens
    (2, 16, 16, 3, 8, 4),     # shifted, 4x4 boxes
    (1, 8, 24, 1, 8, 4),      # 3 windows: ragged last tile
    (1, 8, 12, 2, 4, 0),      # 16-token windows, ragged
    (1, 32, 32, 2, 16, 8),
    (1, 32, 48, 1, 16, 4),
    (1, 64, 64, 1, 32, 16),   # FlashSwin-T stage-1 window, shifted
    (2, 32, 32, 2, 32, 0),    # one window per image
    (1, 64, 64, 1, 64, 32),   # 4096-token window
    (1, 64, 96, 1, 32, 12),
    (1, 16, 16, 6, 8, 4),     # windows inside a tile with more heads than resident RoPE tables
    (1, 32, 32, 12, 32, 16),  # FlashSwin-T stage 3: one shifted window per image, 12 heads
    (1, 16, 16, 24, 16, 0),   # stage 4: the window is the grid, 24 heads
]


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", SMALL)
def test_fwd_bwd_parity(cfg):
    got, ref = run_both(*cfg)
    check("o", got["o"], ref["o"], FWD_TOL)
    check("lse", got["lse"], ref["lse"], FWD_TOL)
    for key in ("dq", "dk", "dv", "dtheta"):
        check(key, got[key], ref[key], GRAD_TOL)


# H or W not a multiple of M: the grid is padded with zero tokens (the Swin
# layer's padding), boxes run partly or wholly past the tokens in memory
PADDED = [  # (B, H, W, heads, M, s)
    (1, 20, 13, 2, 8, 4),     # windows inside a tile, shifted, both axes padded
    (2, 12, 18, 3, 8, 0),
    (1, 10, 6, 1, 4, 0),      # 16-token windows
    (1, 50, 83, 3, 8, 4),     # a detection-sized stage-2 grid (400 x 664 image / 8)
    (1, 40, 36, 2, 16, 8),    # one tile per window
    (1, 33, 20, 1, 16, 4),    # 1 real row in the last window row
    (1, 70, 50, 1, 32, 16),   # several tiles per window
    (1, 100, 70, 1, 64, 32),  # 4096-token windows
]


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", PADDED)
def test_padded_grid_parity(cfg):
    got, ref = run_both(*cfg)
    check("o", got["o"], ref["o"], FWD_TOL)
    check("lse", got["lse"], ref["lse"], FWD_TOL)
    for key in ("dq", "dk", "dv", "dtheta"):
        check(key, got[key], ref[key], GRAD_TOL)


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", [(1, 64, 64, 1, 32, 16), (2, 16, 16, 3, 8, 4), (1, 8, 12, 2, 4, 0),
                                 (1, 20, 13, 2, 8, 4), (1, 33, 20, 1, 16, 4)])
def test_sharp_softmax_parity(cfg):
    """Q, K scaled by 3 (the high-resolution stress recipe) sharpen the softmax:
    both kernel families, and padded grids."""
    got, ref = run_both(*cfg, qk_scale=3.0)
    check("o", got["o"], ref["o"], FWD_TOL)
    check("lse", got["lse"], ref["lse"], FWD_TOL)
    for key in ("dq", "dk", "dv", "dtheta"):
        check(key, got[key], ref[key], GRAD_TOL)


# Upstream gradients at the magnitudes of bf16 training (no loss scaling), and
# large ones: both kernel families, shifted, padded, and a sharpened softmax.
# dS = P o (dP - D) is held in fp16 for the dQ' and dK' products; unscaled, the
# small ones would land in fp16's subnormals or flush to zero, the large ones
# overflow.
GRAD_MAGNITUDE = [  # (B, H, W, heads, M, s, qk_scale)
    (2, 16, 16, 3, 8, 4, 1.0),
    (1, 8, 12, 2, 4, 0, 1.0),
    (1, 20, 13, 2, 8, 4, 1.0),    # padded
    (1, 32, 48, 1, 16, 4, 1.0),
    (1, 64, 64, 1, 32, 16, 1.0),
    (1, 70, 50, 1, 32, 16, 1.0),  # padded, several tiles per window
    (1, 64, 64, 1, 64, 32, 1.0),
    (2, 16, 16, 3, 8, 4, 3.0),    # sharpened softmax: P near 1
    (1, 64, 64, 1, 32, 16, 3.0),
]


@pytest.mark.gpu
@pytest.mark.parametrize("dout_scale", [2.0 ** -20, 2.0 ** -8, 2.0 ** 12], ids=["2^-20", "2^-8", "2^12"])
@pytest.mark.parametrize("cfg", GRAD_MAGNITUDE)
def test_gradient_magnitude_parity(cfg, dout_scale):
    *shape, qk = cfg
    got, ref = run_both(*shape, qk_scale=qk, dout_scale=dout_scale)
    for key in ("dq", "dk", "dv", "dtheta"):
        check(key, got[key], ref[key], GRAD_TOL)


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", [(2, 16, 16, 3, 8, 4), (1, 64, 64, 1, 32, 16), (1, 64, 64, 1, 64, 32)])
def test_gradient_scale_with_uneven_v(cfg):
    """v rows 2^24 apart in magnitude inside a window (the top half of the grid
    scaled down), with dO at 2^-20: the scaling of dS must bound dP - D by the
    largest v row that any output row mixes, not by the key rows of a tile."""
    B, H, W, h, M, s = cfg
    inp = make_inputs(B, H, W, h, 32)
    rows = torch.arange(H).view(1, H, 1, 1, 1)
    inp["v"] = torch.where(rows < H // 2, inp["v"] * 2.0 ** -24, inp["v"])
    dev = {k: v.cuda() for k, v in inp.items()}
    o, lse = ops.winattn_fwd(dev["q"], dev["k"], dev["v"], dev["theta"], M, s)
    scale = 2.0 ** -20
    got = ops.winattn_bwd(dev["q"], dev["k"], dev["v"], o, dev["dout"] * scale, lse, dev["theta"], M, s)
    torch.cuda.synchronize()
    ref = oracle.full(inp["q"], inp["k"], inp["v"], inp["theta"], M, s, dout=inp["dout"])
    for key, t in zip(("dq", "dk", "dv", "dtheta"), got):
        check(key, t.double() / scale, ref[key], GRAD_TOL)


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", [(1, 16, 16, 2, 8, 4), (1, 64, 64, 1, 32, 16), (1, 20, 13, 2, 8, 4),
                                 (1, 64, 64, 1, 64, 32)])
def test_large_qk_forward_parity(cfg):
    """q, k elements in the thousands (N(0, 1) draws times 1000; the rotated
    operands stay inside fp16's range, |q'|, |k'| < 65504), logits of order 1e6.
    With k = q every query's own key leads all others by about 1e6 in the logit,
    far above the ~1e3 that the fp16 rounding of q', k' moves a logit of that
    size, so the near one-hot softmax picks the same key on both sides.  (With
    independent q and k, rows whose two best logits lie within that rounding of
    each other may pick different keys in any bf16/fp16 attention: such a row is
    ill-conditioned, not computed wrongly.)"""
    B, H, W, h, M, s = cfg
    inp = make_inputs(B, H, W, h, 32, with_dout=False)
    inp["q"] = (inp["q"].float() * 1000.0).to(torch.bfloat16)
    inp["k"] = inp["q"].clone()
    dev = {k: v.cuda() for k, v in inp.items()}
    o, lse = ops.winattn_fwd(dev["q"], dev["k"], dev["v"], dev["theta"], M, s)
    torch.cuda.synchronize()
    ref = oracle.full(inp["q"], inp["k"], inp["v"], inp["theta"], M, s)
    assert float(inp["q"].float().abs().max()) > 1000.0 and float(ref["lse"].max()) > 1e6
    check("o", o, ref["o"], FWD_TOL)
    check("lse", lse, ref["lse"], FWD_TOL)


@pytest.mark.gpu
def test_empty_batch():
    inp = make_inputs(0, 16, 16, 2, 32)
    dev = {k: v.cuda() for k, v in inp.items()}
    o, lse = ops.winattn_fwd(dev["q"], dev["k"], dev["v"], dev["theta"], 8, 0)
    dth = torch.full_like(dev["theta"], 7.0)
    ops.winattn_bwd(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, dev["theta"], 8, 0, dtheta=dth)
    torch.cuda.synchronize()
    assert o.numel() == 0 and (dth == 0).all()


@pytest.mark.gpu
def test_forward_is_deterministic():
    inp = make_inputs(2, 32, 32, 2, 32)
    dev = {k: v.cuda() for k, v in inp.items()}
    o1, l1 = ops.winattn_fwd(dev["q"], dev["k"], dev["v"], dev["theta"], 16, 8)
    o2, l2 = ops.winattn_fwd(dev["q"], dev["k"], dev["v"], dev["theta"], 16, 8)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.gpu
def test_bounded_wait_reports_timeout_and_context_survives():
    stream = torch.cuda.current_stream().cuda_stream
    _lib.fs_selftest_bounded_wait(50_000_000, stream)
    torch.cuda.synchronize()
    code = _lib.fs_device_status()
    assert code >> 24 == _lib.FS_ERR_TIMEOUT and (code & 0xFFFFFF) == 0xABC
    got, ref = run_both(1, 16, 16, 2, 8, 0)  # the context is still usable
    check("o", got["o"], ref["o"], FWD_TOL)


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", [(2, 16, 16, 3, 8, 4), (1, 64, 64, 2, 32, 16)])
def test_backward_is_deterministic(cfg):
    """Two runs on the same inputs: every output bit for bit, except at M >= 16 dq,
    whose per-tile sums are reduce-added by several CTAs in any order, and d theta,
    whose query-side terms are taken from that dq (they agree to rounding)."""
    B, H, W, h, M, s = cfg
    inp = make_inputs(B, H, W, h, 32)
    dev = {k: v.cuda() for k, v in inp.items()}
    o, lse = ops.winattn_fwd(dev["q"], dev["k"], dev["v"], dev["theta"], M, s)
    a = ops.winattn_bwd(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, dev["theta"], M, s)
    b = ops.winattn_bwd(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, dev["theta"], M, s)
    torch.cuda.synchronize()
    names = ("dq", "dk", "dv", "dtheta")
    exact = names if M * M < 128 else ("dk", "dv")
    for name, x, y in zip(names, a, b):
        if name in exact:
            assert torch.equal(x, y), name
        else:
            check(name, x, y.float().cpu().numpy(), (1e-3, 1e-6))


@pytest.mark.gpu
def test_side_stream_gives_the_default_stream_results():
    """Work is enqueued on the caller's current stream."""
    inp = make_inputs(2, 32, 32, 2, 32)
    dev = {k: v.cuda() for k, v in inp.items()}
    o0, l0 = ops.winattn_fwd(dev["q"], dev["k"], dev["v"], dev["theta"], 8, 4)
    g0 = ops.winattn_bwd(dev["q"], dev["k"], dev["v"], o0, dev["dout"], l0, dev["theta"], 8, 4)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        o1, l1 = ops.winattn_fwd(dev["q"], dev["k"], dev["v"], dev["theta"], 8, 4)
        g1 = ops.winattn_bwd(dev["q"], dev["k"], dev["v"], o1, dev["dout"], l1, dev["theta"], 8, 4)
    side.synchronize()
    assert torch.equal(o0, o1) and torch.equal(l0, l1)
    for x, y in zip(g0, g1):
        assert torch.equal(x, y)


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", [(2, 16, 16, 3, 8, 4), (1, 64, 64, 2, 32, 16)])
def test_backward_ignores_stale_workspace_contents(cfg):
    """The caller's workspace may hold anything: a zeroed one, one with every
    byte 0xFF, and that one again as the previous call left it give the same
    gradients.  (The d theta reduction's per-head counters live there and are
    reset by the kernel that runs before it.)  dk, dv are bit-identical; dθ too
    at M = 8, and at M >= 16 within the last bits its query-side terms take from
    the unordered dQ' reduce-add."""
    B, H, W, h, M, s = cfg
    inp = make_inputs(B, H, W, h, 32)
    dev = {k: v.cuda() for k, v in inp.items()}
    o, lse = ops.winattn_fwd(dev["q"], dev["k"], dev["v"], dev["theta"], M, s)

    def bwd(ws):
        r = ops.winattn_bwd(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, dev["theta"], M, s, workspace=ws)
        torch.cuda.synchronize()
        return [t.clone() for t in r]

    ref = bwd(ops.alloc_workspace(dev["q"], M, s).fill_(0))
    ws = ops.alloc_workspace(dev["q"], M, s).fill_(0xFF)
    for got in (bwd(ws), bwd(ws)):
        assert torch.equal(got[1], ref[1]) and torch.equal(got[2], ref[2])  # dk, dv
        if M * M < 128:
            assert torch.equal(got[3], ref[3])
        else:
            assert torch.allclose(got[3], ref[3], rtol=1e-5, atol=1e-5)
