"""GPU parity of the low-rank additive bias kernels against the fp64 oracle.

The bias is the FlashBias-T variant (thelatestinai.com/papers/2610.04664,
Table 2 and Table S1 captions: a trainable rank-16 bias factorization).  The
small shape lists of the 32-channel parity tests run element by element (every
window size, shifted and not, ragged tiles, padded grids), with RoPE and
without it (theta = None on the GPU, theta = 0 for the oracle: the identity
rotation), plus upstream gradients at training magnitudes compared at unit scale,
a sharpened softmax, and full-size FlashBias-T stage shapes on sampled windows
(du and dw through dO kept on the sampled windows only: the other windows'
shares are then zero, so the totals are the sampled units' sums).
"""
import numpy as np
import pytest
import torch

import oracle
from vision_transformer_windowed_b200 import _lib, ops
from vision_transformer_windowed_b200.inputs import make_bias, make_inputs

FWD_TOL = (1e-2, 2e-3)
GRAD_TOL = (3e-2, 5e-3)
D = 32


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


def run_both(B, H, W, h, M, s, rope=True, qk_scale=1.0, dout_scale=1.0, bias_std=0.5):
    inp = make_inputs(B, H, W, h, D, qk_scale=qk_scale)
    bias = make_bias(h, M, std=bias_std)
    theta = inp["theta"] if rope else torch.zeros_like(inp["theta"])
    dev = {k: v.cuda() for k, v in inp.items()}
    u, w = bias["u"].cuda(), bias["w"].cuda()
    th = dev["theta"] if rope else None
    o, lse = ops.winattn_lrbias_fwd(dev["q"], dev["k"], dev["v"], th, u, w, M, s)
    dout = dev["dout"] * dout_scale if dout_scale != 1.0 else dev["dout"]
    dq, dk, dv, dth, du, dw = ops.winattn_lrbias_bwd(dev["q"], dev["k"], dev["v"], o, dout, lse, th, u, w, M, s)
    torch.cuda.synchronize()
    grads = {"dq": dq, "dk": dk, "dv": dv, "du": du, "dw": dw}
    if rope:
        grads["dtheta"] = dth
    else:
        assert dth is None
    if dout_scale != 1.0:
        grads = {k: t.double() / dout_scale for k, t in grads.items()}
    ref = oracle.full(inp["q"], inp["k"], inp["v"], theta, M, s, dout=inp["dout"], bias=(bias["u"], bias["w"]))
    return {"o": o, "lse": lse, **grads}, ref


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

PADDED = [  # H or W not a multiple of M: padded with zero tokens (the bias still applies there)
    (1, 20, 13, 2, 8, 4),
    (2, 12, 18, 3, 8, 0),
    (1, 10, 6, 1, 4, 0),
    (1, 50, 83, 3, 8, 4),
    (1, 40, 36, 2, 16, 8),
    (1, 70, 50, 1, 32, 16),
    (1, 100, 70, 1, 64, 32),
]


def _compare(got, ref, keys=("dq", "dk", "dv", "du", "dw", "dtheta")):
    check("o", got["o"], ref["o"], FWD_TOL)
    check("lse", got["lse"], ref["lse"], FWD_TOL)
    for key in keys:
        if key in got:
            check(key, got[key], ref[key], GRAD_TOL)


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", SMALL + PADDED)
def test_lrbias_parity_with_rope(cfg):
    _compare(*run_both(*cfg))


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", [(2, 16, 16, 3, 8, 4), (1, 8, 12, 2, 4, 0), (1, 32, 48, 1, 16, 4),
                                 (1, 64, 64, 1, 32, 16), (1, 64, 64, 1, 64, 32), (1, 70, 50, 1, 32, 16)])
def test_lrbias_parity_without_rope(cfg):
    _compare(*run_both(*cfg, rope=False))


@pytest.mark.gpu
@pytest.mark.parametrize("dout_scale", [2.0 ** -20, 2.0 ** 12], ids=["2^-20", "2^12"])
@pytest.mark.parametrize("cfg", [(2, 16, 16, 3, 8, 4), (1, 20, 13, 2, 8, 4), (1, 64, 64, 1, 32, 16)])
def test_lrbias_gradient_magnitude_parity(cfg, dout_scale):
    got, ref = run_both(*cfg, dout_scale=dout_scale)
    for key in ("dq", "dk", "dv", "du", "dw", "dtheta"):
        check(key, got[key], ref[key], GRAD_TOL)


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", [(2, 16, 16, 3, 8, 4), (1, 64, 64, 1, 32, 16)])
def test_lrbias_sharp_softmax_parity(cfg):
    """Q, K x 3 and a bias twice as wide: peaked rows."""
    _compare(*run_both(*cfg, qk_scale=3.0, bias_std=0.5 * 2 ** 0.5))


@pytest.mark.gpu
def test_lrbias_inference_forward_and_determinism():
    """lse = NULL gives the same O; dk, dv and dw are bit-identical from run to
    run (each key row's sums stay in one CTA; dW's window sum has a fixed
    order).  dq, du and the query side of dtheta come from fp32 reductions
    whose order varies: they agree to rounding."""
    inp = make_inputs(2, 64, 64, 2, D)
    bias = make_bias(2, 32)
    dev = {k: v.cuda() for k, v in inp.items()}
    u, w = bias["u"].cuda(), bias["w"].cuda()
    o, lse = ops.winattn_lrbias_fwd(dev["q"], dev["k"], dev["v"], dev["theta"], u, w, 32, 16)
    o2, none = ops.winattn_lrbias_fwd(dev["q"], dev["k"], dev["v"], dev["theta"], u, w, 32, 16, need_lse=False)
    assert none is None and torch.equal(o, o2)
    r1 = ops.winattn_lrbias_bwd(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, dev["theta"], u, w, 32, 16)
    r2 = ops.winattn_lrbias_bwd(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, dev["theta"], u, w, 32, 16)
    torch.cuda.synchronize()
    for i in (1, 2, 5):  # dk, dv, dw
        assert torch.equal(r1[i], r2[i])
    # dq (bf16): one rounding step apart at most, or fp32 summation-order noise
    # where a sum cancels to near zero
    a, b = r1[0].float(), r2[0].float()
    assert ((a - b).abs() <= a.abs() * 2.0 ** -7 + 1e-5 * a.abs().max()).all()
    for i in (3, 4):  # dtheta, du (fp32)
        scale = r1[i].abs().max()
        assert (r1[i] - r2[i]).abs().max() <= 1e-5 * scale


@pytest.mark.gpu
def test_lrbias_autograd_wrapper():
    inp = make_inputs(1, 32, 32, 2, D)
    bias = make_bias(2, 16)
    leaves = {k: v.cuda().requires_grad_(k != "dout") for k, v in inp.items()}
    u, w = (bias[k].cuda().requires_grad_(True) for k in ("u", "w"))
    o = ops.window_attention_lrbias(leaves["q"], leaves["k"], leaves["v"], leaves["theta"], u, w, 16, 8)
    (o.float() * leaves["dout"].float()).sum().backward()
    ref = oracle.full(inp["q"], inp["k"], inp["v"], inp["theta"], 16, 8, dout=inp["dout"], bias=(bias["u"], bias["w"]))
    for key, t in (("dq", leaves["q"]), ("dk", leaves["k"]), ("dv", leaves["v"]), ("dtheta", leaves["theta"]),
                   ("du", u), ("dw", w)):
        check(key, t.grad, ref[key], GRAD_TOL)


@pytest.mark.gpu
def test_lrbias_empty_batch_zeroes_parameter_gradients():
    inp = make_inputs(0, 16, 16, 2, D)
    bias = make_bias(2, 8)
    dev = {k: v.cuda() for k, v in inp.items()}
    u, w = bias["u"].cuda(), bias["w"].cuda()
    o, lse = ops.winattn_lrbias_fwd(dev["q"], dev["k"], dev["v"], dev["theta"], u, w, 8, 0)
    _, _, _, dth, du, dw = ops.winattn_lrbias_bwd(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, dev["theta"],
                                                  u, w, 8, 0)
    torch.cuda.synchronize()
    assert o.numel() == 0 and (dth == 0).all() and (du == 0).all() and (dw == 0).all()


def _sample_units(B, H, W, heads, M, n_random=5, seed=11):
    nWh, nWw = -(-H // M), -(-W // M)
    nW = nWh * nWw
    picks = {(0, 0, 0), (B - 1, nWh - 1, nWw - 1), (0, nWh - 1, 0), (B // 2, 0, nWw - 1)}
    rng = np.random.default_rng(seed)
    for _ in range(n_random):
        picks.add((int(rng.integers(B)), int(rng.integers(nWh)), int(rng.integers(nWw))))
    hs = range(heads) if heads <= 3 else (0, heads // 2, heads - 1)
    return np.array(sorted((b * nW + wr * nWw + wc) * heads + h for b, wr, wc in picks for h in hs),
                    dtype=np.int64)


# FlashBias-T stage shapes at the benchmark's sizes (Table S1: batch 128 at 256 x 256,
# p = 2 gives the 128 x 128 stage-1 grid; p = 4 the 64 x 64 grid at M = 8)
FULL = [
    ("flashbias_t_stage1_p2_m32_s16", 128, 128, 128, 3, 32, 16),
    ("flashbias_t_stage1_p2_m32_s0", 128, 128, 128, 3, 32, 0),
    ("flashbias_t_stage1_p4_m8_s4", 128, 64, 64, 3, 8, 4),
    # the later FlashSwin-T stages at p = 2: more heads, the window covering the grid
    ("flashbias_t_stage3_p2_m32_s16", 128, 32, 32, 12, 32, 16),
    ("flashbias_t_stage4_p2_m16_s0", 128, 16, 16, 24, 16, 0),
]


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", FULL, ids=[c[0] for c in FULL])
def test_lrbias_full_size_sampled_windows(cfg):
    name, B, H, W, heads, M, s = cfg
    inp = make_inputs(B, H, W, heads, D)
    bias = make_bias(heads, M)
    units = _sample_units(B, H, W, heads, M)
    pos = []
    for uid in units:
        b, rows, cols, h = oracle.unit_token_positions(H, W, M, s, int(uid), heads)
        pos.append((b, rows, cols, h))
    keep = torch.zeros((B, H, W, heads), dtype=torch.bool)
    for b, rows, cols, h in pos:
        keep[b, torch.from_numpy(rows), torch.from_numpy(cols), h] = True
    dout = torch.where(keep[..., None], inp["dout"], torch.zeros((), dtype=inp["dout"].dtype))
    dev = {k: v.cuda() for k, v in inp.items() if k != "dout"}
    u, w = bias["u"].cuda(), bias["w"].cuda()
    o, lse = ops.winattn_lrbias_fwd(dev["q"], dev["k"], dev["v"], dev["theta"], u, w, M, s)
    dq, dk, dv, dth, du, dw = ops.winattn_lrbias_bwd(dev["q"], dev["k"], dev["v"], o, dout.cuda(), lse,
                                                     dev["theta"], u, w, M, s)
    torch.cuda.synchronize()
    bt = (bias["u"], bias["w"])
    ref = oracle.units(inp["q"], inp["k"], inp["v"], inp["theta"], M, s, units, dout=dout, bias=bt)
    idx = lambda t, b, rows, cols, h: t[b, torch.from_numpy(rows), torch.from_numpy(cols), h]
    cat = np.concatenate
    got = {k: [] for k in ("o", "lse", "dq", "dk", "dv")}
    want = {k: [] for k in got}
    for n, (b, rows, cols, h) in enumerate(pos):
        for key, t in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
            got[key].append(idx(t, b, rows, cols, h).float().cpu().numpy())
            want[key].append(ref[key][n])
    check(f"{name} o", cat(got["o"]), cat(want["o"]), FWD_TOL)
    check(f"{name} lse", cat(got["lse"]), cat(want["lse"]), FWD_TOL)
    for key in ("dq", "dk", "dv"):
        check(f"{name} {key}", cat(got[key]), cat(want[key]), GRAD_TOL)
    want_th = np.zeros((heads, 2, D // 4))
    want_du = np.zeros((heads, M * M, 16))
    want_dw = np.zeros((heads, M * M, 16))
    for n, uid in enumerate(units):
        h = int(uid) % heads
        want_th[h] += ref["dtheta"][n]
        want_du[h] += ref["du"][n]
        want_dw[h] += ref["dw"][n]
    check(f"{name} dtheta", dth, want_th, GRAD_TOL)
    check(f"{name} du", du, want_du, GRAD_TOL)
    check(f"{name} dw", dw, want_dw, GRAD_TOL)
