"""GPU parity at the full sizes of the workloads, on sampled windows.

The whole problem runs on the GPU exactly as the benchmark runs it; the fp64
oracle then computes a sample of (image, window, head) units one by one, and
the sampled tokens of O, LSE, dQ, dK, dV are compared.  The sample always
holds windows of the last window row and column (the only ones the shift mask
cuts) and of the first.  dθ sums over every token, so it is checked through a
property that holds at any size: with dO zero outside the sampled units, the
other units contribute nothing, and dθ equals the sum of the sampled units'
shares.  Grids that are not multiples of M (a detection-sized input) are
compared at their real tokens; the padded ones exist only inside the kernels.
"""
import numpy as np
import pytest
import torch

import oracle
from vision_transformer_windowed_b200 import ops
from vision_transformer_windowed_b200.inputs import make_inputs

FWD_TOL = (1e-2, 2e-3)
GRAD_TOL = (3e-2, 5e-3)

# (name, B, H, W, heads, M, s, qk_scale[, dout_scale]): the benchmark workloads
# and the FlashSwin-T stage shapes at 256 x 256 input with patch 2; with a
# dout_scale (a power of two) the GPU gets dO times it, and its gradients,
# divided by it, are compared with the oracle's at scale 1 (upstream gradients
# at the magnitudes of bf16 training, compared at their unit scale)
FULL = [
    ("swin_t_stage1_p4_m8_s0", 128, 64, 64, 3, 8, 0, 1.0),
    ("swin_t_stage1_p4_m8_s4", 128, 64, 64, 3, 8, 4, 1.0),
    ("swin_t_stage1_p4_m8_s4_dout2^-20", 128, 64, 64, 3, 8, 4, 1.0, 2.0 ** -20),
    ("flashswin_t_stage1_p2_m32_s0", 128, 128, 128, 3, 32, 0, 1.0),
    ("flashswin_t_stage1_p2_m32", 128, 128, 128, 3, 32, 16, 1.0),
    ("flashswin_t_stage1_p2_m32_dout2^-20", 128, 128, 128, 3, 32, 16, 1.0, 2.0 ** -20),
    ("flashswin_t_stage2_p2_m32_s0", 128, 64, 64, 6, 32, 0, 1.0),
    ("flashswin_t_stage2_p2_m32_s16", 128, 64, 64, 6, 32, 16, 1.0),
    ("flashswin_t_stage3_p2_m32_s0", 128, 32, 32, 12, 32, 0, 1.0),
    ("flashswin_t_stage3_p2_m32_s16", 128, 32, 32, 12, 32, 16, 1.0),
    ("flashswin_t_stage4_p2_m16", 128, 16, 16, 24, 16, 0, 1.0),
    ("highres_p2_m32", 16, 256, 256, 3, 32, 16, 3.0),
    ("highres_p2_m64", 16, 256, 256, 3, 64, 32, 3.0),
    # an 800 x 1333 detection input at p=4: a 200 x 334 grid, padded per window size
    ("swin_t_det_stage1_p4_m8_s4", 16, 200, 334, 3, 8, 4, 1.0),
    ("flashswin_t_det_stage1_p4_m32_s16", 16, 200, 334, 3, 32, 16, 1.0),
]


def _check(name, got, ref, tol):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, name
    assert np.isfinite(got).all(), f"{name}: non-finite values"
    err = np.abs(got - ref).max()
    bound = tol[0] * np.abs(ref).max() + tol[1]
    assert err <= bound, f"{name}: max|err| {err:.4g} > {bound:.4g}"


def _sample_units(B, H, W, heads, M, n_random=6, seed=7):
    nWh, nWw = -(-H // M), -(-W // M)  # windows of the padded grid
    nW = nWh * nWw
    picks = {(0, 0, 0), (B - 1, nWh - 1, nWw - 1), (0, nWh - 1, 0), (0, 0, nWw - 1), (B // 2, nWh - 1, nWw // 2)}
    rng = np.random.default_rng(seed)
    for _ in range(n_random):
        picks.add((int(rng.integers(B)), int(rng.integers(nWh)), int(rng.integers(nWw))))
    units = []
    for b, wr, wc in sorted(picks):
        for h in range(heads) if heads <= 3 else (0, heads // 2, heads - 1):
            units.append((b * nW + wr * nWw + wc) * heads + h)
    return np.array(sorted(set(units)), dtype=np.int64)


# heads of 64 channels (the wide kernels) at the benchmark's d = 64 workload and a
# detection-sized padded grid: (name, B, H, W, heads, M, s, qk_scale)
FULL64 = [
    ("flashswin_stage1_p2_m32_d64", 64, 128, 128, 3, 32, 16, 1.0),
    ("det_stage1_p4_m8_d64_s4", 16, 200, 334, 3, 8, 4, 1.0),
]


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", FULL, ids=[c[0] for c in FULL])
def test_full_size_sampled_windows(cfg):
    _full_size(*cfg[:8], dscale=cfg[8] if len(cfg) > 8 else 1.0)


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", FULL64, ids=[c[0] for c in FULL64])
def test_full_size_sampled_windows_d64(cfg):
    _full_size(*cfg, d=64)


# the four-stage step's blocks through the training pair, as the benchmark runs them
# (the forward reads the rotated q', k' tiles it left in the backward's workspace)
TRAIN = [c for c in FULL if c[0].startswith("flashswin_t_stage")]


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", TRAIN, ids=[c[0] + "_train" for c in TRAIN])
def test_full_size_sampled_windows_training_pair(cfg):
    _full_size(*cfg[:8], dscale=cfg[8] if len(cfg) > 8 else 1.0, train=True)


def _full_size(name, B, H, W, heads, M, s, qk, dscale=1.0, d=32, train=False):
    inp = make_inputs(B, H, W, heads, d, qk_scale=qk)
    units = _sample_units(B, H, W, heads, M)
    pos = []
    for u in units:  # real tokens of each unit, and their window-local slots
        b, rows, cols, h = oracle.unit_token_positions(H, W, M, s, int(u), heads)
        real = (rows < H) & (cols < W)
        pos.append((b, rows[real], cols[real], h, real))
    # dO kept on the sampled units' tokens only
    keep = torch.zeros((B, H, W, heads), dtype=torch.bool)
    for b, rows, cols, h, _ in pos:
        keep[b, torch.from_numpy(rows), torch.from_numpy(cols), h] = True
    dout = torch.where(keep[..., None], inp["dout"], torch.zeros((), dtype=inp["dout"].dtype))

    dev = {k: v.cuda() for k, v in inp.items() if k != "dout"}
    ws = ops.alloc_workspace(dev["q"], M, s) if train else None
    o, lse = ops.winattn_fwd(dev["q"], dev["k"], dev["v"], dev["theta"], M, s, workspace=ws)
    dq, dk, dv, dth = ops.winattn_bwd(dev["q"], dev["k"], dev["v"], o, dout.cuda() * dscale, lse, dev["theta"], M, s,
                                      workspace=ws, after_train_fwd=train)
    torch.cuda.synchronize()
    if dscale != 1.0:
        dq, dk, dv, dth = (t.double() / dscale for t in (dq, dk, dv, dth))

    ref = oracle.units(inp["q"], inp["k"], inp["v"], inp["theta"], M, s, units, dout=dout)
    idx = lambda t, b, rows, cols, h: t[b, torch.from_numpy(rows), torch.from_numpy(cols), h]
    got = {k: [] for k in ("o", "lse", "dq", "dk", "dv")}
    want = {k: [] for k in got}
    for n, (b, rows, cols, h, real) in enumerate(pos):
        for key, t in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
            got[key].append(idx(t, b, rows, cols, h).float().cpu().numpy())
            want[key].append(ref[key][n][real])
    cat = np.concatenate
    _check(f"{name} o", cat(got["o"]), cat(want["o"]), FWD_TOL)
    _check(f"{name} lse", cat(got["lse"]), cat(want["lse"]), FWD_TOL)
    for key in ("dq", "dk", "dv"):
        _check(f"{name} {key}", cat(got[key]), cat(want[key]), GRAD_TOL)
    # dθ: only the sampled units carry dO, so the total is their sum
    want_th = np.zeros((heads, 2, d // 4))
    for u, share in zip(units, ref["dtheta"]):
        want_th[int(u) % heads] += share
    _check(f"{name} dtheta", dth.float().cpu().numpy(), want_th, GRAD_TOL)
