"""CPU checks of the kernels' window/box/tile geometry and work scheduling.

The kernels' own headers (geometry.cuh, schedule.cuh) are compiled for the host
with g++ and their output is checked against the oracle's definition of the
shifted windows (roll by -s, M x M windows, Swin region labels):
  * token slots cover every token of the grid, padded to multiples of M when
    H or W is not one, exactly once (slots of padding windows only at the end),
    and mark as real exactly the H x W tokens in memory;
  * in-window positions, labels and windows agree with the oracle's definition;
  * TMA boxes never straddle the wrap of the cyclic shift and stay inside the
    padded grid;
  * forward items visit exactly the (query tile, key tile) pairs that hold at
    least one attending token pair, every query tile once per head;
  * backward items visit the same pairs, every key tile once per head.
"""
import os
import subprocess
from collections import defaultdict

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "vision_transformer_windowed_b200", "csrc")
BIN = os.path.join(ROOT, "tests", "_build", "geometry_harness")


@pytest.fixture(scope="module")
def harness():
    os.makedirs(os.path.dirname(BIN), exist_ok=True)
    src = os.path.join(ROOT, "tests", "geometry_harness.cpp")
    subprocess.check_call(["g++", "-std=c++17", "-O1", "-D__host__=", "-D__device__=", "-I", CSRC, "-o", BIN, src])
    return BIN


def run(harness, shape):
    out = subprocess.check_output([harness, *map(str, shape)], text=True)
    return out.splitlines()


SHAPES = [  # (B, H, W, heads, d, M, s)
    (1, 16, 16, 2, 32, 8, 0),
    (2, 16, 16, 2, 32, 8, 4),
    (1, 8, 24, 1, 32, 8, 4),     # 3 windows: ragged last tile
    (1, 8, 12, 2, 32, 4, 0),     # 6 windows of 16 tokens: ragged
    (1, 32, 32, 2, 32, 16, 8),
    (1, 32, 48, 1, 32, 16, 4),
    (1, 64, 64, 1, 32, 32, 16),
    (2, 32, 32, 2, 32, 32, 0),
    (1, 64, 64, 1, 32, 64, 32),
    (1, 128, 64, 1, 32, 64, 0),
    (1, 64, 96, 1, 32, 32, 12),
    # H or W not a multiple of M: the grid is padded
    (1, 12, 20, 2, 32, 8, 4),
    (2, 20, 13, 2, 32, 8, 0),
    (1, 10, 6, 1, 32, 4, 0),
    (1, 40, 36, 1, 32, 16, 8),
    (1, 33, 20, 1, 32, 16, 4),
    (1, 70, 50, 1, 32, 32, 16),
    (1, 100, 70, 1, 32, 64, 32),
]


@pytest.mark.parametrize("shape", SHAPES)
def test_geometry_and_schedule(harness, shape):
    B, H, W, heads, d, M, s = shape
    lines = run(harness, shape)
    g = lines[0].split()
    N, BT, bpt, tiles, tpw, bh, bw, Hp, Wp = map(int, g[1:])
    assert (Hp, Wp) == (-(-H // M) * M, -(-W // M) * M)
    slots = np.array([list(map(int, l.split()[1:])) for l in lines if l[0] == "S"], dtype=np.int64)
    assert slots.shape[0] == tiles * 128
    valid = slots[:, 8] == 1          # slot of a real window (padded positions included)
    ntok = B * Hp * Wp
    assert valid.sum() == ntok
    assert valid[:ntok].all() and not valid[ntok:].any()
    v = slots[valid]
    b, row, col, i, j, lab, gw = (v[:, k] for k in range(1, 8))
    assert (row >= 0).all() and (row < Hp).all() and (col >= 0).all() and (col < Wp).all()
    tok = (b * Hp + row) * Wp + col
    assert np.unique(tok).size == ntok
    real = (row < H) & (col < W)
    assert (v[:, 9] == real).all() and (slots[~valid][:, 9] == 0).all()
    assert real.sum() == B * H * W
    r, c = (row - s) % Hp, (col - s) % Wp
    assert (i == r % M).all() and (j == c % M).all()
    labels = oracle.labels(Hp, Wp, M, s)
    assert (lab == labels[r, c]).all()
    nW = (Hp // M) * (Wp // M)
    assert (gw == b * nW + (r // M) * (Wp // M) + c // M).all()

    boxes = np.array([list(map(int, l.split()[1:])) for l in lines if l[0] == "X"], dtype=np.int64)
    bv = boxes[boxes[:, 4] == 1]
    # columns: box id, image, first row, first column, valid
    assert (bv[:, 2] >= 0).all() and (bv[:, 2] + bh <= Hp).all()
    assert (bv[:, 3] >= 0).all() and (bv[:, 3] + bw <= Wp).all()
    assert (bv[:, 1] < B).all()
    assert (boxes[boxes[:, 4] == 0][:, 1] >= B).all()  # padding boxes fall outside the tensor

    # tile pairs holding at least one attending (query, key) token pair
    seg = np.where(valid, slots[:, 7] * 9 + slots[:, 6], -1 - np.arange(slots.shape[0]))
    tile_of = np.arange(slots.shape[0]) // 128
    need = set()
    by_seg = defaultdict(set)
    for t, sg in zip(tile_of, seg):
        by_seg[sg].add(int(t))
    for ts in by_seg.values():
        for a in ts:
            for bb in ts:
                need.add((a, bb))
    for h in range(heads):
        fwd = [tuple(map(int, l.split()[3:5])) for l in lines if l[0] == "F" and int(l.split()[2]) == h]
        bwd = [tuple(map(int, l.split()[3:5])) for l in lines if l[0] == "B" and int(l.split()[2]) == h]
        assert len(fwd) == len(set(fwd)) and len(bwd) == len(set(bwd))
        assert set(fwd) == need, (sorted(set(fwd) ^ need))[:10]
        assert {(q, k) for k, q in bwd} == need
        # every query tile in exactly one forward item, every key tile in one backward item
        qitems = defaultdict(set)
        for l in lines:
            if l[0] == "F" and int(l.split()[2]) == h:
                qitems[int(l.split()[3])].add(int(l.split()[1]))
        assert all(len(x) == 1 for x in qitems.values()) and len(qitems) == tiles
        kitems = defaultdict(set)
        for l in lines:
            if l[0] == "B" and int(l.split()[2]) == h:
                kitems[int(l.split()[3])].add(int(l.split()[1]))
        assert all(len(x) == 1 for x in kitems.values()) and len(kitems) == tiles


def test_invariant_division_matches_hardware_divide(harness):
    """The 32-bit division by set-up constants used for window and item indices."""
    out = subprocess.run([harness, "D"], capture_output=True, text=True)
    tag, checked, bad = out.stdout.split()
    assert tag == "D" and int(checked) > 100000 and int(bad) == 0 and out.returncode == 0
