"""Host-side checks of the C ABI: the library loads, exports every entry point
declared in include/fswin.h, and validates arguments without launching work
(these calls return before touching any device)."""
import ctypes
import os
import re

import pytest
import torch

from vision_transformer_windowed_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "fswin.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fs_[a-z_0-9]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    names = _declared_functions()
    assert "fs_winattn_fwd" in names and "fs_winattn_bwd" in names
    for n in names:
        assert hasattr(lib, n), n
        assert ctypes.cast(getattr(lib, n), ctypes.c_void_p).value


def test_status_strings():
    for code, name in enumerate(_lib.STATUS_NAMES):
        assert _lib.status_string(code).startswith(name)


GOOD = [(1, 16, 16, 2, 32, 8, 0), (128, 64, 64, 3, 32, 8, 4), (128, 128, 128, 3, 32, 32, 16),
        (16, 256, 256, 3, 32, 64, 32), (128, 16, 16, 24, 32, 16, 0), (0, 16, 16, 2, 32, 8, 0),
        (2, 8, 24, 1, 32, 4, 0), (1, 32, 32, 1, 32, 32, 0),
        # H or W not a multiple of M: padded to the next multiple
        (1, 20, 16, 2, 32, 8, 0), (1, 16, 20, 2, 32, 8, 4), (2, 200, 334, 3, 32, 8, 4),
        (1, 33, 17, 1, 32, 16, 8), (1, 65, 100, 1, 32, 64, 32),
        (1, 16, 16, 2, 64, 8, 4), (1, 64, 64, 1, 64, 32, 16), (1, 20, 13, 2, 64, 8, 4)]
BAD = [(1, 16, 16, 2, 48, 8, 0),    # d not 32 or 64
       (1, 16, 16, 2, 16, 8, 0),
       (1, 16, 16, 2, 32, 12, 0),   # M not supported
       (1, 7, 16, 2, 32, 8, 0),     # H < M
       (1, 16, 15, 2, 32, 16, 0),   # W < M
       (1, 16, 16, 2, 32, 8, 8),    # s >= M
       (1, 16, 16, 2, 32, 8, 2),    # s % 4
       (1, 16, 16, 2, 32, 8, -4),   # s < 0
       (-1, 16, 16, 2, 32, 8, 0),   # B < 0
       (1, 16, 16, 0, 32, 8, 0),    # heads
       (1, 4, 4, 1, 32, 8, 0)]      # grid smaller than a window


@pytest.mark.parametrize("shape", GOOD)
def test_supported_shapes(shape):
    assert _lib.fs_winattn_check_shape(_lib.make_shape(*shape)) == _lib.FS_OK


@pytest.mark.parametrize("shape", BAD)
def test_rejected_shapes(shape):
    sh = _lib.make_shape(*shape)
    assert _lib.fs_winattn_check_shape(sh) == _lib.FS_ERR_SHAPE
    assert _lib.fs_winattn_bwd_workspace_bytes(sh) == 0
    with pytest.raises(_lib.FswinError) as e:
        _lib.fs_winattn_fwd(sh, 16, 16, 16, 16, 16, 16, 0)
    assert e.value.status == _lib.FS_ERR_SHAPE


def test_null_and_alignment_rejected_before_launch():
    sh = _lib.make_shape(1, 16, 16, 2, 32, 8, 0)
    with pytest.raises(_lib.FswinError) as e:
        _lib.fs_winattn_fwd(sh, 0, 16, 16, 16, 16, 16, 0)
    assert e.value.status == _lib.FS_ERR_NULL
    with pytest.raises(_lib.FswinError) as e:
        _lib.fs_winattn_fwd(sh, 24, 16, 16, 16, 16, 16, 0)
    assert e.value.status == _lib.FS_ERR_ALIGN
    n = _lib.fs_winattn_bwd_workspace_bytes(sh)
    with pytest.raises(_lib.FswinError) as e:
        _lib.fs_winattn_bwd(sh, *([256] * 11), 256, n - 1, 0)
    assert e.value.status == _lib.FS_ERR_WORKSPACE
    with pytest.raises(_lib.FswinError) as e:
        _lib.fs_winattn_bwd(sh, *([256] * 11), 128, n, 0)   # misaligned workspace
    assert e.value.status == _lib.FS_ERR_WORKSPACE
    with pytest.raises(_lib.FswinError) as e:
        _lib.fs_winattn_bwd(sh, *([256] * 10), 0, 256, n, 0)  # dtheta NULL
    assert e.value.status == _lib.FS_ERR_NULL


def test_workspace_flat_in_window_size():
    """Backward scratch depends on the token count only, not on M (memory flat in M)."""
    a = _lib.fs_winattn_bwd_workspace_bytes(_lib.make_shape(16, 256, 256, 3, 32, 32, 16))
    b = _lib.fs_winattn_bwd_workspace_bytes(_lib.make_shape(16, 256, 256, 3, 32, 64, 32))
    c = _lib.fs_winattn_bwd_workspace_bytes(_lib.make_shape(16, 256, 256, 3, 32, 8, 4))
    assert a == b == c > 0
    # and linear in the number of tokens, up to a fixed per-head part (the d theta
    # reduction's second level: heads x 64 x 16 floats)
    d = _lib.fs_winattn_bwd_workspace_bytes(_lib.make_shape(32, 256, 256, 3, 32, 32, 16))
    assert abs(d - 2 * a) <= 3 * 64 * 16 * 4 + 4096


def test_padded_grid_workspace_is_that_of_the_padded_grid():
    """A grid that is not a multiple of M is worked on padded: the backward
    scratch is that of the padded grid."""
    ws = _lib.fs_winattn_bwd_workspace_bytes
    assert ws(_lib.make_shape(2, 200, 334, 3, 32, 8, 4)) == ws(_lib.make_shape(2, 200, 336, 3, 32, 8, 4))
    assert ws(_lib.make_shape(1, 33, 17, 1, 32, 16, 8)) == ws(_lib.make_shape(1, 48, 32, 1, 32, 16, 8))
    assert ws(_lib.make_shape(1, 20, 16, 2, 32, 8, 0)) == ws(_lib.make_shape(1, 24, 16, 2, 32, 8, 0))


@pytest.mark.skipif(torch.cuda.is_available(), reason="would launch on the placeholder pointers")
def test_inference_forward_takes_a_null_lse():
    """lse may be NULL (inference forward): the call passes argument checking and,
    with no GPU here, stops at the device check."""
    sh = _lib.make_shape(1, 16, 16, 2, 32, 8, 0)
    with pytest.raises(_lib.FswinError) as e:
        _lib.fs_winattn_fwd(sh, 16, 16, 16, 16, 16, 0, 0)
    assert e.value.status not in (_lib.FS_ERR_NULL, _lib.FS_ERR_ALIGN, _lib.FS_ERR_SHAPE)


def test_block_forward_rejects_before_launch():
    """Windows inside one tile and at most three heads; NULL and misaligned pointers."""
    def call(shape, *ptrs):
        with pytest.raises(_lib.FswinError) as e:
            _lib.fs_winattn_block_fwd(_lib.make_shape(*shape), *ptrs, 0)
        return e.value.status
    ok = [16] * 7
    assert call((1, 32, 32, 3, 32, 16, 0), *ok) == _lib.FS_ERR_SHAPE   # 256-token windows
    assert call((1, 16, 16, 4, 32, 8, 0), *ok) == _lib.FS_ERR_SHAPE    # four heads
    assert call((1, 16, 16, 3, 32, 8, 0), 0, *ok[1:]) == _lib.FS_ERR_NULL
    assert call((1, 16, 16, 3, 32, 8, 0), 24, *ok[1:]) == _lib.FS_ERR_ALIGN


def test_workspace_flat_in_window_size_at_d64():
    """64-channel heads: the backward scratch depends on the token count only."""
    a = _lib.fs_winattn_bwd_workspace_bytes(_lib.make_shape(16, 256, 256, 3, 64, 32, 16))
    b = _lib.fs_winattn_bwd_workspace_bytes(_lib.make_shape(16, 256, 256, 3, 64, 64, 32))
    c = _lib.fs_winattn_bwd_workspace_bytes(_lib.make_shape(16, 256, 256, 3, 64, 8, 4))
    assert a == b == c > 0


def test_lrbias_entry_points_reject_before_launch():
    """Low-rank bias: d = 32 and rank 16 only; NULL factors, gradients and
    misaligned pointers; theta without dtheta; a short workspace."""
    good = _lib.make_shape(1, 16, 16, 2, 32, 8, 4)
    n = _lib.fs_winattn_lrbias_bwd_workspace_bytes(good)
    assert n > 0
    assert _lib.fs_winattn_lrbias_bwd_workspace_bytes(_lib.make_shape(1, 16, 16, 2, 64, 8, 4)) == 0

    def fwd(shape, *a):
        with pytest.raises(_lib.FswinError) as e:
            _lib.fs_winattn_lrbias_fwd(shape, *a, 0)
        return e.value.status

    p = 256
    #              q  k  v  theta u  w  rank o  lse
    assert fwd(_lib.make_shape(1, 16, 16, 2, 64, 8, 4), p, p, p, p, p, p, 16, p, p) == _lib.FS_ERR_SHAPE
    assert fwd(good, p, p, p, p, p, p, 8, p, p) == _lib.FS_ERR_SHAPE
    assert fwd(good, p, p, p, p, 0, p, 16, p, p) == _lib.FS_ERR_NULL
    assert fwd(good, p, p, p, p, p + 4, p, 16, p, p) == _lib.FS_ERR_ALIGN

    def bwd(shape, dtheta=p, du=p, ws=p, nbytes=n, theta=p, rank=16):
        with pytest.raises(_lib.FswinError) as e:
            _lib.fs_winattn_lrbias_bwd(shape, p, p, p, p, p, p, theta, p, p, rank, p, p, p, dtheta, du, p, ws,
                                       nbytes, 0)
        return e.value.status

    assert bwd(good, rank=32) == _lib.FS_ERR_SHAPE
    assert bwd(good, dtheta=0) == _lib.FS_ERR_NULL      # theta given, dtheta NULL
    assert bwd(good, du=0) == _lib.FS_ERR_NULL
    assert bwd(good, du=p + 8) == _lib.FS_ERR_ALIGN
    assert bwd(good, nbytes=n - 1) == _lib.FS_ERR_WORKSPACE
    assert bwd(good, ws=p + 16) == _lib.FS_ERR_WORKSPACE


def test_lrbias_workspace_size():
    """The bias backward's scratch: 256 B of accumulator rows and 8 B of lse2 and
    D per token-head (on the padded grid), the fp16 factor rows (64 B per head
    and window position), 8 x 16 fp32 d theta partials and the norms per (head,
    tile), a fixed d theta part, and one [head][window slot][32] fp32 block per
    16 windows for the first level of the dU / dW sum."""
    B, H, W, heads, M = 4, 64, 64, 3, 16
    n = _lib.fs_winattn_lrbias_bwd_workspace_bytes(_lib.make_shape(B, H, W, heads, 32, M, 8))
    tokens = B * H * W * heads
    wins = B * (H // M) * (W // M)
    chunks = -(-wins // 16)
    tiles = B * H * W // 128
    expect = tokens * (256 + 8) + heads * M * M * 64 + heads * tiles * 8 + heads * tiles * 8 * 16 * 4 + \
        heads * 64 * 16 * 4 + heads * 4 + \
        chunks * heads * M * M * 32 * 4
    assert expect <= n <= expect + 8 * 256


def test_train_pair_rejects_before_launch():
    """The training forward needs lse and the backward's workspace."""
    sh = _lib.make_shape(1, 64, 64, 2, 32, 32, 16)
    n = _lib.fs_winattn_bwd_workspace_bytes(sh)
    p = 256

    def fwd(lse=p, ws=p, nbytes=n):
        with pytest.raises(_lib.FswinError) as e:
            _lib.fs_winattn_fwd_train(sh, p, p, p, p, p, lse, ws, nbytes, 0)
        return e.value.status

    assert fwd(lse=0) == _lib.FS_ERR_NULL
    assert fwd(ws=0) == _lib.FS_ERR_WORKSPACE
    assert fwd(ws=p + 16) == _lib.FS_ERR_WORKSPACE
    assert fwd(nbytes=n - 1) == _lib.FS_ERR_WORKSPACE
    with pytest.raises(_lib.FswinError) as e:
        _lib.fs_winattn_bwd_train(sh, *([p] * 11), p, n - 1, 0)
    assert e.value.status == _lib.FS_ERR_WORKSPACE
