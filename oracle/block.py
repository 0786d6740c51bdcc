"""fp64 oracle of the window-attention block of a Swin layer (test infrastructure).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle``: the product package
never imports it.

The block around FlashSwin's attention (thelatestinai.com/papers/2610.04664,
Figure 1B: the attention module of each FlashSwin block) is the Swin layer's
qkv linear map, the windowed RoPE attention per head, and the output linear
map.  Written out as that definition:

    qkv = x W_qkv^T + b_qkv          x [B, H, W, C], W_qkv [3C, C], C = heads * d
    q, k, v = qkv split in (3, heads, d) along the channels
    o = windowed-RoPE attention of (q, k, v) per head, as in ``oracle.full``
    y = o W_o^T + b_o                o flattened to [B, H, W, C], W_o [C, C]

The projections are fp64 matrix products (a library primitive); the attention
is the C oracle.  The shift needs no separate handling: the projections act
token by token, so they commute with the cyclic roll of the windows.  A grid
that is not a multiple of M is padded as a Swin layer pads it: x gets zero
tokens up to the next multiple of M before the qkv map (so padded q, k, v
equal the bias), attention runs on the padded grid, and y is cropped.
"""
from __future__ import annotations

import numpy as np

from . import full


def _f64(a):
    try:
        import torch
        if isinstance(a, torch.Tensor):
            return a.detach().cpu().to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(a, dtype=np.float64)


def project_qkv(x, w_qkv, b_qkv, heads: int):
    """q, k, v [B, H, W, heads, d] (float64) of the block's input x."""
    x, w, b = _f64(x), _f64(w_qkv), _f64(b_qkv)
    B, H, W, C = x.shape
    d = C // heads
    qkv = x @ w.T + b  # [B, H, W, 3C]
    qkv = qkv.reshape(B, H, W, 3, heads, d)
    return qkv[..., 0, :, :], qkv[..., 1, :, :], qkv[..., 2, :, :]


def block_forward(x, w_qkv, b_qkv, w_o, b_o, theta, M: int, s: int, heads: int, nthreads: int | None = None):
    """y [B, H, W, C] (float64) of the attention block; also returns the attention output o."""
    x = _f64(x)
    B, H, W, C = x.shape
    Hp, Wp = -(-H // M) * M, -(-W // M) * M
    xp = np.zeros((B, Hp, Wp, C))
    xp[:, :H, :W] = x
    q, k, v = project_qkv(xp, w_qkv, b_qkv, heads)
    o = full(q, k, v, theta, M, s, nthreads=nthreads)["o"][:, :H, :W]  # [B, H, W, heads, d]
    of = o.reshape(B, H, W, -1)
    return of @ _f64(w_o).T + _f64(b_o), o


def block_backward(x, w_qkv, b_qkv, w_o, b_o, theta, M: int, s: int, heads: int, dy, nthreads: int | None = None):
    """Gradients of sum(y * dy) for the block's output y, dy [B, H, W, C]:
    dict of dx [B, H, W, C], dw_qkv [3C, C], db_qkv [3C], dw_o [C, C], db_o [C]
    and dtheta [heads, 2, d/4], all float64.

    The chain rule through the block's three steps in reverse order: the output
    map (dW_o = sum over tokens of dy^T o, db_o = sum of dy, do = dy W_o), the
    attention backward of ``oracle.full`` with do as its upstream gradient, and
    the qkv map (dqkv = [dq, dk, dv] in the channel order of the forward split,
    dW_qkv = sum over tokens of dqkv^T x, db_qkv = sum of dqkv, dx = dqkv W_qkv).
    On a padded grid the padding tokens' outputs are cropped, so their dy is 0;
    their q, k, v (the bias) still take part in the attention, so their dqkv
    reaches db_qkv, while x is 0 there and dx is cropped.
    """
    x, dy = _f64(x), _f64(dy)
    w_qkv, w_o = _f64(w_qkv), _f64(w_o)
    B, H, W, C = x.shape
    d = C // heads
    Hp, Wp = -(-H // M) * M, -(-W // M) * M
    xp = np.zeros((B, Hp, Wp, C))
    xp[:, :H, :W] = x
    dyp = np.zeros((B, Hp, Wp, C))
    dyp[:, :H, :W] = dy
    q, k, v = project_qkv(xp, w_qkv, b_qkv, heads)
    dop = (dyp @ w_o).reshape(B, Hp, Wp, heads, d)
    att = full(q, k, v, theta, M, s, dout=dop, nthreads=nthreads)
    o = att["o"].reshape(B, Hp, Wp, C)
    dqkv = np.stack([att["dq"], att["dk"], att["dv"]], axis=3).reshape(B, Hp, Wp, 3 * C)
    return {
        "dx": (dqkv @ w_qkv)[:, :H, :W],
        "dw_qkv": dqkv.reshape(-1, 3 * C).T @ xp.reshape(-1, C),
        "db_qkv": dqkv.reshape(-1, 3 * C).sum(axis=0),
        "dw_o": dyp.reshape(-1, C).T @ o.reshape(-1, C),
        "db_o": dyp.reshape(-1, C).sum(axis=0),
        "dtheta": att["dtheta"],
    }
