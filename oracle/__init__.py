"""fp64 CPU oracle for FlashSwin windowed-RoPE attention (test infrastructure).

TEST INFRASTRUCTURE ONLY: the product package never imports this module.  Only
``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may use it.  It shares no code with the CUDA library.

Two independent restatements of the same definition live here:

* ``fswin_oracle.c`` (wrapped below through ctypes): plain loops over
  (batch, window, head) units, one query row at a time, in double precision,
  threaded over units.  It is the oracle the GPU path is compared against.
* ``literal.py``: the same computation written with tensor-level torch float64
  ops (``torch.roll``, reshape into windows, complex multiplication for RoPE,
  the mask built from the Swin slice rule) and autograd for the gradients.  It
  exists to pin the C oracle, on tiny grids only.

Both also take an optional low-rank additive bias (the FlashBias-T variant of
the same pages: thelatestinai.com/papers/2610.04664, Table 2 and Table S1
captions, a trainable rank-16 bias factorization): per head, factors U, W of
shape [M*M, rank] over window-local positions t = i*M + j, and S_tu = scale
q'_t.k'_u + U_t.W_u for every window.

Both follow "FLASHSWIN: Unlocking Large Windows and Dense Tokens in Swin Vision
Transformers with Memory Efficient Attention" (arxivdaily.com/papers/2610.04664,
English abstract: exact softmax attention per M x M window, window-local
learnable 2D RoPE; thelatestinai.com/papers/2610.04664, Figure 1B and
Figure S4: theta_i = exp(omega_i) are inverse frequencies).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fswin_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libfswin_oracle.so")
_lock = threading.Lock()
_lib = None


class _Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "H", "W", "heads", "d", "M", "s")]


class _In(ctypes.Structure):
    _fields_ = [("p", ctypes.c_void_p), ("dtype", ctypes.c_int)]


class _Bias(ctypes.Structure):
    _fields_ = [("u", ctypes.c_void_p), ("w", ctypes.c_void_p), ("rank", ctypes.c_int)]


_BF16, _F64 = 0, 1


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc into ``oracle/_build`` (plain C, -O2)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            vp, P = ctypes.c_void_p, ctypes.POINTER(_Shape)
            lib.fso_units.restype = ctypes.c_int
            lib.fso_units.argtypes = [P, _In, _In, _In, _In, vp, _Bias, vp, ctypes.c_int64] + [vp] * 8 + [ctypes.c_int]
            lib.fso_full.restype = ctypes.c_int
            lib.fso_full.argtypes = [P, _In, _In, _In, _In, vp, _Bias] + [vp] * 8 + [ctypes.c_int]
            lib.fso_labels.restype = ctypes.c_int
            lib.fso_labels.argtypes = [ctypes.c_int] * 4 + [vp]
            _lib = lib
    return _lib


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def _as_input(x):
    """Accept bf16 torch tensors, uint16 bf16 bit arrays, or float arrays.

    Returns (numpy array kept alive, _In)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                x = x.view(torch.int16).numpy().view(np.uint16)
            else:
                x = x.to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return x, _In(x.ctypes.data, _BF16)
    x = np.ascontiguousarray(x, dtype=np.float64)
    return x, _In(x.ctypes.data, _F64)


def _theta64(theta):
    try:
        import torch
        if isinstance(theta, torch.Tensor):
            theta = theta.detach().cpu().to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(theta, dtype=np.float64)


def _dptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _bias_arg(bias, heads: int, N: int):
    """(kept-alive arrays, _Bias) for optional factors (u, w), each [heads, N, rank]."""
    if bias is None:
        return (), _Bias(None, None, 0), 0
    u, w = (_theta64(x) for x in bias)
    assert u.ndim == 3 and u.shape == w.shape and u.shape[:2] == (heads, N), (u.shape, w.shape)
    return (u, w), _Bias(u.ctypes.data, w.ctypes.data, u.shape[2]), u.shape[2]


def labels(H: int, W: int, M: int, s: int) -> np.ndarray:
    """Region label of every rolled token, [H, W] (0 everywhere when s == 0)."""
    out = np.zeros((H, W), dtype=np.int32)
    _load().fso_labels(H, W, M, s, out.ctypes.data_as(ctypes.c_void_p))
    return out


def full(q, k, v, theta, M: int, s: int, dout=None, nthreads: int | None = None, bias=None) -> dict:
    """Whole-tensor forward (and backward when ``dout`` is given).

    q, k, v, dout: [B, H, W, heads, d] (bf16 torch tensors or bit arrays are
    upcast exactly; float arrays are used as is).  theta: [heads, 2, d/4].
    Returns float64 arrays at original token positions: o, lse [B,H,W,heads]
    and, with dout, dq, dk, dv and dtheta [heads, 2, d/4].  H or W that is not
    a multiple of M is padded with zero tokens up to the next multiple (the
    Swin layer's padding); the windows, the shift and its mask then refer to
    the padded grid.  ``bias = (u, w)``, each [heads, M*M, rank], adds the
    low-rank bias u_t.w_u to every window's scores; the backward then also
    returns du and dw [heads, M*M, rank].
    """
    qa, qi = _as_input(q)
    ka, ki = _as_input(k)
    va, vi = _as_input(v)
    B, H, W, heads, d = qa.shape
    th = _theta64(theta)
    assert th.shape == (heads, 2, d // 4), th.shape
    sh = _Shape(B, H, W, heads, d, M, s)
    keep, bi, rank = _bias_arg(bias, heads, M * M)
    o = np.zeros((B, H, W, heads, d))
    lse = np.zeros((B, H, W, heads))
    res = {"o": o, "lse": lse}
    di = _In(None, 0)
    da = None
    grads = [None] * 6
    if dout is not None:
        da, di = _as_input(dout)
        grads = [np.zeros((B, H, W, heads, d)) for _ in range(3)] + [np.zeros((heads, 2, d // 4))]
        res.update(dq=grads[0], dk=grads[1], dv=grads[2], dtheta=grads[3])
        if rank:
            grads += [np.zeros((heads, M * M, rank)) for _ in range(2)]
            res.update(du=grads[4], dw=grads[5])
        else:
            grads += [None, None]
    st = _load().fso_full(ctypes.byref(sh), qi, ki, vi, di, _dptr(th), bi, _dptr(o), _dptr(lse),
                          *[_dptr(g) for g in grads], int(nthreads or default_threads()))
    if st:
        raise ValueError(f"oracle rejected the problem (status {st})")
    del qa, ka, va, da, keep
    return res


def units(q, k, v, theta, M: int, s: int, unit_ids, dout=None, nthreads: int | None = None, bias=None) -> dict:
    """Forward (and backward with ``dout``) for selected (batch, window, head) units.

    unit = (b * nW + w) * heads + h, windows w = wr * (Wp/M) + wc in the rolled
    frame of the padded grid (Hp, Wp = H, W rounded up to multiples of M).
    Outputs are per unit in window-local token order t = i*M + j, padded tokens
    included:
    o, dq, dk, dv [n, M*M, d]; lse [n, M*M]; dtheta [n, 2, d/4] (the unit's share);
    with ``bias = (u, w)`` also du, dw [n, M*M, rank] (the unit's shares).
    """
    qa, qi = _as_input(q)
    ka, ki = _as_input(k)
    va, vi = _as_input(v)
    B, H, W, heads, d = qa.shape
    th = _theta64(theta)
    uid = np.ascontiguousarray(np.asarray(unit_ids, dtype=np.int64))
    n = uid.shape[0]
    N = M * M
    sh = _Shape(B, H, W, heads, d, M, s)
    keep, bi, rank = _bias_arg(bias, heads, N)
    o = np.zeros((n, N, d))
    lse = np.zeros((n, N))
    res = {"o": o, "lse": lse}
    di = _In(None, 0)
    da = None
    grads = [None] * 6
    if dout is not None:
        da, di = _as_input(dout)
        grads = [np.zeros((n, N, d)) for _ in range(3)] + [np.zeros((n, 2, d // 4))]
        res.update(dq=grads[0], dk=grads[1], dv=grads[2], dtheta=grads[3])
        if rank:
            grads += [np.zeros((n, N, rank)) for _ in range(2)]
            res.update(du=grads[4], dw=grads[5])
        else:
            grads += [None, None]
    st = _load().fso_units(ctypes.byref(sh), qi, ki, vi, di, _dptr(th), bi, _dptr(uid), ctypes.c_int64(n),
                           _dptr(o), _dptr(lse), *[_dptr(g) for g in grads],
                           int(nthreads or default_threads()))
    if st:
        raise ValueError(f"oracle rejected the problem (status {st})")
    del qa, ka, va, da, keep
    return res


def unit_token_positions(H: int, W: int, M: int, s: int, unit: int, heads: int):
    """Original (b, row, col, head) of every token of a unit, in window-local order.

    Positions of padded tokens (grids that are not multiples of M) have
    row >= H or col >= W."""
    Hp, Wp = -(-H // M) * M, -(-W // M) * M
    nWw = Wp // M
    nW = (Hp // M) * nWw
    b, rem = divmod(unit, nW * heads)
    w, h = divmod(rem, heads)
    wr, wc = divmod(w, nWw)
    t = np.arange(M * M)
    rows = (wr * M + t // M + s) % Hp
    cols = (wc * M + t % M + s) % Wp
    return b, rows, cols, h
