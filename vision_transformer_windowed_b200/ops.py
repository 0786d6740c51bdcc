"""Torch-facing wrappers of the C ABI: they allocate outputs with PyTorch, pass
raw device pointers and the current CUDA stream, and nothing else.  Every step
of the attention runs in the CUDA kernels of libfswin.so.

Method: FlashSwin ("FLASHSWIN: Unlocking Large Windows and Dense Tokens in Swin
Vision Transformers with Memory Efficient Attention", thelatestinai.com/papers/
2610.04664, Figure 1B): exact windowed softmax attention with window-local
learnable 2D RoPE, the fused FlashAttention-style kernel replacing Swin's
materialised score matrix.

Shapes: q, k, v [B, H, W, heads, d] bf16 with d = 32 or 64, H >= M and W >= M.  H or W
need not be a multiple of the window M: the grid is then worked on padded at
the bottom and right with zero tokens to the next multiple (the Swin layer's
padding), and only the H x W real tokens are read and written.
"""
from __future__ import annotations

import torch

from . import _lib

HEAD_DIM = 32


def _shape(q: torch.Tensor, M: int, s: int) -> _lib.Shape:
    if q.dim() != 5:
        raise ValueError("expected a [B, H, W, heads, d] tensor")
    B, H, W, heads, d = q.shape
    return _lib.make_shape(B, H, W, heads, d, M, s)


def _check_tensor(name: str, t: torch.Tensor, shape, dtype) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def winattn_fwd(q, k, v, theta, M: int, s: int, o=None, lse=None, need_lse: bool = True, workspace=None):
    """O, LSE = fused windowed-RoPE attention forward (bf16 in/out, fp32 LSE).

    need_lse=False (and no lse buffer): inference forward, O only; LSE is returned as None.
    workspace (the backward's, from alloc_workspace): the training forward, which
    also leaves the rotated q', k' tiles there for winattn_bwd(..., after_train_fwd=True)."""
    sh = _shape(q, M, s)
    B, H, W, heads, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_tensor(name, t, q.shape, torch.bfloat16)
    _check_tensor("theta", theta, (heads, 2, d // 4), torch.float32)
    if o is None:
        o = torch.empty_like(q)
    if lse is None and need_lse:
        lse = torch.empty((B, H, W, heads), device=q.device, dtype=torch.float32)
    _check_tensor("o", o, q.shape, torch.bfloat16)
    if lse is not None:
        _check_tensor("lse", lse, (B, H, W, heads), torch.float32)
    if workspace is not None:
        if lse is None:
            raise ValueError("the training forward writes lse")
        _lib.fs_winattn_fwd_train(sh, q.data_ptr(), k.data_ptr(), v.data_ptr(), theta.data_ptr(), o.data_ptr(),
                                  lse.data_ptr(), workspace.data_ptr(), workspace.numel(), _stream(q.device))
        return o, lse
    _lib.fs_winattn_fwd(sh, q.data_ptr(), k.data_ptr(), v.data_ptr(), theta.data_ptr(), o.data_ptr(),
                        lse.data_ptr() if lse is not None else 0, _stream(q.device))
    return o, lse


def winattn_block_fwd(x, w_qkv, b_qkv, w_o, b_o, theta, M: int, s: int, heads: int, y=None):
    """y = windowed-RoPE attention of (x W_qkv^T + b_qkv) per head, then W_o, b_o
    (the attention block of a Swin layer, inference; M*M < 128, heads <= 3)."""
    B, H, W, C = x.shape
    d = C // heads
    sh = _lib.make_shape(B, H, W, heads, d, M, s)
    _check_tensor("x", x, (B, H, W, C), torch.bfloat16)
    _check_tensor("w_qkv", w_qkv, (3 * C, C), torch.bfloat16)
    _check_tensor("b_qkv", b_qkv, (3 * C,), torch.float32)
    _check_tensor("w_o", w_o, (C, C), torch.bfloat16)
    _check_tensor("b_o", b_o, (C,), torch.float32)
    _check_tensor("theta", theta, (heads, 2, d // 4), torch.float32)
    if y is None:
        y = torch.empty_like(x)
    _check_tensor("y", y, (B, H, W, C), torch.bfloat16)
    _lib.fs_winattn_block_fwd(sh, x.data_ptr(), w_qkv.data_ptr(), b_qkv.data_ptr(), w_o.data_ptr(), b_o.data_ptr(),
                              theta.data_ptr(), y.data_ptr(), _stream(x.device))
    return y


def bwd_workspace_bytes(B: int, H: int, W: int, heads: int, M: int, s: int, d: int = HEAD_DIM) -> int:
    return _lib.fs_winattn_bwd_workspace_bytes(_lib.make_shape(B, H, W, heads, d, M, s))


def alloc_workspace(q: torch.Tensor, M: int, s: int) -> torch.Tensor:
    n = _lib.fs_winattn_bwd_workspace_bytes(_shape(q, M, s))
    return torch.empty(max(n, 256), device=q.device, dtype=torch.uint8)


def winattn_bwd(q, k, v, o, dout, lse, theta, M: int, s: int, workspace=None, dq=None, dk=None, dv=None,
                dtheta=None, after_train_fwd: bool = False):
    """dQ, dK, dV, dtheta of sum(O * dout) (recompute-based backward).

    after_train_fwd: `workspace` is the one a training forward (winattn_fwd with
    that workspace) of the same q, k, theta filled, unchanged since; its rotated
    q', k' tiles are reused."""
    sh = _shape(q, M, s)
    B, H, W, heads, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _check_tensor(name, t, q.shape, torch.bfloat16)
    _check_tensor("lse", lse, (B, H, W, heads), torch.float32)
    _check_tensor("theta", theta, (heads, 2, d // 4), torch.float32)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    dtheta = torch.empty_like(theta) if dtheta is None else dtheta
    if workspace is None:
        if after_train_fwd:
            raise ValueError("after_train_fwd needs the training forward's workspace")
        workspace = alloc_workspace(q, M, s)
    call = _lib.fs_winattn_bwd_train if after_train_fwd else _lib.fs_winattn_bwd
    call(sh, q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(), lse.data_ptr(),
         theta.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), dtheta.data_ptr(),
         workspace.data_ptr(), workspace.numel(), _stream(q.device))
    return dq, dk, dv, dtheta


class WindowAttentionRoPE(torch.autograd.Function):
    """Autograd wrapper: forward and backward both run in libfswin.so.

    theta are the inverse frequencies; with the log parameterisation of the
    paper (theta = exp(omega), thelatestinai.com/papers/2610.04664, Figure S4)
    autograd through ``torch.exp`` gives d omega = theta * d theta.
    """

    @staticmethod
    def forward(ctx, q, k, v, theta, M: int, s: int, reuse_rotated: bool = False):
        # reuse_rotated: the training pair, whose forward leaves the rotated q', k'
        # tiles in the backward's workspace; the workspace (about 262 bytes per
        # token-head) then stays allocated until the backward, beside the saved
        # q, k, v, o (256 bytes per token-head)
        ws = alloc_workspace(q, M, s) if reuse_rotated else None
        o, lse = winattn_fwd(q, k, v, theta, M, s, workspace=ws)
        ctx.save_for_backward(q, k, v, o, lse, theta, *(() if ws is None else (ws,)))
        ctx.M, ctx.s, ctx.reuse = M, s, reuse_rotated
        return o

    @staticmethod
    def backward(ctx, dout):
        q, k, v, o, lse, theta, *ws = ctx.saved_tensors
        dq, dk, dv, dth = winattn_bwd(q, k, v, o, dout.contiguous(), lse, theta, ctx.M, ctx.s,
                                      workspace=ws[0] if ctx.reuse else None, after_train_fwd=ctx.reuse)
        return dq, dk, dv, dth, None, None, None


def window_attention(q, k, v, theta, M: int, s: int, reuse_rotated: bool = False):
    """Autograd windowed-RoPE attention.  reuse_rotated=True runs the training
    pair (faster at windows of >= 128 tokens; keeps the backward's workspace
    from the forward to the backward)."""
    return WindowAttentionRoPE.apply(q, k, v, theta, M, s, reuse_rotated)


# ------------------------------------------------------------ low-rank bias
# The FlashBias-T variant of the same pages (thelatestinai.com/papers/2610.04664,
# Table 2 and Table S1 captions): a trainable rank-16 factorization U_h W_h^T of
# an additive bias over window-local positions, shared by every window and added
# to the scaled scores before the shift mask.  Heads of 32 channels; theta may be
# None (no rotation).
LRBIAS_RANK = 16


def _check_factors(q, u, w, M: int) -> None:
    heads = q.shape[3]
    for name, t in (("u", u), ("w", w)):
        _check_tensor(name, t, (heads, M * M, LRBIAS_RANK), torch.float32)


def winattn_lrbias_fwd(q, k, v, theta, u, w, M: int, s: int, o=None, lse=None, need_lse: bool = True):
    """O, LSE of windowed attention with the low-rank bias u_t . w_u (bf16 in/out, fp32 LSE)."""
    sh = _shape(q, M, s)
    B, H, W, heads, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_tensor(name, t, q.shape, torch.bfloat16)
    if theta is not None:
        _check_tensor("theta", theta, (heads, 2, d // 4), torch.float32)
    _check_factors(q, u, w, M)
    if o is None:
        o = torch.empty_like(q)
    if lse is None and need_lse:
        lse = torch.empty((B, H, W, heads), device=q.device, dtype=torch.float32)
    _check_tensor("o", o, q.shape, torch.bfloat16)
    if lse is not None:
        _check_tensor("lse", lse, (B, H, W, heads), torch.float32)
    _lib.fs_winattn_lrbias_fwd(sh, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                               theta.data_ptr() if theta is not None else 0, u.data_ptr(), w.data_ptr(),
                               LRBIAS_RANK, o.data_ptr(), lse.data_ptr() if lse is not None else 0,
                               _stream(q.device))
    return o, lse


def alloc_lrbias_workspace(q: torch.Tensor, M: int, s: int) -> torch.Tensor:
    n = _lib.fs_winattn_lrbias_bwd_workspace_bytes(_shape(q, M, s))
    return torch.empty(max(n, 256), device=q.device, dtype=torch.uint8)


def winattn_lrbias_bwd(q, k, v, o, dout, lse, theta, u, w, M: int, s: int, workspace=None, dq=None, dk=None,
                       dv=None, dtheta=None, du=None, dw=None):
    """dQ, dK, dV, dtheta (None without theta), dU, dW of sum(O * dout)."""
    sh = _shape(q, M, s)
    B, H, W, heads, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _check_tensor(name, t, q.shape, torch.bfloat16)
    _check_tensor("lse", lse, (B, H, W, heads), torch.float32)
    if theta is not None:
        _check_tensor("theta", theta, (heads, 2, d // 4), torch.float32)
    _check_factors(q, u, w, M)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    dtheta = (torch.empty_like(theta) if dtheta is None else dtheta) if theta is not None else None
    du = torch.empty_like(u) if du is None else du
    dw = torch.empty_like(w) if dw is None else dw
    for name, t, ref in (("dq", dq, q), ("dk", dk, q), ("dv", dv, q), ("du", du, u), ("dw", dw, w)):
        _check_tensor(name, t, ref.shape, ref.dtype)
    if dtheta is not None:
        _check_tensor("dtheta", dtheta, theta.shape, torch.float32)
    if workspace is None:
        workspace = alloc_lrbias_workspace(q, M, s)
    _lib.fs_winattn_lrbias_bwd(sh, q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(),
                               lse.data_ptr(), theta.data_ptr() if theta is not None else 0, u.data_ptr(),
                               w.data_ptr(), LRBIAS_RANK, dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                               dtheta.data_ptr() if dtheta is not None else 0, du.data_ptr(), dw.data_ptr(),
                               workspace.data_ptr(), workspace.numel(), _stream(q.device))
    return dq, dk, dv, dtheta, du, dw


class WindowAttentionLowRankBias(torch.autograd.Function):
    """Autograd wrapper of the low-rank-bias attention (forward and backward in libfswin.so)."""

    @staticmethod
    def forward(ctx, q, k, v, theta, u, w, M: int, s: int):
        o, lse = winattn_lrbias_fwd(q, k, v, theta, u, w, M, s)
        ctx.save_for_backward(q, k, v, o, lse, u, w, *(() if theta is None else (theta,)))
        ctx.M, ctx.s, ctx.has_theta = M, s, theta is not None
        return o

    @staticmethod
    def backward(ctx, dout):
        q, k, v, o, lse, u, w, *rest = ctx.saved_tensors
        theta = rest[0] if ctx.has_theta else None
        dq, dk, dv, dth, du, dw = winattn_lrbias_bwd(q, k, v, o, dout.contiguous(), lse, theta, u, w, ctx.M, ctx.s)
        return dq, dk, dv, dth, du, dw, None, None


def window_attention_lrbias(q, k, v, theta, u, w, M: int, s: int):
    return WindowAttentionLowRankBias.apply(q, k, v, theta, u, w, M, s)
