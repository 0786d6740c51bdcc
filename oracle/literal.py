"""Tensor-level restatement of windowed-RoPE attention in torch float64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  Used on tiny grids to
pin the C oracle: it shares no arithmetic with it.  The cyclic shift is
``torch.roll``, windows come from a reshape, RoPE is a multiplication of
channel pairs viewed as complex numbers, the shift mask is built with the Swin
slice rule, softmax is ``torch.softmax`` and the gradients come from autograd.
A grid that is not a multiple of M is zero-padded with
``torch.nn.functional.pad`` before the roll and cropped after it, as a Swin
layer does.

The optional low-rank bias (FlashBias-T, thelatestinai.com/papers/2610.04664,
Table 2 and Table S1 captions) is the per-head matrix product U_h W_h^T over
window-local positions, broadcast to every window and added to the scaled
scores before the mask.

Method: "FLASHSWIN ..." (arxivdaily.com/papers/2610.04664, English abstract:
exact softmax attention inside each M x M window, window-local learnable 2D
RoPE); the mask slices [0, H-M), [H-M, H-s), [H-s, H) are the Swin shifted-
window rule.
"""
from __future__ import annotations

import math

import torch
import torch.nn.functional as F


def region_labels(H: int, W: int, M: int, s: int) -> torch.Tensor:
    """Swin's shifted-window region map: each (row-slice, column-slice) cell of
    the rolled grid gets its own counter value, row slices outermost."""
    img = torch.zeros(H, W, dtype=torch.int64)
    if s == 0:
        return img
    cnt = 0
    for hs in (slice(0, H - M), slice(H - M, H - s), slice(H - s, H)):
        for ws in (slice(0, W - M), slice(W - M, W - s), slice(W - s, W)):
            img[hs, ws] = cnt
            cnt += 1
    return img


def _windows(x: torch.Tensor, M: int) -> torch.Tensor:
    """[B, H, W, h, d] -> [B, nWh, nWw, h, M*M, d] (token t = i*M + j)."""
    B, H, W, h, d = x.shape
    x = x.reshape(B, H // M, M, W // M, M, h, d)
    x = x.permute(0, 1, 3, 5, 2, 4, 6)
    return x.reshape(B, H // M, W // M, h, M * M, d)


def _unwindows(x: torch.Tensor, H: int, W: int, M: int) -> torch.Tensor:
    B, nh, nw, h, N, d = x.shape
    x = x.reshape(B, nh, nw, h, M, M, d).permute(0, 1, 4, 2, 5, 3, 6)
    return x.reshape(B, H, W, h, d)


def rope(x: torch.Tensor, theta: torch.Tensor, pos_i: torch.Tensor, pos_j: torch.Tensor) -> torch.Tensor:
    """Rotate pairs (2k, 2k+1) of the first half by pos_j * theta[h, 0, k] and of
    the second half by pos_i * theta[h, 1, k]; x: [..., h, N, d], positions [N]."""
    d = x.shape[-1]
    half = d // 2
    out = []
    for ax, pos in ((0, pos_j), (1, pos_i)):
        part = x[..., ax * half:(ax + 1) * half]
        z = torch.view_as_complex(part.reshape(*part.shape[:-1], half // 2, 2).contiguous())
        ang = pos.to(torch.float64)[:, None] * theta[:, ax, :][:, None, :]   # [h, N, d/4]
        z = z * torch.polar(torch.ones_like(ang), ang)
        out.append(torch.view_as_real(z).reshape(part.shape))
    return torch.cat(out, dim=-1)


def forward(q, k, v, theta, M: int, s: int, bias=None):
    """Returns (o [B,H,W,h,d], lse [B,H,W,h]) in float64; bias = (u, w), each
    [h, M*M, rank], adds u @ w^T to every window's scores."""
    B, H0, W0, h, d = q.shape
    H, W = -(-H0 // M) * M, -(-W0 // M) * M
    q, k, v = (F.pad(t, (0, 0, 0, 0, 0, W - W0, 0, H - H0)) for t in (q, k, v))
    shifted = [torch.roll(t, shifts=(-s, -s), dims=(1, 2)) for t in (q, k, v)]
    qw, kw, vw = (_windows(t, M) for t in shifted)
    t = torch.arange(M * M)
    pos_i, pos_j = t // M, t % M
    qr = rope(qw, theta, pos_i, pos_j)
    kr = rope(kw, theta, pos_i, pos_j)
    scores = (qr @ kr.transpose(-1, -2)) / math.sqrt(d)          # [B,nh,nw,h,N,N]
    if bias is not None:
        scores = scores + bias[0] @ bias[1].transpose(-1, -2)     # [h,N,N] broadcast over windows
    lab = _windows(region_labels(H, W, M, s)[None, :, :, None, None], M)[..., 0]  # [1,nh,nw,1,N]
    allowed = lab[..., :, None] == lab[..., None, :]
    scores = scores.masked_fill(~allowed, float("-inf"))
    lse = torch.logsumexp(scores, dim=-1)
    o = torch.softmax(scores, dim=-1) @ vw
    o = torch.roll(_unwindows(o, H, W, M), shifts=(s, s), dims=(1, 2))
    lse = torch.roll(_unwindows(lse[..., None], H, W, M)[..., 0], shifts=(s, s), dims=(1, 2))
    return o[:, :H0, :W0], lse[:, :H0, :W0]


def forward_backward(q, k, v, theta, M: int, s: int, dout, bias=None):
    """Forward plus autograd gradients of sum(o * dout) w.r.t. q, k, v, theta
    (and the bias factors u, w when given)."""
    tensors = (q, k, v, theta) + (tuple(bias) if bias is not None else ())
    leaves = [torch.as_tensor(t).detach().to(torch.float64).clone().requires_grad_(True) for t in tensors]
    o, lse = forward(*leaves[:4], M, s, bias=leaves[4:] if bias is not None else None)
    (o * dout.to(torch.float64)).sum().backward()
    dq, dk, dv, dth = (t.grad for t in leaves[:4])
    res = {"o": o.detach(), "lse": lse.detach(), "dq": dq, "dk": dk, "dv": dv, "dtheta": dth}
    if bias is not None:
        res.update(du=leaves[4].grad, dw=leaves[5].grad)
    return res
