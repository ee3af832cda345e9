"""User-facing PyTorch entry points over the C ABI.

``triangle_attention(q, k, v, bias, mask=None, scale=None, orientation="start")``
returns the BF16 output and is differentiable in q, k, v and bias.  The
forward saves (o, resid, lse) -- the BF16 output, its BF16 rounding residual
and the FP32 log-sum-exp -- and the backward consumes exactly that state.

Orientation: for triangle attention around the ending node, pass the pair
tensors as stored (``[B,N,N,H,d]`` in the pair frame); this module hands the
kernels transposed views (axes 1 and 2 swapped, i.e. swapped strides), so no
data is copied.  bias and mask are in the attention's own frame.

PyTorch supplies device memory and streams only; all arithmetic runs in the
library's kernels.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import _binding as B


def _frame(x: torch.Tensor, orientation: str) -> torch.Tensor:
    if orientation == "start":
        return x
    if orientation == "end":
        return x.transpose(1, 2)
    raise ValueError("orientation must be 'start' or 'end'")


def forward(q, k, v, bias, mask=None, scale: Optional[float] = None, stream=None):
    """Attention-frame forward.  Returns (o, resid, lse); o and resid get q's
    strides (``empty_like`` keeps a dense layout's strides), so ending-node
    outputs come back in the caller's storage frame."""
    Bn, N, _, H, d = q.shape
    o = torch.empty_like(q)
    resid = torch.empty_like(q)
    lse = torch.empty((Bn, H, N, N), dtype=torch.float32, device=q.device)
    B.tri_attn_fwd(q, k, v, bias, mask, o, resid, lse, 0.0 if scale is None else scale, stream)
    return o, resid, lse


def backward(q, k, v, bias, mask, o, resid, lse, dout, scale: Optional[float] = None,
             flags: int = 0, workspace: Optional[torch.Tensor] = None, stream=None):
    """Attention-frame backward.  Returns (dq, dk, dv, dbias)."""
    Bn, N, _, H, d = q.shape
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    # rows padded to a multiple of 8 elements (the ABI wants 16-byte aligned row strides)
    Npad = (N + 7) // 8 * 8
    dbias = torch.empty((Bn, H, N, Npad), dtype=torch.bfloat16, device=q.device)[..., :N]
    need = B.tri_attn_bwd_workspace_bytes(Bn, N, H, d)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    B.tri_attn_bwd(q, k, v, bias, mask, o, resid, lse, dout, dq, dk, dv, dbias, workspace,
                   0.0 if scale is None else scale, flags, stream)
    return dq, dk, dv, dbias


def _abi_layout(t: torch.Tensor) -> torch.Tensor:
    """t itself if the C ABI accepts its layout (innermost stride 1, other strides
    non-negative multiples of 8 elements, 16-byte aligned data), else a dense copy
    (e.g. the stride-0 gradient that ``out.sum().backward()`` hands over)."""
    st = t.stride()
    ok = st[-1] == 1 and all(s >= 0 and s % 8 == 0 for s in st[:-1]) and t.data_ptr() % 16 == 0
    return t if ok else t.contiguous()


class TriangleAttentionFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, bias, mask, scale, orientation):
        qf, kf, vf = (_frame(x, orientation) for x in (q, k, v))
        o, resid, lse = forward(qf, kf, vf, bias, mask, scale)
        ctx.save_for_backward(qf, kf, vf, bias, mask if mask is not None else torch.empty(0), o, resid, lse)
        ctx.has_mask = mask is not None
        ctx.scale = scale
        ctx.orientation = orientation
        return _frame(o, orientation)

    @staticmethod
    def backward(ctx, grad_out):
        qf, kf, vf, bias, mask, o, resid, lse = ctx.saved_tensors
        mask = mask if ctx.has_mask else None
        g = _frame(_abi_layout(grad_out.to(torch.bfloat16)), ctx.orientation)
        dq, dk, dv, dbias = backward(qf, kf, vf, bias, mask, o, resid, lse, g, ctx.scale)
        f = lambda x: _frame(x, ctx.orientation)
        return f(dq), f(dk), f(dv), dbias, None, None, None


def triangle_attention(q, k, v, bias, mask=None, scale: Optional[float] = None, orientation: str = "start"):
    """Differentiable triangle attention (BF16 in/out) on a B200."""
    return TriangleAttentionFunction.apply(q, k, v, bias, mask, scale, orientation)
