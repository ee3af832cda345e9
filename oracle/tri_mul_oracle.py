"""FP64 CPU oracle for the contraction at the heart of the triangle
multiplicative update -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The product path (the C-ABI library and
its Python binding) never imports, links or executes anything under
``oracle/``; the two share no code.

What it computes.  The pages name the Triangle Multiplicative Update as the
second operation TurboPairFormer optimises beside triangle attention
("16张H100，训练步提速1.73倍：TurboPairFormer…", biocloudservice.com, opening
paragraph; "TurboPairFormer: более быстрое…", dev48.org, the paragraph that
introduces TurboPairFormer), without a formula.  The plain reading is the
AlphaFold-style update, whose only cubic-cost step is a per-channel contraction
of two projected pair tensors over the third residue k:

    outgoing edges:  x[b,c,i,j] = sum_k a[b,c,i,k] * b[b,c,j,k]
    incoming edges:  x[b,c,i,j] = sum_k a[b,c,k,i] * b[b,c,k,j]

with a, b, x held channel-first ([B, C, N, N]; the model's projections,
gates and LayerNorms around this step are elementwise or per-position and off
the cubic path).  The backward of the contraction, for the upstream gradient
dx:

    outgoing:  da[i,k] = sum_j dx[i,j] b[j,k]     db[j,k] = sum_i dx[i,j] a[i,k]
    incoming:  da[k,i] = sum_j dx[i,j] b[k,j]     db[k,j] = sum_i dx[i,j] a[k,i]

Every step is one FP64 matrix product per (b, c) (a library matmul), with no
blocking, fusion or reordering beyond the definitions above.  Pinned by
``tests/test_tri_mul_oracle_pins.py`` against explicit loops, closed forms,
the incoming/outgoing transpose relation, finite differences and torch
autograd.
"""
from __future__ import annotations

import numpy as np

ORIENTATIONS = ("outgoing", "incoming")


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def fwd(a, b, orientation: str = "outgoing", planted: int = 0):
    """x = the contraction of a and b over k for every (batch, channel).

    ``planted`` introduces a known mistake (1: contract over the wrong index of
    b, 2: drop the last k) so the pins can show they catch it."""
    a, b = _f64(a), _f64(b)
    if orientation == "outgoing":
        bb = b if planted != 1 else np.swapaxes(b, -1, -2)
        if planted == 2:
            return a[..., :-1] @ np.swapaxes(bb[..., :-1], -1, -2)
        return a @ np.swapaxes(bb, -1, -2)          # x[i,j] = sum_k a[i,k] b[j,k]
    if orientation == "incoming":
        return np.swapaxes(a, -1, -2) @ b          # x[i,j] = sum_k a[k,i] b[k,j]
    raise ValueError(orientation)


def bwd(a, b, dx, orientation: str = "outgoing"):
    """(da, db), the gradients of sum(dx * x) with respect to a and b."""
    a, b, dx = _f64(a), _f64(b), _f64(dx)
    if orientation == "outgoing":
        da = dx @ b                                 # da[i,k] = sum_j dx[i,j] b[j,k]
        db = np.swapaxes(dx, -1, -2) @ a            # db[j,k] = sum_i dx[i,j] a[i,k]
        return da, db
    if orientation == "incoming":
        da = b @ np.swapaxes(dx, -1, -2)            # da[k,i] = sum_j b[k,j] dx[i,j]
        db = a @ dx                                 # db[k,j] = sum_i a[k,i] dx[i,j]
        return da, db
    raise ValueError(orientation)
