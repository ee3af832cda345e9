"""FP64 CPU oracle for the gated output projection around triangle attention --
TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module; the product path shares no code with it.

What it computes.  The pages describe only the attention itself; the steps on
either side of it are the model's.  Read the AlphaFold way, the attention
output leaves through a sigmoid gate computed from the pair representation and
a linear output projection, position by position (b, i, j):

    g = sigmoid(z Wg)          z: [R, cz]   Wg: [cz, co]    (no bias)
    y = (g * o) Wo             o: [R, co]   Wo: [co, cz]    (no bias)

with R = B*N*N pair positions, z the attention block's (normalised) pair input,
o the attention output with heads concatenated (co = H*d, channel h*d + c).
Backward for the upstream gradient dy:

    a   = g * o
    da  = dy Wo^T
    do  = da * g
    dl  = da * o * g * (1 - g)            (gradient of the gate logits)
    dz  = dl Wg^T
    dWo = a^T dy                          (sum over all positions)
    dWg = z^T dl

Every product is one FP64 matmul (a library primitive) and every other step
is elementwise; pinned by ``tests/test_tri_gate_oracle_pins.py``.
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def fwd(z, o, wg, wo, planted: int = 0):
    """y for every row.  ``planted``: 1 gates with the wrong sign, 2 skips the gate."""
    z, o, wg, wo = _f64(z), _f64(o), _f64(wg), _f64(wo)
    logit = z @ wg
    g = sigmoid(-logit) if planted == 1 else sigmoid(logit)
    a = o if planted == 2 else g * o
    return a @ wo


def bwd(z, o, wg, wo, dy):
    """(dz, do, dWg, dWo)."""
    z, o, wg, wo, dy = _f64(z), _f64(o), _f64(wg), _f64(wo), _f64(dy)
    g = sigmoid(z @ wg)
    a = g * o
    da = dy @ wo.T
    do = da * g
    dl = da * o * g * (1.0 - g)
    dz = dl @ wg.T
    return dz, do, z.T @ dl, a.T @ dy
