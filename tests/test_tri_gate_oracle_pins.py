"""Pins of the gated output projection oracle (oracle/tri_gate_oracle.py) against
things other than itself: explicit per-row loops, closed forms (zero logits give
the gate 1/2, huge logits saturate it), finite differences and torch autograd on
an independent formulation.  Each planted mistake must be caught."""
import math

import numpy as np
import pytest
import torch

from oracle import tri_gate_oracle as G


def rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def loops(z, o, wg, wo):
    R, cz = z.shape
    co = o.shape[1]
    y = np.zeros((R, cz))
    for r in range(R):
        for c in range(co):
            s = sum(z[r, k] * wg[k, c] for k in range(cz))
            g = 1.0 / (1.0 + math.exp(-s))
            for t in range(cz):
                y[r, t] += g * o[r, c] * wo[c, t]
    return y


def test_matches_explicit_loops():
    z, o = rand((6, 5), 1), rand((6, 4), 2)
    wg, wo = rand((5, 4), 3), rand((4, 5), 4)
    np.testing.assert_allclose(G.fwd(z, o, wg, wo), loops(z, o, wg, wo), rtol=1e-12, atol=1e-12)


def test_closed_forms():
    o, wo = rand((7, 4), 5), rand((4, 3), 6)
    z0 = np.zeros((7, 3))
    np.testing.assert_allclose(G.fwd(z0, o, rand((3, 4), 7), wo), 0.5 * (o @ wo), rtol=1e-14)   # gate 1/2
    z1 = np.ones((7, 3))
    wg_big = np.full((3, 4), 50.0)
    np.testing.assert_allclose(G.fwd(z1, o, wg_big, wo), o @ wo, rtol=1e-12)                      # gate saturates at 1
    np.testing.assert_allclose(G.fwd(z1, o, -wg_big, wo), np.zeros((7, 3)), atol=1e-50)             # and at 0


def test_backward_matches_finite_differences():
    z, o = rand((3, 4), 8), rand((3, 4), 9)
    wg, wo, dy = rand((4, 4), 10), rand((4, 4), 11), rand((3, 4), 12)
    grads = G.bwd(z, o, wg, wo, dy)
    loss = lambda zz, oo, ww, vv: float(np.sum(dy * G.fwd(zz, oo, ww, vv)))
    args = [z, o, wg, wo]
    eps = 1e-6
    for which, grad in enumerate((grads[0], grads[1], grads[2], grads[3])):
        num = np.zeros_like(grad)
        for idx in np.ndindex(grad.shape):
            p = [a.copy() for a in args]
            m = [a.copy() for a in args]
            p[which][idx] += eps
            m[which][idx] -= eps
            num[idx] = (loss(*p) - loss(*m)) / (2 * eps)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-8)


def test_backward_matches_torch_autograd():
    z, o = rand((16, 8), 13), rand((16, 6), 14)
    wg, wo, dy = rand((8, 6), 15), rand((6, 8), 16), rand((16, 8), 17)
    t = [torch.tensor(a, requires_grad=True) for a in (z, o, wg, wo)]
    y = torch.einsum("rc,rc,ct->rt", torch.sigmoid(torch.einsum("rk,kc->rc", t[0], t[2])), t[1], t[3])
    y.backward(torch.tensor(dy))
    for got, ref in zip(G.bwd(z, o, wg, wo, dy), t):
        np.testing.assert_allclose(got, ref.grad.numpy(), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("planted", [1, 2])
def test_planted_mistakes_are_caught(planted):
    z, o = rand((6, 5), 18), rand((6, 4), 19)
    wg, wo = rand((5, 4), 20), rand((4, 5), 21)
    assert np.max(np.abs(G.fwd(z, o, wg, wo, planted=planted) - loops(z, o, wg, wo))) > 1e-2
