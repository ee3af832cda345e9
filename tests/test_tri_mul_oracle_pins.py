"""Pins of the triangle-multiplicative contraction oracle (oracle/tri_mul_oracle.py)
against things other than itself: explicit loops over (i, j, k), closed forms,
the incoming/outgoing transpose relation, central finite differences and torch
autograd through an einsum formulation.  Each planted mistake must be caught."""
import numpy as np
import pytest
import torch

from oracle import tri_mul_oracle as T


def rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def loops(a, b, orientation):
    B, C, N, _ = a.shape
    x = np.zeros((B, C, N, N))
    for bi in range(B):
        for c in range(C):
            for i in range(N):
                for j in range(N):
                    s = 0.0
                    for k in range(N):
                        if orientation == "outgoing":
                            s += a[bi, c, i, k] * b[bi, c, j, k]
                        else:
                            s += a[bi, c, k, i] * b[bi, c, k, j]
                    x[bi, c, i, j] = s
    return x


@pytest.mark.parametrize("orientation", T.ORIENTATIONS)
def test_matches_explicit_loops(orientation):
    a, b = rand((2, 3, 5, 5), 1), rand((2, 3, 5, 5), 2)
    np.testing.assert_allclose(T.fwd(a, b, orientation), loops(a, b, orientation), rtol=1e-12, atol=1e-12)


def test_identity_partner_returns_the_other_operand():
    a = rand((1, 4, 7, 7), 3)
    eye = np.broadcast_to(np.eye(7), (1, 4, 7, 7))
    np.testing.assert_allclose(T.fwd(a, eye, "outgoing"), a, atol=1e-15)           # sum_k a[i,k] d[j,k] = a[i,j]
    np.testing.assert_allclose(T.fwd(eye, a, "incoming"), a, atol=1e-15)           # sum_k d[k,i] a[k,j] = a[i,j]


def test_incoming_is_outgoing_on_transposed_operands():
    a, b = rand((1, 2, 9, 9), 4), rand((1, 2, 9, 9), 5)
    tr = lambda x: np.swapaxes(x, -1, -2)
    np.testing.assert_allclose(T.fwd(a, b, "incoming"), T.fwd(tr(a), tr(b), "outgoing"), rtol=1e-13)


def test_self_contraction_is_symmetric_positive_semidefinite():
    a = rand((1, 3, 8, 8), 6)
    x = T.fwd(a, a, "outgoing")
    np.testing.assert_allclose(x, np.swapaxes(x, -1, -2), rtol=1e-13)
    assert np.all(np.linalg.eigvalsh(x) > -1e-9)


@pytest.mark.parametrize("orientation", T.ORIENTATIONS)
def test_backward_matches_finite_differences(orientation):
    a, b, dx = rand((1, 2, 4, 4), 7), rand((1, 2, 4, 4), 8), rand((1, 2, 4, 4), 9)
    da, db = T.bwd(a, b, dx, orientation)
    eps = 1e-6
    loss = lambda aa, bb: float(np.sum(dx * loops(aa, bb, orientation)))
    for grad, which in ((da, 0), (db, 1)):
        num = np.zeros_like(grad)
        for idx in np.ndindex(grad.shape):
            p, m = [a.copy(), b.copy()], [a.copy(), b.copy()]
            p[which][idx] += eps
            m[which][idx] -= eps
            num[idx] = (loss(*p) - loss(*m)) / (2 * eps)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-7)


@pytest.mark.parametrize("orientation", T.ORIENTATIONS)
def test_backward_matches_torch_autograd(orientation):
    a, b, dx = rand((2, 3, 6, 6), 10), rand((2, 3, 6, 6), 11), rand((2, 3, 6, 6), 12)
    ta = torch.tensor(a, requires_grad=True)
    tb = torch.tensor(b, requires_grad=True)
    eq = "bcik,bcjk->bcij" if orientation == "outgoing" else "bcki,bckj->bcij"
    torch.einsum(eq, ta, tb).backward(torch.tensor(dx))
    da, db = T.bwd(a, b, dx, orientation)
    np.testing.assert_allclose(da, ta.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(db, tb.grad.numpy(), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("planted", [1, 2])
def test_planted_mistakes_are_caught(planted):
    a, b = rand((1, 2, 5, 5), 13), rand((1, 2, 5, 5), 14)
    assert np.max(np.abs(T.fwd(a, b, "outgoing", planted=planted) - loops(a, b, "outgoing"))) > 1e-2
