"""The kernels' FMA-pipe exponential (ex2_fma2 in csrc/sm100.cuh): range
reduction to x = n + f with n = floor(x), a fitted cubic for 2^f on [0, 1), and
n added into the exponent field.  Checked here on the CPU, in float32 arithmetic,
with the coefficients read from the source: the relative error bound the kernels
rely on (far below the BF16 rounding of the probabilities they feed), the
behaviour at integer arguments, the clamp for very negative arguments, the large
positive arguments the gated projection uses, and that projection's sigmoid and
its complement (sigmoid2 in csrc/tri_gate.cuh)."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "triangle_attention_biomolecular_b200", "csrc", "sm100.cuh")


def coefficients():
    text = open(SRC).read()
    c = [float(re.search(rf"kEx2C{k}\s*=\s*([-0-9.eE+]+)f", text).group(1)) for k in range(4)]
    return np.array(c, dtype=np.float32)


def fma32(a, b, c):
    # a, b, c float32: the float64 product is exact, one rounding to float32 after the add
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def ex2_fma(x):
    """The kernel's steps, element by element, in float32."""
    c = coefficients()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)  # 1.5 * 2^23
    t = (np.floor(x.astype(np.float64)) + 12582912.0).astype(np.float32)  # add rounded toward -inf
    n = (t - magic).astype(np.float32)
    f = fma32(n, np.full_like(n, -1.0), x)
    q = fma32(np.full_like(f, c[3]), f, np.full_like(f, c[2]))
    q = fma32(q, f, np.full_like(f, c[1]))
    q = fma32(q, f, np.full_like(f, c[0]))
    bits = q.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_relative_error_bound():
    rng = np.random.default_rng(5)
    x = np.concatenate([np.linspace(-125, 8, 200001), -rng.random(100000) * 40, rng.random(10000) * 8]).astype(np.float32)
    got = ex2_fma(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 2e-4, rel.max()
    # far below the BF16 half-ulp (2^-9) that every probability is rounded to afterwards
    assert rel.max() < 2.0 ** -9 / 10


def test_integer_arguments_and_monotone_steps():
    n = np.arange(-125, 9, dtype=np.float32)
    got = ex2_fma(n).astype(np.float64)
    assert np.all(np.abs(got / np.exp2(n.astype(np.float64)) - 1) < 1e-4)
    x = np.linspace(-3, 3, 60001).astype(np.float32)
    y = ex2_fma(x)
    assert np.all(np.diff(y.astype(np.float64)) > -1e-6 * y[1:])  # no jumps at the integer seams


def test_very_negative_arguments_are_tiny_and_finite():
    y = ex2_fma(np.array([-125.5, -200.0, -1e9, -np.inf], dtype=np.float32))
    assert np.all(np.isfinite(y)) and np.all(y > 0) and np.all(y < 3e-38)


def test_coefficients_are_near_the_taylor_series():
    # a guard against a mistyped constant: the fit stays close to (ln 2)^k / k!
    c = coefficients().astype(np.float64)
    taylor = np.array([1.0, np.log(2), np.log(2) ** 2 / 2, np.log(2) ** 3 / 6])
    assert np.all(np.abs(c - taylor) < 0.03)


def test_large_positive_arguments_up_to_the_gate_clamp():
    # the gated projection evaluates 2^x for x = -G log2(e) clamped to <= 126: n is added
    # into the exponent field, which must not carry into the sign bit anywhere up to 126
    x = np.concatenate([np.linspace(8, 126, 100001), np.arange(8, 127)]).astype(np.float32)
    got = ex2_fma(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.all(np.isfinite(got)) and np.all(got > 0)
    assert (np.abs(got - ref) / ref).max() < 2e-4


def sigmoid2(x):
    """The gate's g = 1 / (1 + e) and h = 1 - g = e g with e = 2^(-x log2 e) from the
    FMA-pipe exp2 (argument clamped to [-125, 126]); the hardware reciprocal is taken
    as the correctly rounded float32 one here."""
    a = np.minimum(x.astype(np.float32) * np.float32(-1.4426950408889634), np.float32(126.0))
    e = ex2_fma(a)
    g = (np.float32(1.0) / (np.float32(1.0) + e)).astype(np.float32)
    return g, (e * g).astype(np.float32)


def test_gate_sigmoid_and_its_complement():
    x = np.concatenate([np.linspace(-80, 80, 160001), [0.0]]).astype(np.float32)
    g, h = sigmoid2(x)
    x64 = x.astype(np.float64)
    ref_g = 1.0 / (1.0 + np.exp(-x64))
    ref_h = 1.0 / (1.0 + np.exp(x64))  # 1 - g without cancellation
    assert (np.abs(g - ref_g) / ref_g).max() < 3e-4
    assert (np.abs(h - ref_h) / ref_h).max() < 3e-4  # the complement keeps its relative accuracy
    g0, h0 = sigmoid2(np.array([0.0], dtype=np.float32))
    assert abs(g0[0] - 0.5) < 1e-4 and abs(h0[0] - 0.5) < 1e-4
    # saturated logits: g rounds to 1 or to a tiny normal number, never to NaN or inf
    gs, hs = sigmoid2(np.array([-1e4, -200.0, 200.0, 1e4], dtype=np.float32))
    assert np.all(np.isfinite(gs)) and np.all(np.isfinite(hs))
    assert gs[0] < 1e-37 and gs[1] < 1e-37 and gs[2] == 1.0 and gs[3] == 1.0
    assert abs(hs[0] - 1.0) < 1e-6 and hs[3] < 1e-37
