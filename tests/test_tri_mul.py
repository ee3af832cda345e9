"""The triangle-multiplicative contraction (tri_mul_fwd / tri_mul_bwd): host-side
argument checks and struct layout (no GPU), and GPU parity against the FP64 oracle
(oracle/tri_mul_oracle.py) on the same BF16 inputs."""
import ctypes
import os

import numpy as np
import pytest
import torch

from triangle_attention_biomolecular_b200 import _binding as Bd
from triangle_attention_biomolecular_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# BF16 rounding of the outputs alone gives ~2^-9/sqrt(3) = 1.1e-3 relative RMS; the
# FP32 sums over N <= 1024 terms add < 1e-6.  The gate leaves a 4x margin and is far
# below what a wrong index or a missing term produces (>= 1e-1, see the oracle pins).
GATE = 5e-3


def rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return Bd.load()


def _fake_args(B=1, C=2, N=64, base=0x10000):
    m = Bd.MulFwdArgs()
    m.B, m.C, m.N = B, C, N
    for idx, t in enumerate((m.a, m.b, m.x)):
        t.ptr = base + idx * 0x1000000
        for x, s in enumerate((C * N * N, N * N, N, 1)):
            t.stride[x] = s
    m.flags = 0
    return m


def test_host_side_rejections(lib):
    assert lib.tri_mul_fwd(None, None) == Bd.TRI_ATTN_ERR_NULL
    m = _fake_args(N=0)
    assert lib.tri_mul_fwd(ctypes.byref(m), None) == Bd.TRI_ATTN_ERR_SHAPE
    m = _fake_args(N=20000)
    assert lib.tri_mul_fwd(ctypes.byref(m), None) == Bd.TRI_ATTN_ERR_UNSUPPORTED
    m = _fake_args()
    m.b.stride[3] = 2
    assert lib.tri_mul_fwd(ctypes.byref(m), None) == Bd.TRI_ATTN_ERR_STRIDE
    m = _fake_args()
    m.x.ptr += 8
    assert lib.tri_mul_fwd(ctypes.byref(m), None) == Bd.TRI_ATTN_ERR_ALIGN
    m = _fake_args()
    m.flags = 6
    assert lib.tri_mul_fwd(ctypes.byref(m), None) == Bd.TRI_ATTN_ERR_UNSUPPORTED
    bw = Bd.MulBwdArgs()
    bw.f = _fake_args()
    assert lib.tri_mul_bwd(ctypes.byref(bw), None) == Bd.TRI_ATTN_ERR_NULL  # dx, da, db missing


def test_struct_layout_matches_header():
    src = r'''
#include <stddef.h>
#include <stdio.h>
#include "tri_attn.h"
int main(void){
  printf("%zu %zu %zu %zu %zu\n", sizeof(tri_mul_fwd_args), offsetof(tri_mul_fwd_args, x),
         offsetof(tri_mul_fwd_args, flags), sizeof(tri_mul_bwd_args), offsetof(tri_mul_bwd_args, db));
  return 0; }
'''
    import subprocess
    import tempfile
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "l.c")
        open(c, "w").write(src)
        exe = os.path.join(d, "l")
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", exe], check=True)
        got = list(map(int, subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split()))
    want = [ctypes.sizeof(Bd.MulFwdArgs), Bd.MulFwdArgs.x.offset, Bd.MulFwdArgs.flags.offset,
            ctypes.sizeof(Bd.MulBwdArgs), Bd.MulBwdArgs.db.offset]
    assert got == want


def inputs(B, C, N, seed):
    g = torch.Generator().manual_seed(seed)
    mk = lambda: torch.randn((B, C, N, N), generator=g).to(torch.bfloat16)
    return mk(), mk(), mk()


def padded(t, dev):
    """The same values on the device with rows padded to a multiple of 8 elements (the
    ABI wants 16-byte row strides); returns a [B,C,N,N] view."""
    B, C, N, _ = t.shape
    Np = (N + 7) // 8 * 8
    buf = torch.zeros((B, C, N, Np), dtype=t.dtype, device=dev)
    buf[..., :N] = t.to(dev)
    return buf[..., :N]


def run_gpu(a, b, dx, incoming):
    dev = torch.device("cuda")
    a, b, dx = padded(a, dev), padded(b, dev), padded(dx, dev)
    z = torch.zeros_like(a)
    x, da, db = padded(z, dev), padded(z, dev), padded(z, dev)
    Bd.tri_mul_fwd(a, b, x, incoming)
    Bd.tri_mul_bwd(a, b, dx, da, db, incoming)
    torch.cuda.synchronize()
    st, word = Bd.tri_attn_device_error(True)
    assert st == Bd.TRI_ATTN_OK, f"device error word {word:#x}"
    return x.float().cpu().numpy(), da.float().cpu().numpy(), db.float().cpu().numpy()


@pytest.mark.gpu
@pytest.mark.parametrize("incoming", [False, True], ids=["outgoing", "incoming"])
@pytest.mark.parametrize("B,C,N", [(2, 3, 200), (1, 2, 64), (1, 1, 1), (1, 4, 300)])
def test_parity_full(B, C, N, incoming):
    from oracle import tri_mul_oracle as T
    a, b, dx = inputs(B, C, N, 100 + N)
    x, da, db = run_gpu(a, b, dx, incoming)
    o = "incoming" if incoming else "outgoing"
    f64 = lambda t: t.double().numpy()
    rx = T.fwd(f64(a), f64(b), o)
    rda, rdb = T.bwd(f64(a), f64(b), f64(dx), o)
    for name, got, want in (("x", x, rx), ("da", da, rda), ("db", db, rdb)):
        assert np.all(np.isfinite(got)), name
        e = rel(got, want)
        assert e <= GATE, f"{name}: rel-RMSE {e:.3e}"


@pytest.mark.gpu
@pytest.mark.parametrize("incoming", [False, True], ids=["outgoing", "incoming"])
def test_parity_pair_stack_768_sampled_channels(incoming):
    # the 768-residue crop with the 128 pair channels; every output of four channels
    from oracle import tri_mul_oracle as T
    B, C, N = 1, 128, 768
    a, b, dx = inputs(B, C, N, 7)
    x, da, db = run_gpu(a, b, dx, incoming)
    o = "incoming" if incoming else "outgoing"
    for c in (0, 37, 90, 127):
        f64 = lambda t: t[:, c:c + 1].double().numpy()
        rx = T.fwd(f64(a), f64(b), o)
        rda, rdb = T.bwd(f64(a), f64(b), f64(dx), o)
        for name, got, want in (("x", x[:, c:c + 1], rx), ("da", da[:, c:c + 1], rda), ("db", db[:, c:c + 1], rdb)):
            e = rel(got, want)
            assert e <= GATE, f"channel {c} {name}: rel-RMSE {e:.3e}"


@pytest.mark.gpu
def test_bitwise_repeatable():
    a, b, dx = inputs(1, 8, 256, 3)
    r1 = run_gpu(a, b, dx, False)
    r2 = run_gpu(a, b, dx, False)
    for u, v in zip(r1, r2):
        assert np.array_equal(u, v)
