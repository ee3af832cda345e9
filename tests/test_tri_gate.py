"""The fused gated output projection (tri_gate_fwd): host-side argument checks (no
GPU) and GPU parity against the FP64 oracle (oracle/tri_gate_oracle.py) on the same
BF16 inputs."""
import ctypes

import numpy as np
import pytest
import torch

from triangle_attention_biomolecular_b200 import _binding as Bd
from triangle_attention_biomolecular_b200 import build as build_mod

# y passes through BF16 twice: the gated a = g*o is rounded to BF16 before the second
# contraction and y itself is stored in BF16 (each ~2^-9/sqrt(3) = 1.1e-3 relative
# RMS); the approximate exp2/reciprocal of the gate add ~1e-6.  Gate: 5e-3.
GATE = 5e-3


def rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return Bd.load()


def fake(R=300, base=0x10000):
    a = Bd.GateFwdArgs()
    a.R = R
    a.z, a.o, a.wg, a.wo, a.y = (base + k * 0x1000000 for k in range(5))
    a.z_stride = a.o_stride = a.y_stride = 128
    return a


def test_host_side_rejections(lib):
    assert lib.tri_gate_fwd(None, None) == Bd.TRI_ATTN_ERR_NULL
    a = fake()
    a.wo = None
    assert lib.tri_gate_fwd(ctypes.byref(a), None) == Bd.TRI_ATTN_ERR_NULL
    a = fake(R=0)
    assert lib.tri_gate_fwd(ctypes.byref(a), None) == Bd.TRI_ATTN_ERR_SHAPE
    a = fake()
    a.o_stride = 132
    assert lib.tri_gate_fwd(ctypes.byref(a), None) == Bd.TRI_ATTN_ERR_STRIDE
    a = fake()
    a.y += 2
    assert lib.tri_gate_fwd(ctypes.byref(a), None) == Bd.TRI_ATTN_ERR_ALIGN


def inputs(R, seed, zscale=1.0):
    g = torch.Generator().manual_seed(seed)
    z = (torch.randn((R, 128), generator=g) * zscale).to(torch.bfloat16)
    o = torch.randn((R, 128), generator=g).to(torch.bfloat16)
    wg = (torch.randn((128, 128), generator=g) / 128 ** 0.5).to(torch.bfloat16)
    wo = (torch.randn((128, 128), generator=g) / 128 ** 0.5).to(torch.bfloat16)
    return z, o, wg, wo


@pytest.mark.gpu
@pytest.mark.parametrize("R,zscale", [(1, 1.0), (200, 1.0), (128 * 148 * 2 + 77, 1.0), (4096, 8.0)])
def test_parity(R, zscale):
    from oracle import tri_gate_oracle as G
    z, o, wg, wo = inputs(R, 31 + R, zscale)
    dev = torch.device("cuda")
    # rows of z and y padded to 136 elements, to exercise the row strides
    zp = torch.zeros((R, 136), dtype=torch.bfloat16, device=dev)
    zp[:, :128] = z.to(dev)
    yp = torch.full((R, 136), float("nan"), dtype=torch.bfloat16, device=dev)
    Bd.tri_gate_fwd(zp[:, :128], o.to(dev), wg.to(dev), wo.to(dev), yp[:, :128])
    torch.cuda.synchronize()
    st, word = Bd.tri_attn_device_error(True)
    assert st == Bd.TRI_ATTN_OK, f"device error word {word:#x}"
    got = yp[:, :128].float().cpu().numpy()
    want = G.fwd(z.double().numpy(), o.double().numpy(), wg.double().numpy(), wo.double().numpy())
    assert np.all(np.isfinite(got))
    assert rel(got, want) <= GATE, rel(got, want)
    assert torch.isnan(yp[:, 128:].float()).all()  # padding untouched
