"""The fused gated output projection (tri_gate_fwd, tri_gate_bwd): host-side argument
checks (no GPU) and GPU parity against the FP64 oracle (oracle/tri_gate_oracle.py) on
the same BF16 inputs."""
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


def fake_bwd(R=300, base=0x10000):
    a = Bd.GateBwdArgs()
    a.f = fake(R, base)
    a.dy, a.dz, a.d_o, a.dwg, a.dwo, a.workspace = (base + k * 0x1000000 for k in range(5, 11))
    a.dy_stride = a.dz_stride = a.do_stride = 128
    a.workspace_bytes = Bd.tri_gate_bwd_workspace_bytes(R)
    return a


def test_bwd_host_side_rejections(lib):
    assert Bd.tri_gate_bwd_workspace_bytes(0) == 0
    assert Bd.tri_gate_bwd_workspace_bytes(1) == 2 * 128 * 128 * 4            # one CTA's partial sums
    assert Bd.tri_gate_bwd_workspace_bytes(10 ** 7) == 148 * 2 * 128 * 128 * 4  # one CTA per SM at most
    assert lib.tri_gate_bwd(None, None) == Bd.TRI_ATTN_ERR_NULL
    a = fake_bwd()
    a.dwo = None
    assert lib.tri_gate_bwd(ctypes.byref(a), None) == Bd.TRI_ATTN_ERR_NULL
    a = fake_bwd()
    a.f.R = 0
    assert lib.tri_gate_bwd(ctypes.byref(a), None) == Bd.TRI_ATTN_ERR_SHAPE
    a = fake_bwd()
    a.dz_stride = 100
    assert lib.tri_gate_bwd(ctypes.byref(a), None) == Bd.TRI_ATTN_ERR_STRIDE
    a = fake_bwd()
    a.dwg += 4
    assert lib.tri_gate_bwd(ctypes.byref(a), None) == Bd.TRI_ATTN_ERR_ALIGN
    a = fake_bwd()
    a.workspace_bytes -= 1
    assert lib.tri_gate_bwd(ctypes.byref(a), None) == Bd.TRI_ATTN_ERR_WORKSPACE
    a = fake_bwd()
    a.workspace = None
    assert lib.tri_gate_bwd(ctypes.byref(a), None) == Bd.TRI_ATTN_ERR_WORKSPACE


# dz, do: dA = dy Wo^T in FP32, then g and s = o g (1 - g) rounded to BF16 before the
# products (2^-9 relative each), dl rounded to BF16 before dz = dl Wg^T, outputs stored
# in BF16 -- three or four roundings of ~1.1e-3 RMS.  dWg, dWo: sums over R rows of
# BF16 products (a and dl rounded to BF16) accumulated in FP32.  Gate: 1e-2.
GATE_BWD = 1e-2


@pytest.mark.gpu
@pytest.mark.parametrize("R,zscale", [(1, 1.0), (200, 1.0), (128 * 148 * 2 + 77, 1.0), (4096, 8.0)])
def test_bwd_parity(R, zscale):
    from oracle import tri_gate_oracle as G
    z, o, wg, wo = inputs(R, 71 + R, zscale)
    dy = torch.randn((R, 128), generator=torch.Generator().manual_seed(R)).to(torch.bfloat16)
    dev = torch.device("cuda")
    # o and dz rows padded to 136 elements, to exercise the row strides
    op = torch.zeros((R, 136), dtype=torch.bfloat16, device=dev)
    op[:, :128] = o.to(dev)
    dzp = torch.full((R, 136), float("nan"), dtype=torch.bfloat16, device=dev)
    d_o = torch.full((R, 128), float("nan"), dtype=torch.bfloat16, device=dev)
    dwg = torch.full((128, 128), float("nan"), device=dev)
    dwo = torch.full((128, 128), float("nan"), device=dev)
    ws = torch.empty(Bd.tri_gate_bwd_workspace_bytes(R), dtype=torch.uint8, device=dev)
    args = (z.to(dev), op[:, :128], wg.to(dev), wo.to(dev), dy.to(dev), dzp[:, :128], d_o, dwg, dwo, ws)
    Bd.tri_gate_bwd(*args)
    torch.cuda.synchronize()
    st, word = Bd.tri_attn_device_error(True)
    assert st == Bd.TRI_ATTN_OK, f"device error word {word:#x}"
    want = G.bwd(*(t.double().numpy() for t in (z, o, wg, wo, dy)))
    got = (dzp[:, :128].float().cpu().numpy(), d_o.float().cpu().numpy(), dwg.cpu().numpy(), dwo.cpu().numpy())
    for name, gv, wv in zip(("dz", "do", "dWg", "dWo"), got, want):
        assert np.all(np.isfinite(gv)), name
        assert rel(gv, wv) <= GATE_BWD, (name, rel(gv, wv))
    assert torch.isnan(dzp[:, 128:].float()).all()  # padding untouched
    # the weight gradients are summed in a fixed order: a second call is bitwise identical
    first = [t.clone() for t in (dzp, d_o, dwg, dwo)]
    Bd.tri_gate_bwd(*args)
    torch.cuda.synchronize()
    for a_, b_ in zip(first, (dzp, d_o, dwg, dwo)):
        assert torch.equal(a_.view(torch.int32) if a_.dtype == torch.float32 else a_.view(torch.int16),
                           b_.view(torch.int32) if b_.dtype == torch.float32 else b_.view(torch.int16))
