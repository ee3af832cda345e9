"""tri_attn_bwd_static_scratch: the backward on the library's fixed per-device
scratch array, which allocates nothing.  This file is collected last, so in a
full run it also exercises the entry point after every other test has used the
library in the same process; it passes on its own as well."""
import ctypes

import pytest
import torch

from triangle_attention_biomolecular_b200 import _binding as Bd
from triangle_attention_biomolecular_b200 import api
from triangle_attention_biomolecular_b200 import build as build_mod
from triangle_attention_biomolecular_b200 import synthetic as S


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return Bd.load()


def _fake_bwd_args(N, d=32, H=4, base=0x10000):
    """Aligned but fake device pointers; every case below is rejected on the host
    before anything could dereference them."""
    a = Bd.BwdArgs()
    f = a.f
    f.B, f.N, f.H, f.d, f.scale = 1, N, H, d, 0.0
    st5 = (N * N * H * d, N * H * d, H * d, d, 1)
    names5 = [(f, n) for n in ("q", "k", "v", "o", "resid")] + [(a, n) for n in ("dout", "dq", "dk", "dv")]
    for idx, (obj, name) in enumerate(names5):
        t = getattr(obj, name)
        t.ptr = base + idx * 0x1000000
        for x in range(5):
            t.stride[x] = st5[x]
    for idx, t in enumerate((f.bias, a.dbias)):
        t.ptr = base + (10 + idx) * 0x1000000
        for x, s in enumerate((H * N * N, N * N, N, 1)):
            t.stride[x] = s
    f.mask.ptr = None
    f.lse = base + 12 * 0x1000000
    a.workspace, a.workspace_bytes, a.flags = None, 0, 0
    return a


def test_static_scratch_host_side_rejections(lib):
    assert lib.tri_attn_bwd_static_scratch(None, None) == Bd.TRI_ATTN_ERR_NULL
    # sizes needing more than the fixed area: their own status, before any device access
    assert Bd.tri_attn_bwd_workspace_bytes(1, 2048, 4, 32) > Bd.TRI_ATTN_STATIC_SCRATCH_BYTES
    a = _fake_bwd_args(2048)
    assert lib.tri_attn_bwd_static_scratch(ctypes.byref(a), None) == Bd.TRI_ATTN_ERR_SCRATCH_LIMIT
    assert "static scratch" in Bd.tri_attn_strerror(Bd.TRI_ATTN_ERR_SCRATCH_LIMIT)
    # invalid sizes keep the regular argument errors
    a = _fake_bwd_args(64, d=48)
    assert lib.tri_attn_bwd_static_scratch(ctypes.byref(a), None) == Bd.TRI_ATTN_ERR_UNSUPPORTED
    # argument errors come before the size limit and before any CUDA call: on a
    # machine without a GPU every CUDA call fails, so these statuses also show
    # that nothing reached the runtime
    a = _fake_bwd_args(64)
    a.dq.ptr = None
    assert lib.tri_attn_bwd_static_scratch(ctypes.byref(a), None) == Bd.TRI_ATTN_ERR_NULL
    a = _fake_bwd_args(2048)
    a.dk.ptr = None  # oversized and a NULL gradient: the argument error wins
    assert lib.tri_attn_bwd_static_scratch(ctypes.byref(a), None) == Bd.TRI_ATTN_ERR_NULL
    a = _fake_bwd_args(64)
    a.dv.ptr += 2
    assert lib.tri_attn_bwd_static_scratch(ctypes.byref(a), None) == Bd.TRI_ATTN_ERR_ALIGN
    a = _fake_bwd_args(64)
    a.dout.stride[2] = 12
    assert lib.tri_attn_bwd_static_scratch(ctypes.byref(a), None) == Bd.TRI_ATTN_ERR_STRIDE
    # the documented limit covers the 768-residue crop at both head widths
    for d in (32, 64):
        assert Bd.tri_attn_bwd_workspace_bytes(1, 768, 4, d) <= Bd.TRI_ATTN_STATIC_SCRATCH_BYTES


# cases that between them use every region of the scratch: dBias partial sums
# (few tiles), dQ staging slots (more key tiles than TMEM holds), both head widths
CASES = [
    S.Workload("N=200 ragged", 1, 200, 4, 32, mask="ragged", len_lo=150, len_hi=200),
    S.Workload("N=1024 ragged", 1, 1024, 4, 32, mask="ragged", len_lo=900, len_hi=1024),
    S.Workload("N=256 d=64", 1, 256, 4, 64, mask="zeros"),
]


@pytest.mark.gpu
@pytest.mark.parametrize("wl", CASES, ids=[c.name for c in CASES])
def test_static_scratch_matches_workspace_entry_point(lib, wl):
    x = S.make_inputs(wl, 17)
    dev = torch.device("cuda")
    q, k, v, do, bias = (x[n].to(dev) for n in ("q", "k", "v", "dout", "bias"))
    mask = x["mask"].to(dev) if x["mask"] is not None else None
    o, r, lse = api.forward(q, k, v, bias, mask)
    ref = api.backward(q, k, v, bias, mask, o, r, lse, do)
    runs = []
    for _ in range(2):  # two calls in a row on the same (now dirty) scratch
        Npad = (wl.N + 7) // 8 * 8  # dbias rows padded to a 16-byte multiple, as api.backward does
        db = torch.full((wl.B, wl.H, wl.N, Npad), float("nan"), dtype=torch.bfloat16, device=dev)[..., :wl.N]
        grads = tuple(torch.full_like(t, float("nan")) for t in ref[:3]) + (db,)
        Bd.tri_attn_bwd_static_scratch(q, k, v, bias, mask, o, r, lse, do, *grads)
        runs.append(grads)
    torch.cuda.synchronize()
    st, word = Bd.tri_attn_device_error(True)
    assert st == Bd.TRI_ATTN_OK, f"device error word {word:#x}"
    # Same kernels, fixed-order reductions, scratch fully rewritten before use:
    # the tolerance is zero (bitwise-identical gradients).
    for got in runs:
        for name, g, want in zip(("dq", "dk", "dv", "dbias"), got, ref):
            assert torch.isfinite(g.float()).all(), name
            assert torch.equal(g, want), f"{name}: max |diff| {(g.float() - want.float()).abs().max().item():.3e}"
