"""The binding fills the C argument blocks with one flat pack per call; every field must
land where the ctypes structures (checked against the C header by test_abi) put it."""
import torch

from triangle_attention_biomolecular_b200 import _binding as B


def _tensors(with_mask=True):
    g = torch.Generator().manual_seed(5)
    q = torch.randn((2, 24, 24, 4, 32), generator=g).to(torch.bfloat16)
    k, v, o, r, do, dq, dk, dv = (torch.empty_like(q) for _ in range(8))
    # a strided view for one of them: every stride must travel as given
    big = torch.empty((2, 24, 24, 8, 32), dtype=torch.bfloat16)
    v = big[:, :, :, :4, :]
    bias = torch.empty((2, 4, 24, 32), dtype=torch.bfloat16)[..., :24]
    mask = torch.zeros((2, 1, 24)).expand(2, 24, 24) if with_mask else None
    lse = torch.empty((2, 4, 24, 24))
    dbias = torch.empty((2, 4, 24, 24), dtype=torch.bfloat16)
    ws = torch.empty(4096, dtype=torch.uint8)
    return q, k, v, bias, mask, o, r, lse, do, dq, dk, dv, dbias, ws


def _same(t5, t):
    return t5.ptr == t.data_ptr() and list(t5.stride) == list(t.stride())


def test_fwd_block_fields():
    q, k, v, bias, mask, o, r, lse, *_ = _tensors()
    a = B.fwd_args(q, k, v, bias, mask, o, r, lse, 0.25)
    assert (a.B, a.N, a.H, a.d, a.scale) == (2, 24, 4, 32, 0.25)
    for s, t in ((a.q, q), (a.k, k), (a.v, v), (a.o, o), (a.resid, r), (a.bias, bias), (a.mask, mask)):
        assert _same(s, t)
    assert list(a.mask.stride) == [24, 0, 1]  # broadcast over rows i
    assert a.lse == lse.data_ptr()


def test_bwd_block_fields():
    q, k, v, bias, mask, o, r, lse, do, dq, dk, dv, dbias, ws = _tensors()
    a = B.bwd_args(q, k, v, bias, mask, o, r, lse, do, dq, dk, dv, dbias, ws, 0.5, 1)
    assert _same(a.f.q, q) and _same(a.f.v, v) and a.f.scale == 0.5 and a.f.lse == lse.data_ptr()
    for s, t in ((a.dout, do), (a.dq, dq), (a.dk, dk), (a.dv, dv), (a.dbias, dbias)):
        assert _same(s, t)
    assert (a.workspace, a.workspace_bytes, a.flags) == (ws.data_ptr(), 4096, 1)


def test_absent_optional_arguments_are_null():
    q, k, v, bias, _, o, r, lse, do, dq, dk, dv, _, _ = _tensors(with_mask=False)
    a = B.bwd_args(q, k, v, bias, None, o, r, lse, do, dq, dk, dv, None, None)
    assert not a.f.mask.ptr and list(a.f.mask.stride) == [0, 0, 0]
    assert not a.dbias.ptr and not a.workspace and a.workspace_bytes == 0 and a.flags == 0
