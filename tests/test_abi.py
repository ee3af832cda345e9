"""C-ABI checks that need no GPU: the library loads, exports every entry point
include/tri_attn.h declares, and rejects bad arguments on the host (with the
documented status) before touching any device."""
import ctypes
import os
import re

import pytest
import torch

from triangle_attention_biomolecular_b200 import _binding as B
from triangle_attention_biomolecular_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tri_attn.h")


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tri_(?:attn|mul|gate)_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    for n in ("tri_attn_fwd", "tri_attn_bwd", "tri_attn_fwd_rows", "tri_attn_dbias_sum", "tri_mul_fwd",
              "tri_gate_bwd"):
        assert n in names
    for n in names:
        assert hasattr(lib, n), f"missing export {n}"


def test_library_does_not_link_the_driver():
    out = os.popen(f"ldd {build_mod.LIB}").read()
    assert "libcuda.so" not in out and "libcudart" not in out


def test_strerror_covers_every_status(lib):
    seen = set()
    for code in range(12):
        s = B.tri_attn_strerror(code)
        assert s and s not in seen
        seen.add(s)
    assert B.tri_attn_strerror(99) == "unknown status"
    assert B.tri_attn_abi_version() == 1


def test_workspace_bytes_is_a_pure_function_of_sizes(lib):
    assert B.tri_attn_bwd_workspace_bytes(1, 768, 4, 32) == B.tri_attn_bwd_workspace_bytes(1, 768, 4, 32)
    assert B.tri_attn_bwd_workspace_bytes(1, 768, 4, 32) >= 4 * 768 * 768 * 4
    assert B.tri_attn_bwd_workspace_bytes(0, 768, 4, 32) == 0
    assert B.tri_attn_bwd_workspace_bytes(1, 768, 4, 48) == 0
    assert B.tri_attn_bwd_workspace_bytes(1, 5000, 4, 32) == 0


def _fake_args(Bn=1, N=64, H=2, d=32, base=0x10000):
    """Argument struct with aligned but fake device pointers (never dereferenced:
    every case below fails validation, or fails the device check, before any launch)."""
    a = B.FwdArgs()
    a.B, a.N, a.H, a.d, a.scale = Bn, N, H, d, 0.0
    st5 = (N * N * H * d, N * H * d, H * d, d, 1)
    for idx, name in enumerate(("q", "k", "v", "o", "resid")):
        t = getattr(a, name)
        t.ptr = base + idx * 0x100000
        for x in range(5):
            t.stride[x] = st5[x]
    a.bias.ptr = base + 0x800000
    for x, s in enumerate((H * N * N, N * N, N, 1)):
        a.bias.stride[x] = s
    a.mask.ptr = None
    a.lse = base + 0x900000
    return a


def _fwd(lib, a):
    return lib.tri_attn_fwd(ctypes.byref(a), None)


def test_fwd_validation_codes(lib):
    assert lib.tri_attn_fwd(None, None) == B.TRI_ATTN_ERR_NULL
    a = _fake_args(); a.q.ptr = None
    assert _fwd(lib, a) == B.TRI_ATTN_ERR_NULL
    a = _fake_args(); a.lse = None
    assert _fwd(lib, a) == B.TRI_ATTN_ERR_NULL
    a = _fake_args(Bn=0)
    assert _fwd(lib, a) == B.TRI_ATTN_ERR_SHAPE
    a = _fake_args(); a.H = 0
    assert _fwd(lib, a) == B.TRI_ATTN_ERR_SHAPE
    a = _fake_args(d=48)
    assert _fwd(lib, a) == B.TRI_ATTN_ERR_UNSUPPORTED
    a = _fake_args(); a.N = 5000
    assert _fwd(lib, a) == B.TRI_ATTN_ERR_UNSUPPORTED
    a = _fake_args(); a.k.stride[4] = 2
    assert _fwd(lib, a) == B.TRI_ATTN_ERR_STRIDE
    a = _fake_args(); a.v.stride[2] = 12
    assert _fwd(lib, a) == B.TRI_ATTN_ERR_STRIDE
    a = _fake_args(); a.bias.stride[2] = 60
    assert _fwd(lib, a) == B.TRI_ATTN_ERR_STRIDE
    a = _fake_args(); a.o.stride[1] = -64
    assert _fwd(lib, a) == B.TRI_ATTN_ERR_STRIDE
    a = _fake_args(); a.resid.ptr += 8
    assert _fwd(lib, a) == B.TRI_ATTN_ERR_ALIGN
    a = _fake_args(); a.lse += 4
    assert _fwd(lib, a) == B.TRI_ATTN_ERR_ALIGN
    a = _fake_args(); a.mask.ptr = 0x20002
    assert _fwd(lib, a) == B.TRI_ATTN_ERR_ALIGN
    a = _fake_args(); a.scale = float("nan")
    assert _fwd(lib, a) == B.TRI_ATTN_ERR_SHAPE


def _bwd_args(lib, ws_bytes=None):
    a = B.BwdArgs()
    a.f = _fake_args()
    st5 = (64 * 64 * 2 * 32, 64 * 2 * 32, 2 * 32, 32, 1)
    for idx, name in enumerate(("dout", "dq", "dk", "dv")):
        t = getattr(a, name)
        t.ptr = 0x2000000 + idx * 0x100000
        for x in range(5):
            t.stride[x] = st5[x]
    a.dbias.ptr = 0x3000000
    for x, s in enumerate((2 * 64 * 64, 64 * 64, 64, 1)):
        a.dbias.stride[x] = s
    need = lib.tri_attn_bwd_workspace_bytes(1, 64, 2, 32)
    a.workspace = 0x4000000
    a.workspace_bytes = need if ws_bytes is None else ws_bytes
    return a


def test_bwd_validation_codes(lib):
    assert lib.tri_attn_bwd(None, None) == B.TRI_ATTN_ERR_NULL
    a = _bwd_args(lib); a.dq.ptr = None
    assert lib.tri_attn_bwd(ctypes.byref(a), None) == B.TRI_ATTN_ERR_NULL
    a = _bwd_args(lib); a.dbias.stride[3] = 2
    assert lib.tri_attn_bwd(ctypes.byref(a), None) == B.TRI_ATTN_ERR_STRIDE
    a = _bwd_args(lib, ws_bytes=1024)
    assert lib.tri_attn_bwd(ctypes.byref(a), None) == B.TRI_ATTN_ERR_WORKSPACE
    a = _bwd_args(lib); a.workspace = None
    assert lib.tri_attn_bwd(ctypes.byref(a), None) == B.TRI_ATTN_ERR_WORKSPACE
    a = _bwd_args(lib); a.workspace += 16
    assert lib.tri_attn_bwd(ctypes.byref(a), None) == B.TRI_ATTN_ERR_ALIGN


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_arguments_without_a_device_report_cuda_error(lib):
    # arguments pass validation; the device check then fails -- nothing is launched
    assert _fwd(lib, _fake_args()) in (B.TRI_ATTN_ERR_CUDA, B.TRI_ATTN_ERR_ARCH)
    a = _bwd_args(lib)
    assert lib.tri_attn_bwd(ctypes.byref(a), None) in (B.TRI_ATTN_ERR_CUDA, B.TRI_ATTN_ERR_ARCH)


def test_row_shard_validation_codes(lib):
    a = _fake_args()
    assert lib.tri_attn_fwd_rows(ctypes.byref(a), 0, None) == B.TRI_ATTN_ERR_SHAPE
    assert lib.tri_attn_fwd_rows(ctypes.byref(a), 65, None) == B.TRI_ATTN_ERR_SHAPE  # more rows than N
    assert lib.tri_attn_fwd_rows(None, 8, None) == B.TRI_ATTN_ERR_NULL
    # sizes: a block needs no more workspace than the whole problem, and P partials >= 1
    whole = lib.tri_attn_bwd_workspace_bytes(1, 64, 2, 32)
    for rows in (1, 7, 32, 64):
        assert 0 < lib.tri_attn_bwd_rows_workspace_bytes(1, rows, 64, 2, 32) <= whole
        assert lib.tri_attn_bwd_rows_dbias_parts(1, rows, 64, 2, 32) >= 1
    assert lib.tri_attn_bwd_rows_workspace_bytes(1, 0, 64, 2, 32) == 0
    assert lib.tri_attn_bwd_rows_dbias_parts(1, 65, 64, 2, 32) == 0
    assert lib.tri_attn_bwd_rows_dbias_parts(1, 64, 64, 2, 48) == 0
    parts = 0x5000000
    b = _bwd_args(lib)
    b.dbias.ptr = None  # not used by a shard call
    b.workspace_bytes = lib.tri_attn_bwd_rows_workspace_bytes(1, 32, 64, 2, 32)
    assert lib.tri_attn_bwd_rows(ctypes.byref(b), 32, None, None) == B.TRI_ATTN_ERR_NULL
    assert lib.tri_attn_bwd_rows(ctypes.byref(b), 32, ctypes.c_void_p(parts + 4), None) == B.TRI_ATTN_ERR_ALIGN
    assert lib.tri_attn_bwd_rows(ctypes.byref(b), 0, ctypes.c_void_p(parts), None) == B.TRI_ATTN_ERR_SHAPE
    b.workspace_bytes -= 256
    assert lib.tri_attn_bwd_rows(ctypes.byref(b), 32, ctypes.c_void_p(parts), None) == B.TRI_ATTN_ERR_WORKSPACE
    db = B.Tensor4()
    db.ptr = 0x3000000
    for x, st in enumerate((2 * 64 * 64, 64 * 64, 64, 1)):
        db.stride[x] = st
    assert lib.tri_attn_dbias_sum(None, 2, 1, 2, 64, db, None) == B.TRI_ATTN_ERR_NULL
    assert lib.tri_attn_dbias_sum(ctypes.c_void_p(parts), 0, 1, 2, 64, db, None) == B.TRI_ATTN_ERR_SHAPE
    assert lib.tri_attn_dbias_sum(ctypes.c_void_p(parts + 8), 2, 1, 2, 64, db, None) == B.TRI_ATTN_ERR_ALIGN
    db.stride[2] = 60
    assert lib.tri_attn_dbias_sum(ctypes.c_void_p(parts), 2, 1, 2, 64, db, None) == B.TRI_ATTN_ERR_STRIDE


def test_binding_rejects_wrong_dtypes_before_the_library():
    q = torch.zeros(1, 8, 8, 2, 32, dtype=torch.float32)
    with pytest.raises(B.TriAttnError) as e:
        B.t5(q, "q")
    assert e.value.status == B.TRI_ATTN_ERR_DTYPE
    with pytest.raises(B.TriAttnError):
        B.mask3(torch.zeros(1, 8, 8, dtype=torch.float64))


def test_header_struct_layout_matches_binding():
    # offsets of the C structs as a C compiler lays them out
    src = r'''
#include <stddef.h>
#include <stdio.h>
#include "tri_attn.h"
int main(void){
  printf("%zu %zu %zu %zu %zu %zu\n", sizeof(tri_attn_fwd_args), offsetof(tri_attn_fwd_args, q),
         offsetof(tri_attn_fwd_args, lse), sizeof(tri_attn_bwd_args), offsetof(tri_attn_bwd_args, workspace),
         offsetof(tri_attn_bwd_args, flags));
  printf("%zu %zu %zu %zu %zu %zu\n", sizeof(tri_mul_fwd_args), offsetof(tri_mul_fwd_args, flags),
         sizeof(tri_mul_bwd_args), offsetof(tri_mul_bwd_args, db), sizeof(tri_gate_fwd_args),
         offsetof(tri_gate_fwd_args, y_stride));
  printf("%zu %zu %zu %zu\n", sizeof(tri_gate_bwd_args), offsetof(tri_gate_bwd_args, dy_stride),
         offsetof(tri_gate_bwd_args, dwo), offsetof(tri_gate_bwd_args, workspace_bytes));
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
    want = [ctypes.sizeof(B.FwdArgs), B.FwdArgs.q.offset, B.FwdArgs.lse.offset, ctypes.sizeof(B.BwdArgs),
            B.BwdArgs.workspace.offset, B.BwdArgs.flags.offset,
            ctypes.sizeof(B.MulFwdArgs), B.MulFwdArgs.flags.offset, ctypes.sizeof(B.MulBwdArgs),
            B.MulBwdArgs.db.offset, ctypes.sizeof(B.GateFwdArgs), B.GateFwdArgs.y_stride.offset,
            ctypes.sizeof(B.GateBwdArgs), B.GateBwdArgs.dy_stride.offset, B.GateBwdArgs.dwo.offset,
            B.GateBwdArgs.workspace_bytes.offset]
    assert got == want


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    # no fallback of any kind: without the built library every entry point raises
    monkeypatch.setattr(B, "_lib", None)
    monkeypatch.setattr(B, "LIB_PATH", str(tmp_path / "absent" / "libtriattn.so"))
    for call in (lambda: B.tri_attn_bwd_workspace_bytes(1, 64, 2, 32), lambda: B.tri_gate_bwd_workspace_bytes(1),
                 lambda: B.tri_attn_abi_version()):
        with pytest.raises(RuntimeError, match="not found"):
            call()
