"""ctypes binding of libtriattn.so (include/tri_attn.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI.  PyTorch tensors supply device memory and the
stream; their data pointers and element strides are copied into the C
argument structs.  If the shared library is missing the first call raises --
there is no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os
import struct
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtriattn.so")

TRI_ATTN_OK = 0
TRI_ATTN_ERR_NULL = 1
TRI_ATTN_ERR_SHAPE = 2
TRI_ATTN_ERR_STRIDE = 3
TRI_ATTN_ERR_ALIGN = 4
TRI_ATTN_ERR_DTYPE = 5
TRI_ATTN_ERR_UNSUPPORTED = 6
TRI_ATTN_ERR_WORKSPACE = 7
TRI_ATTN_ERR_ARCH = 8
TRI_ATTN_ERR_CUDA = 9
TRI_ATTN_ERR_DEVICE_TIMEOUT = 10
TRI_ATTN_ERR_SCRATCH_LIMIT = 11
TRI_ATTN_STATIC_SCRATCH_BYTES = 64 << 20
TRI_ATTN_BWD_NO_RESIDUAL = 1


class TriAttnError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = int(status)
        msg = tri_attn_strerror(self.status) if _lib is not None else f"status {status}"
        super().__init__(f"{where}: {msg} (status {self.status})" if where else msg)


class Tensor5(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("stride", ctypes.c_int64 * 5)]


class Tensor4(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("stride", ctypes.c_int64 * 4)]


class Mask(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("stride", ctypes.c_int64 * 3)]


class FwdArgs(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("N", ctypes.c_int), ("H", ctypes.c_int), ("d", ctypes.c_int),
                ("scale", ctypes.c_float),
                ("q", Tensor5), ("k", Tensor5), ("v", Tensor5), ("bias", Tensor4), ("mask", Mask),
                ("o", Tensor5), ("resid", Tensor5), ("lse", ctypes.c_void_p)]


class MulFwdArgs(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("C", ctypes.c_int), ("N", ctypes.c_int), ("a", Tensor4), ("b", Tensor4),
                ("x", Tensor4), ("flags", ctypes.c_uint)]


class GateFwdArgs(ctypes.Structure):
    _fields_ = [("R", ctypes.c_int), ("z", ctypes.c_void_p), ("z_stride", ctypes.c_int64), ("o", ctypes.c_void_p),
                ("o_stride", ctypes.c_int64), ("wg", ctypes.c_void_p), ("wo", ctypes.c_void_p), ("y", ctypes.c_void_p),
                ("y_stride", ctypes.c_int64)]


class GateBwdArgs(ctypes.Structure):
    _fields_ = [("f", GateFwdArgs), ("dy", ctypes.c_void_p), ("dy_stride", ctypes.c_int64), ("dz", ctypes.c_void_p),
                ("dz_stride", ctypes.c_int64), ("d_o", ctypes.c_void_p), ("do_stride", ctypes.c_int64),
                ("dwg", ctypes.c_void_p), ("dwo", ctypes.c_void_p), ("workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_size_t)]


class MulBwdArgs(ctypes.Structure):
    _fields_ = [("f", MulFwdArgs), ("dx", Tensor4), ("da", Tensor4), ("db", Tensor4)]


class BwdArgs(ctypes.Structure):
    _fields_ = [("f", FwdArgs), ("dout", Tensor5), ("dq", Tensor5), ("dk", Tensor5), ("dv", Tensor5),
                ("dbias", Tensor4), ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
                ("flags", ctypes.c_uint)]


# The same two argument blocks as flat little-endian layouts (explicit padding), so a
# call fills one buffer with a single pack instead of building a ctypes structure per
# tensor; checked against the ctypes structures above at import.
_FWD_PACK = struct.Struct("<4if4x" + "Q5q" * 3 + "Q4q" + "Q3q" + "Q5q" * 2 + "Q")
_BWD_TAIL = struct.Struct("<" + "Q5q" * 4 + "Q4q" + "QQi4x")
assert _FWD_PACK.size == ctypes.sizeof(FwdArgs) and FwdArgs.lse.offset == _FWD_PACK.size - 8
assert _FWD_PACK.size + _BWD_TAIL.size == ctypes.sizeof(BwdArgs) and BwdArgs.dout.offset == _FWD_PACK.size


_lib = None
_lock = threading.Lock()


def load() -> ctypes.CDLL:
    """Load libtriattn.so (built in-tree by build.py); raise if it is missing."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"libtriattn.so not found at {LIB_PATH}; build it with "
                    "`python -m triangle_attention_biomolecular_b200.build`")
            lib = ctypes.CDLL(LIB_PATH)
            lib.tri_attn_fwd.argtypes = [ctypes.POINTER(FwdArgs), ctypes.c_void_p]
            lib.tri_attn_fwd.restype = ctypes.c_int
            lib.tri_attn_bwd.argtypes = [ctypes.POINTER(BwdArgs), ctypes.c_void_p]
            lib.tri_attn_bwd.restype = ctypes.c_int
            lib.tri_attn_bwd_marked.argtypes = [ctypes.POINTER(BwdArgs), ctypes.c_void_p,
                                                ctypes.POINTER(ctypes.c_void_p)]
            lib.tri_attn_bwd_marked.restype = ctypes.c_int
            lib.tri_gate_fwd.argtypes = [ctypes.POINTER(GateFwdArgs), ctypes.c_void_p]
            lib.tri_gate_fwd.restype = ctypes.c_int
            lib.tri_gate_bwd.argtypes = [ctypes.POINTER(GateBwdArgs), ctypes.c_void_p]
            lib.tri_gate_bwd.restype = ctypes.c_int
            lib.tri_gate_bwd_workspace_bytes.argtypes = [ctypes.c_int]
            lib.tri_gate_bwd_workspace_bytes.restype = ctypes.c_size_t
            lib.tri_mul_fwd.argtypes = [ctypes.POINTER(MulFwdArgs), ctypes.c_void_p]
            lib.tri_mul_fwd.restype = ctypes.c_int
            lib.tri_mul_bwd.argtypes = [ctypes.POINTER(MulBwdArgs), ctypes.c_void_p]
            lib.tri_mul_bwd.restype = ctypes.c_int
            lib.tri_attn_bwd_static_scratch.argtypes = [ctypes.POINTER(BwdArgs), ctypes.c_void_p]
            lib.tri_attn_bwd_static_scratch.restype = ctypes.c_int
            lib.tri_attn_bwd_workspace_bytes.argtypes = [ctypes.c_int] * 4
            lib.tri_attn_bwd_workspace_bytes.restype = ctypes.c_size_t
            lib.tri_attn_fwd_rows.argtypes = [ctypes.POINTER(FwdArgs), ctypes.c_int, ctypes.c_void_p]
            lib.tri_attn_fwd_rows.restype = ctypes.c_int
            lib.tri_attn_bwd_rows.argtypes = [ctypes.POINTER(BwdArgs), ctypes.c_int, ctypes.c_void_p,
                                              ctypes.c_void_p]
            lib.tri_attn_bwd_rows.restype = ctypes.c_int
            lib.tri_attn_bwd_rows_workspace_bytes.argtypes = [ctypes.c_int] * 5
            lib.tri_attn_bwd_rows_workspace_bytes.restype = ctypes.c_size_t
            lib.tri_attn_bwd_rows_dbias_parts.argtypes = [ctypes.c_int] * 5
            lib.tri_attn_bwd_rows_dbias_parts.restype = ctypes.c_int
            lib.tri_attn_dbias_sum.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int, Tensor4, ctypes.c_void_p]
            lib.tri_attn_dbias_sum.restype = ctypes.c_int
            lib.tri_attn_strerror.argtypes = [ctypes.c_int]
            lib.tri_attn_strerror.restype = ctypes.c_char_p
            lib.tri_attn_device_error.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_uint32)]
            lib.tri_attn_device_error.restype = ctypes.c_int
            lib.tri_attn_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
            lib.tri_attn_set_wait_limit_ns.restype = None
            lib.tri_attn_selftest_expire_wait.argtypes = [ctypes.c_void_p]
            lib.tri_attn_selftest_expire_wait.restype = ctypes.c_int
            lib.tri_attn_abi_version.argtypes = []
            lib.tri_attn_abi_version.restype = ctypes.c_int
            _lib = lib
    return _lib


# ---------------------------------------------------------------------------
# marshalling helpers (torch tensors -> C structs)
# ---------------------------------------------------------------------------

def _check_tensor(t, name, dtype, dims):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TriAttnError(TRI_ATTN_ERR_DTYPE, f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != dims:
        raise TriAttnError(TRI_ATTN_ERR_SHAPE, f"{name} must have {dims} dims")


_I64x5, _I64x4, _I64x3 = ctypes.c_int64 * 5, ctypes.c_int64 * 4, ctypes.c_int64 * 3


def t5(t, name="tensor") -> Tensor5:
    import torch
    _check_tensor(t, name, torch.bfloat16, 5)
    return Tensor5(t.data_ptr(), _I64x5(*t.stride()))


def t4(t, name="bias") -> Tensor4:
    import torch
    _check_tensor(t, name, torch.bfloat16, 4)
    return Tensor4(t.data_ptr(), _I64x4(*t.stride()))


def mask3(m) -> Mask:
    import torch
    if m is None:
        return Mask()
    _check_tensor(m, "mask", torch.float32, 3)
    return Mask(m.data_ptr(), _I64x3(*m.stride()))


def _stream_handle(stream):
    import torch
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def fwd_args(q, k, v, bias, mask, o, resid, lse, scale: float = 0.0, rows_ok: bool = False,
             _room: bool = False) -> FwdArgs:
    """Pair tensors [B,R,N,H,d]: R = N for the whole problem; with rows_ok, R <= N rows
    of a row shard (views starting at its first row), lse [B,H,R,N], mask [B,R,N]."""
    import torch
    B, R, N, H, d = q.shape
    if R != N and not (rows_ok and 1 <= R <= N):
        raise TriAttnError(TRI_ATTN_ERR_SHAPE, "q must be [B,N,N,H,d]")
    for name, t in (("k", k), ("v", v), ("o", o), ("resid", resid)):
        if tuple(t.shape) != (B, R, N, H, d):
            raise TriAttnError(TRI_ATTN_ERR_SHAPE, f"{name} shape {tuple(t.shape)} != {(B, R, N, H, d)}")
    if tuple(bias.shape) != (B, H, N, N):
        raise TriAttnError(TRI_ATTN_ERR_SHAPE, "bias must be [B,H,N,N]")
    if mask is not None and tuple(mask.shape) != (B, R, N):
        raise TriAttnError(TRI_ATTN_ERR_SHAPE, "mask must be [B,N,N] (b,i,k)")
    _check_tensor(lse, "lse", torch.float32, 4)
    if tuple(lse.shape) != (B, H, R, N) or not lse.is_contiguous():
        raise TriAttnError(TRI_ATTN_ERR_SHAPE, "lse must be a contiguous [B,H,N,N] float32 tensor")
    buf = bytearray(ctypes.sizeof(BwdArgs) if _room else _FWD_PACK.size)
    _pack_fwd(buf, B, N, H, d, scale, q, k, v, bias, mask, o, resid, lse)
    return buf if _room else FwdArgs.from_buffer(buf)


def _v5(t, name):
    import torch
    _check_tensor(t, name, torch.bfloat16, 5)
    return (t.data_ptr(), *t.stride())


def _v4(t, name):
    import torch
    _check_tensor(t, name, torch.bfloat16, 4)
    return (t.data_ptr(), *t.stride())


def _pack_fwd(buf, B, N, H, d, scale, q, k, v, bias, mask, o, resid, lse):
    import torch
    if mask is None:
        vm = (0, 0, 0, 0)
    else:
        _check_tensor(mask, "mask", torch.float32, 3)
        vm = (mask.data_ptr(), *mask.stride())
    _FWD_PACK.pack_into(buf, 0, B, N, H, d, float(scale), *_v5(q, "q"), *_v5(k, "k"), *_v5(v, "v"),
                        *_v4(bias, "bias"), *vm, *_v5(o, "o"), *_v5(resid, "resid"), lse.data_ptr())


# ---------------------------------------------------------------------------
# the C entry points, same names
# ---------------------------------------------------------------------------

def tri_attn_strerror(status: int) -> str:
    return load().tri_attn_strerror(int(status)).decode()


def tri_attn_abi_version() -> int:
    return load().tri_attn_abi_version()


def tri_attn_bwd_workspace_bytes(B: int, N: int, H: int, d: int) -> int:
    return int(load().tri_attn_bwd_workspace_bytes(B, N, H, d))


def tri_attn_fwd(q, k, v, bias, mask, o, resid, lse, scale: float = 0.0, stream=None) -> None:
    """Enqueue the forward; o, resid (BF16) and lse (FP32 [B,H,N,N]) are written."""
    a = fwd_args(q, k, v, bias, mask, o, resid, lse, scale)
    st = load().tri_attn_fwd(ctypes.byref(a), _stream_handle(stream))
    if st != TRI_ATTN_OK:
        raise TriAttnError(st, "tri_attn_fwd")


def bwd_args(q, k, v, bias, mask, o, resid, lse, dout, dq, dk, dv, dbias, workspace,
             scale: float = 0.0, flags: int = 0, rows_ok: bool = False) -> BwdArgs:
    import torch
    buf = fwd_args(q, k, v, bias, mask, o, resid, lse, scale, rows_ok, _room=True)
    shape = q.shape
    for name, t in (("dout", dout), ("dq", dq), ("dk", dk), ("dv", dv)):
        if t.shape != shape:
            raise TriAttnError(TRI_ATTN_ERR_SHAPE, f"{name} shape {tuple(t.shape)} != {tuple(shape)}")
    vb = (0, 0, 0, 0, 0) if dbias is None else _v4(dbias, "dbias")
    if workspace is None:
        ws = (0, 0)
    else:
        if workspace.dtype != torch.uint8:
            raise TriAttnError(TRI_ATTN_ERR_DTYPE, "workspace must be a uint8 tensor")
        ws = (workspace.data_ptr(), workspace.numel())
    _BWD_TAIL.pack_into(buf, _FWD_PACK.size, *_v5(dout, "dout"), *_v5(dq, "dq"), *_v5(dk, "dk"), *_v5(dv, "dv"),
                        *vb, *ws, int(flags))
    return BwdArgs.from_buffer(buf)


def tri_attn_bwd(q, k, v, bias, mask, o, resid, lse, dout, dq, dk, dv, dbias, workspace,
                 scale: float = 0.0, flags: int = 0, stream=None) -> None:
    """Enqueue the backward; dq, dk, dv, dbias (BF16) are written.  workspace is a
    caller-owned uint8 CUDA tensor of at least tri_attn_bwd_workspace_bytes bytes."""
    a = bwd_args(q, k, v, bias, mask, o, resid, lse, dout, dq, dk, dv, dbias, workspace, scale, flags)
    st = load().tri_attn_bwd(ctypes.byref(a), _stream_handle(stream))
    if st != TRI_ATTN_OK:
        raise TriAttnError(st, "tri_attn_bwd")


def tri_attn_bwd_marked(q, k, v, bias, mask, o, resid, lse, dout, dq, dk, dv, dbias, workspace,
                        markers, scale: float = 0.0, flags: int = 0, stream=None) -> None:
    """tri_attn_bwd recording four caller-owned torch.cuda.Event markers between
    its phases (D pre-pass | dq/dk/dv | dbias | end)."""
    a = bwd_args(q, k, v, bias, mask, o, resid, lse, dout, dq, dk, dv, dbias, workspace, scale, flags)
    arr = (ctypes.c_void_p * 4)(*[ctypes.c_void_p(int(ev.cuda_event)) for ev in markers])
    st = load().tri_attn_bwd_marked(ctypes.byref(a), _stream_handle(stream), arr)
    if st != TRI_ATTN_OK:
        raise TriAttnError(st, "tri_attn_bwd_marked")


def tri_attn_bwd_static_scratch(q, k, v, bias, mask, o, resid, lse, dout, dq, dk, dv, dbias,
                                scale: float = 0.0, flags: int = 0, stream=None) -> None:
    """tri_attn_bwd without a workspace argument: the library's fixed per-device
    scratch array is used instead, so nothing is allocated.  Calls on one device
    share that array and must not overlap on the device."""
    a = bwd_args(q, k, v, bias, mask, o, resid, lse, dout, dq, dk, dv, dbias, None, scale, flags)
    st = load().tri_attn_bwd_static_scratch(ctypes.byref(a), _stream_handle(stream))
    if st != TRI_ATTN_OK:
        raise TriAttnError(st, "tri_attn_bwd_static_scratch")


def tri_attn_bwd_rows_workspace_bytes(B: int, rows: int, N: int, H: int, d: int) -> int:
    return int(load().tri_attn_bwd_rows_workspace_bytes(B, rows, N, H, d))


def tri_attn_bwd_rows_dbias_parts(B: int, rows: int, N: int, H: int, d: int) -> int:
    return int(load().tri_attn_bwd_rows_dbias_parts(B, rows, N, H, d))


def tri_attn_fwd_rows(q, k, v, bias, mask, o, resid, lse, scale: float = 0.0, stream=None) -> None:
    """Forward of a row shard: pair tensors are [B,R,N,H,d] views starting at the shard's
    first row (mask [B,R,N] likewise), bias the full [B,H,N,N], lse its own [B,H,R,N]."""
    a = fwd_args(q, k, v, bias, mask, o, resid, lse, scale, rows_ok=True)
    st = load().tri_attn_fwd_rows(ctypes.byref(a), q.shape[1], _stream_handle(stream))
    if st != TRI_ATTN_OK:
        raise TriAttnError(st, "tri_attn_fwd_rows")


def tri_attn_bwd_rows(q, k, v, bias, mask, o, resid, lse, dout, dq, dk, dv, dbias_parts, workspace,
                      scale: float = 0.0, flags: int = 0, stream=None) -> None:
    """Backward of a row shard: dq, dk, dv of its rows and its share of dBias as
    FP32 partial sums, dbias_parts a contiguous float32 [P,B,H,N,N] tensor with
    P = tri_attn_bwd_rows_dbias_parts(...)."""
    import torch
    a = bwd_args(q, k, v, bias, mask, o, resid, lse, dout, dq, dk, dv, None, workspace, scale, flags,
                 rows_ok=True)
    B, R, N, H, d = q.shape
    P = tri_attn_bwd_rows_dbias_parts(B, R, N, H, d)
    if (dbias_parts.dtype != torch.float32 or not dbias_parts.is_contiguous()
            or tuple(dbias_parts.shape) != (P, B, H, N, N)):
        raise TriAttnError(TRI_ATTN_ERR_SHAPE, f"dbias_parts must be a contiguous float32 {(P, B, H, N, N)} tensor")
    st = load().tri_attn_bwd_rows(ctypes.byref(a), R, ctypes.c_void_p(dbias_parts.data_ptr()),
                                  _stream_handle(stream))
    if st != TRI_ATTN_OK:
        raise TriAttnError(st, "tri_attn_bwd_rows")


def tri_attn_dbias_sum(parts, dbias, stream=None) -> None:
    """dbias (BF16 [B,H,N,N]) = sum over the first axis of parts (contiguous float32
    [P,B,H,N,N]), added in ascending index order."""
    import torch
    if parts.dtype != torch.float32 or not parts.is_contiguous() or parts.dim() != 5:
        raise TriAttnError(TRI_ATTN_ERR_SHAPE, "parts must be a contiguous float32 [P,B,H,N,N] tensor")
    P, B, H, N, N2 = parts.shape
    if N2 != N or tuple(dbias.shape) != (B, H, N, N):
        raise TriAttnError(TRI_ATTN_ERR_SHAPE, "dbias must be [B,H,N,N] matching parts")
    st = load().tri_attn_dbias_sum(ctypes.c_void_p(parts.data_ptr()), P, B, H, N, t4(dbias, "dbias"),
                                   _stream_handle(stream))
    if st != TRI_ATTN_OK:
        raise TriAttnError(st, "tri_attn_dbias_sum")


TRI_MUL_INCOMING = 1


def _mul_args(a, b, x, incoming: bool) -> MulFwdArgs:
    B, C, N, N2 = a.shape
    if N2 != N or tuple(b.shape) != (B, C, N, N):
        raise TriAttnError(TRI_ATTN_ERR_SHAPE, "a and b must both be [B,C,N,N]")
    m = MulFwdArgs()
    m.B, m.C, m.N = B, C, N
    m.a, m.b = t4(a, "a"), t4(b, "b")
    if x is not None:
        m.x = t4(x, "x")
    m.flags = TRI_MUL_INCOMING if incoming else 0
    return m


def tri_mul_fwd(a, b, x, incoming: bool = False, stream=None) -> None:
    """x[b,c,i,j] = sum_k a[b,c,i,k] b[b,c,j,k] (outgoing) or sum_k a[b,c,k,i] b[b,c,k,j]
    (incoming); BF16 [B,C,N,N] CUDA tensors, x written."""
    m = _mul_args(a, b, x, incoming)
    st = load().tri_mul_fwd(ctypes.byref(m), _stream_handle(stream))
    if st != TRI_ATTN_OK:
        raise TriAttnError(st, "tri_mul_fwd")


def tri_mul_bwd(a, b, dx, da, db, incoming: bool = False, stream=None) -> None:
    """Gradients da, db of the contraction for the upstream gradient dx (all BF16 [B,C,N,N])."""
    m = MulBwdArgs()
    m.f = _mul_args(a, b, None, incoming)
    m.dx, m.da, m.db = t4(dx, "dx"), t4(da, "da"), t4(db, "db")
    st = load().tri_mul_bwd(ctypes.byref(m), _stream_handle(stream))
    if st != TRI_ATTN_OK:
        raise TriAttnError(st, "tri_mul_bwd")


def tri_gate_fwd(z, o, wg, wo, y, stream=None) -> None:
    """y = (sigmoid(z wg) * o) wo row by row; z, o, y BF16 [R, 128] (rows may be padded),
    wg, wo BF16 [128, 128] contiguous."""
    import torch
    for t, n in ((z, "z"), (o, "o"), (y, "y"), (wg, "wg"), (wo, "wo")):
        if t.dtype != torch.bfloat16 or t.dim() != 2 or t.shape[1] != 128 or t.stride(1) != 1:
            raise TriAttnError(TRI_ATTN_ERR_DTYPE, f"{n} must be a BF16 [*, 128] tensor with unit column stride")
    if wg.shape[0] != 128 or wo.shape[0] != 128 or not wg.is_contiguous() or not wo.is_contiguous():
        raise TriAttnError(TRI_ATTN_ERR_SHAPE, "wg and wo must be contiguous [128, 128]")
    if o.shape[0] != z.shape[0] or y.shape[0] != z.shape[0]:
        raise TriAttnError(TRI_ATTN_ERR_SHAPE, "z, o and y must have the same number of rows")
    a = GateFwdArgs()
    a.R = z.shape[0]
    a.z, a.z_stride = z.data_ptr(), z.stride(0)
    a.o, a.o_stride = o.data_ptr(), o.stride(0)
    a.wg, a.wo = wg.data_ptr(), wo.data_ptr()
    a.y, a.y_stride = y.data_ptr(), y.stride(0)
    st = load().tri_gate_fwd(ctypes.byref(a), _stream_handle(stream))
    if st != TRI_ATTN_OK:
        raise TriAttnError(st, "tri_gate_fwd")


def _check_rows128(ts, names):
    import torch
    for t, n in zip(ts, names):
        if t.dtype != torch.bfloat16 or t.dim() != 2 or t.shape[1] != 128 or t.stride(1) != 1:
            raise TriAttnError(TRI_ATTN_ERR_DTYPE, f"{n} must be a BF16 [*, 128] tensor with unit column stride")


def tri_gate_bwd_workspace_bytes(R: int) -> int:
    return int(load().tri_gate_bwd_workspace_bytes(R))


def tri_gate_bwd(z, o, wg, wo, dy, dz, d_o, dwg, dwo, workspace, stream=None) -> None:
    """Gradients of y = (sigmoid(z wg) * o) wo for the upstream dy: dz, d_o BF16 [R, 128]
    (rows may be padded), dwg, dwo FP32 [128, 128] contiguous, workspace a uint8 CUDA
    tensor of at least tri_gate_bwd_workspace_bytes(R) bytes."""
    import torch
    _check_rows128((z, o, dy, dz, d_o, wg, wo), ("z", "o", "dy", "dz", "d_o", "wg", "wo"))
    if wg.shape[0] != 128 or wo.shape[0] != 128 or not wg.is_contiguous() or not wo.is_contiguous():
        raise TriAttnError(TRI_ATTN_ERR_SHAPE, "wg and wo must be contiguous [128, 128]")
    for t, n in ((dwg, "dwg"), (dwo, "dwo")):
        if t.dtype != torch.float32 or tuple(t.shape) != (128, 128) or not t.is_contiguous():
            raise TriAttnError(TRI_ATTN_ERR_DTYPE, f"{n} must be a contiguous FP32 [128, 128] tensor")
    R = z.shape[0]
    if any(t.shape[0] != R for t in (o, dy, dz, d_o)):
        raise TriAttnError(TRI_ATTN_ERR_SHAPE, "z, o, dy, dz and d_o must have the same number of rows")
    a = GateBwdArgs()
    a.f.R = R
    a.f.z, a.f.z_stride = z.data_ptr(), z.stride(0)
    a.f.o, a.f.o_stride = o.data_ptr(), o.stride(0)
    a.f.wg, a.f.wo = wg.data_ptr(), wo.data_ptr()
    a.f.y, a.f.y_stride = None, 128
    a.dy, a.dy_stride = dy.data_ptr(), dy.stride(0)
    a.dz, a.dz_stride = dz.data_ptr(), dz.stride(0)
    a.d_o, a.do_stride = d_o.data_ptr(), d_o.stride(0)
    a.dwg, a.dwo = dwg.data_ptr(), dwo.data_ptr()
    a.workspace, a.workspace_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    st = load().tri_gate_bwd(ctypes.byref(a), _stream_handle(stream))
    if st != TRI_ATTN_OK:
        raise TriAttnError(st, "tri_gate_bwd")


def tri_attn_device_error(clear: bool = True):
    """(status, raw word) of the device error word; synchronises the device."""
    w = ctypes.c_uint32(0)
    st = load().tri_attn_device_error(1 if clear else 0, ctypes.byref(w))
    return int(st), int(w.value)


def tri_attn_set_wait_limit_ns(ns: int) -> None:
    load().tri_attn_set_wait_limit_ns(int(ns))


def tri_attn_selftest_expire_wait(stream=None) -> None:
    st = load().tri_attn_selftest_expire_wait(_stream_handle(stream))
    if st != TRI_ATTN_OK:
        raise TriAttnError(st, "tri_attn_selftest_expire_wait")
