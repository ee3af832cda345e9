"""FP64 CPU oracle for triangle attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The product path (the C-ABI library and
its Python binding) never imports, links or executes anything under
``oracle/``; the two share no code.

This is a thin ctypes wrapper around ``tri_attn_oracle.c`` (plain C loops in
FP64, every sum serial in ascending order, OpenMP only across independent
rows).  The C file states the definition it computes and the page passages it
follows:

* "16张H100，训练步提速1.73倍：TurboPairFormer…" (biocloudservice.com blog),
  section "它优化了什么": gradients for query, key, value and the shared pair
  bias.
* "TurboPairFormer: более быстрое, стабильное и точное дообучение OpenFold3"
  (dev48.org), section "Точность": the reference is FP64 on the identical
  BF16 inputs.

Orientation.  Triangle attention around the ending node is the starting-node
definition applied to the pair tensors with axes 1 and 2 swapped, with the
outputs swapped back; bias and mask stay in the attention's own frame (the
caller supplies them that way).  ``ending_*`` below do exactly that.

Every function here is pinned by ``tests/test_oracle_pins.py`` against things
other than itself (a library attention routine, closed forms, invariants,
finite differences, torch autograd on an independent formulation).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tri_attn_oracle.c")
_LIB = os.path.join(_HERE, "libtri_attn_oracle.so")
_lock = threading.Lock()
_lib = None

ORC_OK, ORC_ERR_ARGS, ORC_ERR_FULLY_MASKED, ORC_ERR_NOMEM = 0, 1, 2, 3


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/libtri_attn_oracle.so`` (gcc, -O2,
    no fast-math so IEEE semantics and the serial summation order hold)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
               "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            dp = ctypes.POINTER(ctypes.c_double)
            ip = ctypes.POINTER(ctypes.c_int)
            i, d = ctypes.c_int, ctypes.c_double
            lib.tri_attn_oracle_fwd.argtypes = [i, i, i, i, d, dp, dp, dp, dp, dp, ip, i, dp, dp, i]
            lib.tri_attn_oracle_bwd_rows.argtypes = [i, i, i, i, d, dp, dp, dp, dp, dp, dp, ip, i,
                                                     dp, dp, dp, i]
            lib.tri_attn_oracle_dbias.argtypes = [i, i, i, i, d, dp, dp, dp, dp, dp, dp, ip, i, dp, i]
            lib.tri_attn_oracle_row.argtypes = [i, i, i, d, dp, dp, dp, dp, dp, dp, dp, dp, dp, dp, dp]
            lib.tri_attn_oracle_dbias_row_add.argtypes = [i, i, i, d, dp, dp, dp, dp, dp, dp, i, i, dp]
            lib.tri_attn_oracle_dbias_row_add_all.argtypes = [i, i, i, d, dp, dp, dp, dp, dp, dp, dp]
            for f in (lib.tri_attn_oracle_fwd, lib.tri_attn_oracle_bwd_rows, lib.tri_attn_oracle_dbias,
                      lib.tri_attn_oracle_row, lib.tri_attn_oracle_dbias_row_add,
                      lib.tri_attn_oracle_dbias_row_add_all):
                f.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(x):
    """Any array-like (numpy, torch CPU tensor of any float dtype) -> C-contiguous float64."""
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _rows_arg(rows):
    """(pointer, count, keep-alive array) for an optional list of (b, i) rows."""
    if rows is None:
        return ctypes.POINTER(ctypes.c_int)(), -1, None
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1))
    return r.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), r.size // 2, r


def _check(st):
    if st == ORC_ERR_FULLY_MASKED:
        raise OracleError("a pair row has every key masked: outside the contract")
    if st != ORC_OK:
        raise OracleError(f"oracle failed with status {st}")


def _shape(q):
    B, N, N2, H, d = q.shape
    assert N == N2, "pair tensors must be [B,N,N,H,d]"
    return B, N, H, d


def default_scale(d: int) -> float:
    return 1.0 / float(np.sqrt(d))


def fwd(q, k, v, bias, mask=None, scale=None, rows=None, planted: int = 0):
    """Starting-node forward.  Returns (out [B,N,N,H,d], lse [B,H,N,N]) in FP64.

    ``rows``: optional list of (b, i) pair rows; only those rows are computed
    (the rest of ``out``/``lse`` is NaN)."""
    q, k, v, bias, mask = map(_f64, (q, k, v, bias, mask))
    B, N, H, d = _shape(q)
    scale = default_scale(d) if scale is None else float(scale)
    out = np.full(q.shape, np.nan)
    lse = np.full((B, H, N, N), np.nan)
    rp, nr, _keep = _rows_arg(rows)
    st = _load().tri_attn_oracle_fwd(B, N, H, d, scale, _ptr(q), _ptr(k), _ptr(v), _ptr(bias),
                                     _ptr(mask), rp, nr, _ptr(out), _ptr(lse), int(planted))
    _check(st)
    return out, lse


def bwd_rows(q, k, v, bias, mask, dout, scale=None, rows=None, planted: int = 0):
    """Starting-node dq, dk, dv (FP64) for the given (b, i) rows (all if None)."""
    q, k, v, bias, mask, dout = map(_f64, (q, k, v, bias, mask, dout))
    B, N, H, d = _shape(q)
    scale = default_scale(d) if scale is None else float(scale)
    dq = np.full(q.shape, np.nan)
    dk = np.full(q.shape, np.nan)
    dv = np.full(q.shape, np.nan)
    rp, nr, _keep = _rows_arg(rows)
    st = _load().tri_attn_oracle_bwd_rows(B, N, H, d, scale, _ptr(q), _ptr(k), _ptr(v), _ptr(bias),
                                          _ptr(mask), _ptr(dout), rp, nr, _ptr(dq), _ptr(dk),
                                          _ptr(dv), int(planted))
    _check(st)
    return dq, dk, dv


def dbias(q, k, v, bias, mask, dout, scale=None, sel=None, planted: int = 0):
    """dbias [B,H,N,N] (FP64); ``sel`` optional list of (b, h, j) rows to compute."""
    q, k, v, bias, mask, dout = map(_f64, (q, k, v, bias, mask, dout))
    B, N, H, d = _shape(q)
    scale = default_scale(d) if scale is None else float(scale)
    db = np.full((B, H, N, N), np.nan)
    if sel is None:
        sp, ns, keep = ctypes.POINTER(ctypes.c_int)(), -1, None
    else:
        keep = np.ascontiguousarray(np.asarray(sel, dtype=np.int32).reshape(-1))
        sp, ns = keep.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), keep.size // 3
    st = _load().tri_attn_oracle_dbias(B, N, H, d, scale, _ptr(q), _ptr(k), _ptr(v), _ptr(bias),
                                       _ptr(mask), _ptr(dout), sp, ns, _ptr(db), int(planted))
    _check(st)
    return db


def bwd(q, k, v, bias, mask, dout, scale=None, planted: int = 0):
    """Full starting-node backward: (dq, dk, dv, dbias) in FP64."""
    dq, dk, dv = bwd_rows(q, k, v, bias, mask, dout, scale, None, planted)
    db = dbias(q, k, v, bias, mask, dout, scale, None, planted)
    return dq, dk, dv, db


# ---- one pair row at a time (crops whose pair stack is too large for FP64 on the host) ----

def row(q_row, k_row, v_row, bias_b, mask_row=None, dout_row=None, scale=None):
    """Pair row (b,i) alone: q_row, k_row, v_row, dout_row are that row's [N,H,d],
    bias_b the batch's [H,N,N], mask_row its [N] (or None).  Returns out [N,H,d],
    lse [H,N] and, with dout_row, dq, dk, dv [N,H,d] -- the same arithmetic as
    ``fwd``/``bwd_rows`` on that row (equal bit for bit)."""
    q_row, k_row, v_row, bias_b, mask_row, dout_row = map(_f64, (q_row, k_row, v_row, bias_b, mask_row, dout_row))
    N, H, d = q_row.shape
    assert k_row.shape == v_row.shape == (N, H, d) and bias_b.shape == (H, N, N)
    scale = default_scale(d) if scale is None else float(scale)
    out = np.full((N, H, d), np.nan)
    lse = np.full((H, N), np.nan)
    grads = dout_row is not None
    dq, dk, dv = ((np.full((N, H, d), np.nan) for _ in range(3)) if grads else (None, None, None))
    st = _load().tri_attn_oracle_row(N, H, d, scale, _ptr(q_row), _ptr(k_row), _ptr(v_row), _ptr(bias_b),
                                     _ptr(mask_row), _ptr(dout_row), _ptr(out), _ptr(lse), _ptr(dq), _ptr(dk),
                                     _ptr(dv))
    _check(st)
    return (out, lse, dq, dk, dv) if grads else (out, lse)


def dbias_streamed(get_row, bias_b, h, j, scale=None):
    """dbias[b,h,j,:] as the ascending sum over rows i of ds[b,i,j,h,:], fetching one
    row at a time: ``get_row(i)`` returns (q_row, k_row, v_row, mask_row, dout_row)
    of row i.  Same FP64 operations and order as ``dbias`` (equal bit for bit)."""
    bias_b = _f64(bias_b)
    H, N, _ = bias_b.shape
    acc = np.zeros(N)
    lib = _load()
    for i in range(N):
        q_row, k_row, v_row, mask_row, dout_row = map(_f64, get_row(i))
        d = q_row.shape[2]
        sc = default_scale(d) if scale is None else float(scale)
        st = lib.tri_attn_oracle_dbias_row_add(N, H, d, sc, _ptr(q_row), _ptr(k_row), _ptr(v_row), _ptr(bias_b),
                                               _ptr(mask_row), _ptr(dout_row), int(h), int(j), _ptr(acc))
        _check(st)
    return acc


def dbias_add_row(acc, q_row, k_row, v_row, bias_b, mask_row, dout_row, scale=None):
    """Add pair row i's ds[b,i,j,h,:] for every (h, j) into acc ([H,N,N] FP64, in
    place).  Over all rows in ascending order this equals ``dbias`` for the batch
    bit for bit."""
    q_row, k_row, v_row, bias_b, mask_row, dout_row = map(_f64, (q_row, k_row, v_row, bias_b, mask_row, dout_row))
    N, H, d = q_row.shape
    assert acc.dtype == np.float64 and acc.shape == (H, N, N) and acc.flags.c_contiguous
    scale = default_scale(d) if scale is None else float(scale)
    st = _load().tri_attn_oracle_dbias_row_add_all(N, H, d, scale, _ptr(q_row), _ptr(k_row), _ptr(v_row),
                                                   _ptr(bias_b), _ptr(mask_row), _ptr(dout_row), _ptr(acc))
    _check(st)
    return acc


# ---- ending-node orientation: swap pair axes 1 and 2 around the starting-node definition ----

def _swap(x):
    return None if x is None else np.ascontiguousarray(np.swapaxes(_f64(x), 1, 2))


def ending_fwd(q, k, v, bias, mask=None, scale=None):
    out, lse = fwd(_swap(q), _swap(k), _swap(v), bias, mask, scale)
    return _swap(out), lse


def ending_bwd(q, k, v, bias, mask, dout, scale=None):
    dq, dk, dv, db = bwd(_swap(q), _swap(k), _swap(v), bias, mask, _swap(dout), scale)
    return _swap(dq), _swap(dk), _swap(dv), db
