"""Python handle on the fp64 CPU oracle (``sdl_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``, never by the library.  It shares no
code with the GPU path; its inputs come from :mod:`synth` (host build).

Every function takes numpy arrays laid out [B, L, heads, d] (uint16 holding
bf16 bits, or float32) and returns float64 results.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(block-sparse path) and ``tests/test_oracle_col_pins.py`` (the column-sparse
path of the PulseCol abstract) against closed forms, invariants, brute force or
an independent library routine.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libsdl_oracle.so")
_SRC = os.path.join(_HERE, "sdl_oracle.c")


def build(force=False):
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-o", _SO, _SRC, "-lm",
                               "-lpthread"])


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int
_L = ctypes.c_int64
_D = ctypes.c_double


def lib():
    global _lib
    if _lib is None:
        build()
        l = ctypes.CDLL(_SO)
        l.oracle_budget.argtypes = [_I, _I, _D]
        l.oracle_budget.restype = _L
        l.oracle_pool.argtypes = [_P, _I, _I, _I, _I, _I, _I, _P, _P]
        l.oracle_block_scores.argtypes = [_P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _D, _P]
        l.oracle_select.argtypes = [_P, _I, _I, _I, _D, _P, _P]
        l.oracle_select.restype = _L
        l.oracle_attention.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P,
                                       _D, _P, _L, _P, _P, _I]
        l.oracle_col_budget.argtypes = [_I, _D]
        l.oracle_col_budget.restype = _L
        l.oracle_col_scores.argtypes = [_P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _D, _P]
        l.oracle_col_select.argtypes = [_P, _I, _I, _I, _D, _P]
        l.oracle_col_select.restype = _L
        l.oracle_col_attention.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P,
                                           _I, _D, _P, _L, _P, _P, _I]
        _lib = l
    return _lib


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.uint16:
        return 0
    if a.dtype == np.float32:
        return 1
    raise TypeError(f"oracle inputs are uint16 (bf16 bits) or float32, got {a.dtype}")


def _strides(a: np.ndarray) -> np.ndarray:
    assert a.ndim == 4 and a.strides[3] == a.itemsize, "head dim must be contiguous"
    return np.array([a.strides[0] // a.itemsize, a.strides[1] // a.itemsize,
                     a.strides[2] // a.itemsize], dtype=np.int64)


def widen(a: np.ndarray) -> np.ndarray:
    """Exact fp64 values of a bf16-bits or fp32 array."""
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def budget(H: int, nb: int, sparsity: float) -> int:
    """Blocks kept per batch element, or -1 when invalid."""
    return int(lib().oracle_budget(H, nb, float(sparsity)))


def pool(x: np.ndarray, bs: int) -> np.ndarray:
    B, L, Hx, d = x.shape
    out = np.empty((B, Hx, L // bs, d), dtype=np.float64)
    st = _strides(x)
    rc = lib().oracle_pool(x.ctypes.data, _dtype_code(x), B, L, Hx, d, bs, st.ctypes.data,
                           out.ctypes.data)
    if rc:
        raise ValueError("oracle_pool rejected its arguments")
    return out


def block_scores(q: np.ndarray, k: np.ndarray, bs: int, scale: float | None = None) -> np.ndarray:
    B, L, H, d = q.shape
    Hkv = k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    nb = L // bs
    out = np.empty((B, H, nb, nb), dtype=np.float64)
    qs, ks = _strides(q), _strides(k)
    rc = lib().oracle_block_scores(q.ctypes.data, k.ctypes.data, _dtype_code(q), B, H, Hkv, L, d,
                                   bs, qs.ctypes.data, ks.ctypes.data, float(scale),
                                   out.ctypes.data)
    if rc:
        raise ValueError("oracle_block_scores rejected its arguments")
    return out


def select(P: np.ndarray, sparsity: float, per_head: bool = False):
    """(mask uint8 [B,H,nb,nb], tau float64 [B] (or [B*H] per head), kept blocks).

    per_head: the uniform per-head budget of the prior methods the Step-dLLM abstract
    compares against (SparseD abstract): the same selection rule applied to every head
    as a sequence of its own."""
    P = np.ascontiguousarray(P, dtype=np.float64)
    if per_head:
        B0, H0, nb0, _ = P.shape
        m, tau, kept = select(P.reshape(B0 * H0, 1, nb0, nb0), sparsity)
        return m.reshape(B0, H0, nb0, nb0), tau, kept
    B, H, nb, _ = P.shape
    mask = np.empty(P.shape, dtype=np.uint8)
    tau = np.empty(B, dtype=np.float64)
    kept = lib().oracle_select(P.ctypes.data, B, H, nb, float(sparsity), mask.ctypes.data,
                               tau.ctypes.data)
    if kept < 0:
        raise ValueError("oracle_select: sparsity outside [0,1) or budget below the diagonal")
    return mask, tau, int(kept)


def attention(q, k, v, bs, mask=None, scale=None, rows=None, nthreads=None):
    """O [n_rows, d] and LSE [n_rows]; rows = int64 [n, 3] of (b, h, t) or None for all
    (then O is returned as [B, H, L, d] and LSE as [B, H, L])."""
    B, L, H, d = q.shape
    Hkv = k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    code = _dtype_code(q)
    assert _dtype_code(k) == code and _dtype_code(v) == code
    if mask is not None:
        mask = np.ascontiguousarray(mask, dtype=np.uint8)
        assert mask.shape == (B, H, L // bs, L // bs)
    if rows is not None:
        rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
        n = rows.shape[0]
    else:
        n = B * H * L
    O = np.empty((n, d), dtype=np.float64)
    lse = np.empty(n, dtype=np.float64)
    qs, ks, vs = _strides(q), _strides(k), _strides(v)
    rc = lib().oracle_attention(q.ctypes.data, k.ctypes.data, v.ctypes.data, code, B, H, Hkv, L,
                                d, bs, qs.ctypes.data, ks.ctypes.data, vs.ctypes.data,
                                None if mask is None else mask.ctypes.data, float(scale),
                                None if rows is None else rows.ctypes.data, n, O.ctypes.data,
                                lse.ctypes.data, nthreads or os.cpu_count() or 1)
    if rc:
        raise ValueError("oracle_attention rejected its arguments")
    if rows is None:
        return O.reshape(B, H, L, d), lse.reshape(B, H, L)
    return O, lse


# ------------------------------------------------ column-sparse (PulseCol)

def col_budget(L: int, sparsity: float) -> int:
    """Columns kept per head: 64 * floor((1 - s) * L / 64 + 0.5), at least 64 (-1 if invalid)."""
    return int(lib().oracle_col_budget(int(L), float(sparsity)))


def col_scores(q: np.ndarray, k: np.ndarray, bs: int, scale: float | None = None) -> np.ndarray:
    """S[b, h, u]: the mean over query blocks of softmax_u(scale * Qbar . k_u), fp64 [B, H, L]."""
    B, L, H, d = q.shape
    Hkv = k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    code = _dtype_code(q)
    assert _dtype_code(k) == code
    S = np.empty((B, H, L), dtype=np.float64)
    qs, ks = _strides(q), _strides(k)
    rc = lib().oracle_col_scores(q.ctypes.data, k.ctypes.data, code, B, H, Hkv, L, d, bs,
                                 qs.ctypes.data, ks.ctypes.data, float(scale), S.ctypes.data)
    if rc:
        raise ValueError("oracle_col_scores rejected its arguments")
    return S


def col_select(S: np.ndarray, sparsity: float) -> np.ndarray:
    """int32 [B, H, Lc]: each head's Lc best columns (ties: lower index), ascending."""
    S = np.ascontiguousarray(S, dtype=np.float64)
    B, H, L = S.shape
    Lc = col_budget(L, sparsity)
    if Lc < 0:
        raise ValueError("sparsity outside [0, 1) or L not a multiple of 64")
    cols = np.empty((B, H, Lc), dtype=np.int32)
    if lib().oracle_col_select(S.ctypes.data, B, H, L, float(sparsity), cols.ctypes.data) != Lc:
        raise ValueError("oracle_col_select failed")
    return cols


def col_attention(q, k, v, cols, scale=None, rows=None, nthreads=None):
    """Attention of every query row of head h over the columns cols[b, h, :] only:
    O [B, H, L, d] and LSE [B, H, L] (or [n, d] / [n] for rows = int64 [n, 3] of (b, h, t))."""
    B, L, H, d = q.shape
    Hkv = k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    code = _dtype_code(q)
    assert _dtype_code(k) == code and _dtype_code(v) == code
    cols = np.ascontiguousarray(cols, dtype=np.int32)
    assert cols.shape[:2] == (B, H)
    Lc = cols.shape[2]
    if rows is not None:
        rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
        n = rows.shape[0]
    else:
        n = B * H * L
    O = np.empty((n, d), dtype=np.float64)
    lse = np.empty(n, dtype=np.float64)
    qs, ks, vs = _strides(q), _strides(k), _strides(v)
    rc = lib().oracle_col_attention(q.ctypes.data, k.ctypes.data, v.ctypes.data, code, B, H,
                                    Hkv, L, d, qs.ctypes.data, ks.ctypes.data, vs.ctypes.data,
                                    cols.ctypes.data, Lc, float(scale),
                                    None if rows is None else rows.ctypes.data, n,
                                    O.ctypes.data, lse.ctypes.data,
                                    nthreads or os.cpu_count() or 1)
    if rc:
        raise ValueError("oracle_col_attention rejected its arguments")
    if rows is None:
        return O.reshape(B, H, L, d), lse.reshape(B, H, L)
    return O, lse
