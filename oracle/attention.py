"""Loader for the fp64 CPU oracle of CSA's sparse attention stage
(si_attn_oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module; the product path
never does.  The oracle shares no code with the CUDA library: it is built
from ``oracle/si_attn_oracle.c`` alone with gcc and loaded with ctypes.

The definition it follows is stated in si_attn_oracle.c (StreamIndex:
Memory-Bounded Compressed Sparse Attention via Streaming Top-k, Abstract:
the sparse attention reads only the keys the indexer selected).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "si_attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "libsi_attn_oracle.so")
_lock = threading.Lock()
_lib = None


def build(src: str = _SRC, out: str = _LIB_PATH, extra_flags=()) -> str:
    """Compile the attention oracle into a shared library with gcc + OpenMP."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", *extra_flags, src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return out


def _declare(lib):
    c = ctypes
    u16p, i32p, i64p, f64p = (c.POINTER(c.c_uint16), c.POINTER(c.c_int32), c.POINTER(c.c_int64),
                              c.POINTER(c.c_double))
    lib.oracle_sparse_attention.restype = c.c_int
    lib.oracle_sparse_attention.argtypes = [u16p, i32p, i64p, c.c_int64, u16p, u16p, c.c_int64, c.c_int64,
                                            c.c_int, c.c_int, c.c_int, c.c_int64, c.c_double, f64p, f64p, f64p]
    return lib


def load_library(path: str | None = None):
    """Load (building first if needed) an attention-oracle shared library."""
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
                build()
            _lib = _declare(ctypes.CDLL(_LIB_PATH))
    return _lib


def _ptr(a, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def sparse_attention_rows(q_rows_bits, idx_rows, row_b, k_bits, v_bits, scale, want_absw=False, lib=None):
    """Sparse attention of the given query rows.

    q_rows_bits uint16 [R,H,D] (bf16 bits), idx_rows int32 [R,k] (< 0 =
    padding), row_b int64 [R], k_bits uint16 [B,T,D], v_bits uint16 [B,T,DV].
    Returns (out float64 [R,H,DV], lse float64 [R,H], absw [R,H,DV] or None).
    """
    lib = lib or load_library()
    q = np.ascontiguousarray(q_rows_bits, dtype=np.uint16)
    idx = np.ascontiguousarray(idx_rows, dtype=np.int32)
    rb = np.ascontiguousarray(row_b, dtype=np.int64)
    kk = np.ascontiguousarray(k_bits, dtype=np.uint16)
    vv = np.ascontiguousarray(v_bits, dtype=np.uint16)
    R, H, D = q.shape
    B, T, D2 = kk.shape
    B2, T2, DV = vv.shape
    if D2 != D or (B2, T2) != (B, T) or idx.shape[0] != R or rb.shape != (R,):
        raise ValueError("attention oracle: inconsistent shapes")
    k = idx.shape[1]
    out = np.empty((R, H, DV), np.float64)
    lse = np.empty((R, H), np.float64)
    absw = np.empty((R, H, DV), np.float64) if want_absw else None
    rc = lib.oracle_sparse_attention(_ptr(q, ctypes.c_uint16), _ptr(idx, ctypes.c_int32), _ptr(rb, ctypes.c_int64),
                                     R, _ptr(kk, ctypes.c_uint16), _ptr(vv, ctypes.c_uint16), B, T, H, D, DV, k,
                                     float(scale), _ptr(out, ctypes.c_double), _ptr(lse, ctypes.c_double),
                                     _ptr(absw, ctypes.c_double) if absw is not None else None)
    if rc != 0:
        raise RuntimeError("oracle_sparse_attention failed")
    return out, lse, absw
