"""Loader for the fp64 CPU oracle of the CSA indexer step (si_oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module; the product path
(the ``streaming_top_indexer_b200`` package) never does.  The oracle shares
no code with the CUDA library: it is built from ``oracle/si_oracle.c`` alone
with gcc and loaded with ctypes.

The definition it follows is stated in si_oracle.c (StreamIndex:
Memory-Bounded Compressed Sparse Attention via Streaming Top-k, Abstract).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "si_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libsi_oracle.so")
_lock = threading.Lock()
_lib = None


def build(src: str = _SRC, out: str = _LIB_PATH, extra_flags=()) -> str:
    """Compile the oracle into a shared library with gcc + OpenMP."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
           *extra_flags, src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return out


def _declare(lib):
    u16p = ctypes.POINTER(ctypes.c_uint16)
    f32p = ctypes.POINTER(ctypes.c_float)
    i64p = ctypes.POINTER(ctypes.c_int64)
    i32p = ctypes.POINTER(ctypes.c_int32)
    f64p = ctypes.POINTER(ctypes.c_double)
    lib.oracle_topk_rows.restype = ctypes.c_int
    lib.oracle_topk_rows.argtypes = [
        u16p, f32p, i64p, i64p, ctypes.c_int64,
        u16p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
        ctypes.c_int64, ctypes.c_int64, i32p, f64p, f64p, f64p]
    lib.oracle_max_threads.restype = ctypes.c_int
    lib.oracle_max_threads.argtypes = []
    lib.oracle_set_threads.restype = None
    lib.oracle_set_threads.argtypes = [ctypes.c_int]
    return lib


def load_library(path: str | None = None):
    """Load (building first if needed) an oracle shared library."""
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            if (not os.path.exists(_LIB_PATH)
                    or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
                build()
            _lib = _declare(ctypes.CDLL(_LIB_PATH))
    return _lib


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def max_threads() -> int:
    return int(load_library().oracle_max_threads())


def set_threads(n: int) -> None:
    load_library().oracle_set_threads(int(n))


def topk_rows(q_rows_bits, w_rows, row_b, row_t, kc_bits, m, k,
              want_scores=False, lib=None):
    """Exact top-k of the given query rows.

    q_rows_bits: uint16 [R, H, D] bf16 bit patterns of the rows' q vectors.
    w_rows:      float32 [R, H].
    row_b, row_t: int64 [R] batch and query position of each row.
    kc_bits:     uint16 [B, T, D] bf16 bit patterns of the compressed keys.

    Returns (idx int32 [R,k], score float64 [R,k], meta float64 [R,4],
    scores float64 [R,T] or None).  meta columns: max |score| over visible
    keys, score at rank k, score at rank k+1 (NaN if absent), visible count.
    """
    lib = lib or load_library()
    q = np.ascontiguousarray(q_rows_bits, dtype=np.uint16)
    w = np.ascontiguousarray(w_rows, dtype=np.float32)
    rb = np.ascontiguousarray(row_b, dtype=np.int64)
    rt = np.ascontiguousarray(row_t, dtype=np.int64)
    kc = np.ascontiguousarray(kc_bits, dtype=np.uint16)
    R, H, D = q.shape
    B, T, D2 = kc.shape
    if D2 != D or w.shape != (R, H) or rb.shape != (R,) or rt.shape != (R,):
        raise ValueError("oracle: inconsistent shapes")
    out_idx = np.empty((R, k), np.int32)
    out_score = np.empty((R, k), np.float64)
    meta = np.empty((R, 4), np.float64)
    scores = np.empty((R, T), np.float64) if want_scores else None
    rc = lib.oracle_topk_rows(
        _ptr(q, ctypes.c_uint16), _ptr(w, ctypes.c_float),
        _ptr(rb, ctypes.c_int64), _ptr(rt, ctypes.c_int64), R,
        _ptr(kc, ctypes.c_uint16), B, T, H, D, int(m), int(k),
        _ptr(out_idx, ctypes.c_int32), _ptr(out_score, ctypes.c_double),
        _ptr(meta, ctypes.c_double),
        _ptr(scores, ctypes.c_double) if scores is not None else None)
    if rc != 0:
        raise RuntimeError("oracle_topk_rows failed")
    return out_idx, out_score, meta, scores


def topk_all_rows(q_bits, w, kc_bits, m, k, want_scores=False, lib=None):
    """Top-k of every row of a full problem (q_bits uint16 [B,S,H,D])."""
    B, S, H, D = q_bits.shape
    rb = np.repeat(np.arange(B, dtype=np.int64), S)
    rt = np.tile(np.arange(S, dtype=np.int64), B)
    idx, sc, meta, scores = topk_rows(q_bits.reshape(B * S, H, D),
                                      np.asarray(w).reshape(B * S, H), rb, rt,
                                      kc_bits, m, k, want_scores, lib)
    T = kc_bits.shape[1]
    return (idx.reshape(B, S, k), sc.reshape(B, S, k), meta.reshape(B, S, 4),
            None if scores is None else scores.reshape(B, S, T))
