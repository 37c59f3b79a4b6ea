"""Streaming top-k indexer (CSA indexer step) for NVIDIA B200, sm_100a.

Thin Python binding of the C ABI in ``include/si.h`` (``lib/libsi.so``):
argument marshalling only.  Every step of the computation runs in the
library's CUDA kernels; there is no CPU fallback, and every call raises if
the library is missing or a tensor is not a CUDA tensor of the right dtype.

The operation (StreamIndex: Memory-Bounded Compressed Sparse Attention via
Streaming Top-k, Abstract): for each query row t, score every compressed
key s it can see, ``score = sum_h w[t,h] * ReLU(q[t,h,:] . kc[s,:])`` with s
visible iff (s+1)*m <= t+1, and return the top-k keys (score descending,
equal scores to the lower index, padding index -1 / score -inf) without
materialising the [B,S,H_I,T] score tensor.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "SIError", "library_path", "load_library", "workspace_bytes", "indexer_topk",
    "select_topk", "sort_topk", "indexer_scores", "check_device_status",
    "selftest_timeout", "set_timeout_ns", "indexer_topk_host", "version", "select_sorts_rows",
    "set_sort_in_select", "sparse_attention", "set_tuning", "indexer_inputs",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "lib", "libsi.so")
_lib = None

SI_STATUS = {0: "SI_OK", 1: "SI_ERR_INVALID_ARG", 2: "SI_ERR_UNSUPPORTED", 3: "SI_ERR_MISALIGNED",
             4: "SI_ERR_WORKSPACE_TOO_SMALL", 5: "SI_ERR_CUDA", 6: "SI_ERR_TIMEOUT"}


class SIError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {SI_STATUS.get(status, status)}")


def library_path() -> str:
    return _LIB_PATH


def _declare(lib):
    c = ctypes
    vp, i64, i32, sz = c.c_void_p, c.c_int64, c.c_int, c.c_size_t
    lib.si_workspace_bytes.restype = sz
    lib.si_workspace_bytes.argtypes = [i64, i64, i64, i32, i32, i32, i32]
    topk_args = [vp, vp, vp, i64, i64, i64, i32, i32, i32, i32, vp, vp, vp, sz, vp]
    for name in ("si_indexer_topk", "si_select_topk"):
        fn = getattr(lib, name)
        fn.restype = c.c_int
        fn.argtypes = topk_args
    lib.si_indexer_topk_rows.restype = c.c_int
    lib.si_indexer_topk_rows.argtypes = topk_args[:10] + [i64, i64] + topk_args[10:]
    lib.si_indexer_topk_host.restype = c.c_int
    lib.si_indexer_topk_host.argtypes = topk_args[:12] + [vp, vp, vp, vp, vp, vp, sz, i32, vp]
    lib.si_host_window_rows.restype = i64
    lib.si_host_window_rows.argtypes = [i64, i32]
    lib.si_sort_topk.restype = c.c_int
    lib.si_sort_topk.argtypes = [vp, vp, i64, i32, vp]
    lib.si_indexer_scores.restype = c.c_int
    lib.si_indexer_scores.argtypes = [vp, vp, vp, i64, i64, i64, i32, i32, i32, vp, vp, sz, vp]
    lib.si_reset_device_status.restype = c.c_int
    lib.si_reset_device_status.argtypes = [vp, vp]
    lib.si_check_device_status.restype = c.c_int
    lib.si_check_device_status.argtypes = [vp, vp]
    lib.si_selftest_timeout.restype = c.c_int
    lib.si_selftest_timeout.argtypes = [vp, sz, c.c_uint64, vp]
    lib.si_set_timeout_ns.restype = None
    lib.si_set_timeout_ns.argtypes = [c.c_uint64]
    lib.si_sparse_attention.restype = c.c_int
    lib.si_sparse_attention.argtypes = [vp, vp, vp, vp, i64, i64, i64, i32, i32, i32, i32, c.c_float, vp, vp, vp,
                                        vp]
    lib.si_indexer_inputs.restype = c.c_int
    lib.si_indexer_inputs.argtypes = [vp, vp, vp, vp, i64, i64, i32, i32, i32, i32, vp, vp, vp, vp, vp]
    lib.si_select_sorts_rows.restype = c.c_int
    lib.si_select_sorts_rows.argtypes = [i32, i32, i32]
    lib.si_set_sort_in_select.restype = None
    lib.si_set_sort_in_select.argtypes = [i32]
    lib.si_set_tuning.restype = c.c_int
    lib.si_set_tuning.argtypes = [i32, i32, i32]
    lib.si_status_string.restype = c.c_char_p
    lib.si_status_string.argtypes = [c.c_int]
    lib.si_version.restype = c.c_char_p
    lib.si_version.argtypes = []
    return lib


def load_library():
    """Load lib/libsi.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"{_LIB_PATH} is missing: build it with `python -m streaming_top_indexer_b200.build`")
        _lib = _declare(ctypes.CDLL(_LIB_PATH))
    return _lib


def version() -> str:
    return load_library().si_version().decode()


def set_timeout_ns(ns: int) -> None:
    load_library().si_set_timeout_ns(int(ns))


def select_sorts_rows(H: int, D: int, k: int) -> bool:
    """Whether the select kernel writes rows already sorted for these sizes
    (si_select_sorts_rows); otherwise indexer_topk adds the row-sort kernel."""
    return bool(load_library().si_select_sorts_rows(int(H), int(D), int(k)))


def set_tuning(pool_entries: int = 0, cut_slack: int = 0, check_tiles: int = 0) -> None:
    """Design parameters of the select kernel (si_set_tuning); 0 = default.
    Results are the exact top-k for every setting; size workspaces after."""
    _check(load_library().si_set_tuning(int(pool_entries), int(cut_slack), int(check_tiles)), "si_set_tuning")


def set_sort_in_select(enable: bool) -> None:
    """Process-wide: sort rows inside the select kernel (default) or always
    in the separate row-sort kernel (si_set_sort_in_select)."""
    load_library().si_set_sort_in_select(1 if enable else 0)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _need(t: torch.Tensor, name: str, dtype, ndim: int):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {ndim}-d tensor")


def _check(rc: int, what: str):
    if rc != 0:
        raise SIError(rc, what)


def _dims(q, w, kc):
    _need(q, "q", torch.bfloat16, 4)
    _need(w, "w", torch.float32, 3)
    _need(kc, "kc", torch.bfloat16, 3)
    B, S, H, D = q.shape
    if tuple(w.shape) != (B, S, H) or kc.shape[0] != B or kc.shape[2] != D:
        raise ValueError(f"shape mismatch: q {tuple(q.shape)} w {tuple(w.shape)} kc {tuple(kc.shape)}")
    return B, S, kc.shape[1], H, D


def workspace_bytes(B: int, S: int, T: int, H: int, D: int, m: int, k: int) -> int:
    n = load_library().si_workspace_bytes(B, S, T, H, D, m, k)
    if n == 0:
        raise SIError(2, "si_workspace_bytes")
    return int(n)


def _outputs(B, S, k, device, out_idx, out_score):
    if out_idx is None:
        out_idx = torch.empty((B, S, k), dtype=torch.int32, device=device)
    if out_score is None:
        out_score = torch.empty((B, S, k), dtype=torch.float32, device=device)
    _need(out_idx, "out_idx", torch.int32, 3)
    _need(out_score, "out_score", torch.float32, 3)
    if tuple(out_idx.shape) != (B, S, k) or tuple(out_score.shape) != (B, S, k):
        raise ValueError("outputs must be [B,S,k]")
    return out_idx, out_score


def _workspace(B, S, T, H, D, m, k, device, workspace):
    need = workspace_bytes(B, S, T, H, D, m, k)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    if not workspace.is_cuda or workspace.dtype != torch.uint8:
        raise ValueError("workspace must be a CUDA uint8 tensor")
    return workspace


def _topk_call(fn_name, q, w, kc, m, k, out_idx, out_score, workspace, stream):
    B, S, T, H, D = _dims(q, w, kc)
    out_idx, out_score = _outputs(B, S, k, q.device, out_idx, out_score)
    workspace = _workspace(B, S, T, H, D, m, k, q.device, workspace)
    fn = getattr(load_library(), fn_name)
    _check(fn(q.data_ptr(), w.data_ptr(), kc.data_ptr() if T > 0 else None, B, S, T, H, D, m, k,
              out_idx.data_ptr(), out_score.data_ptr(), workspace.data_ptr(), workspace.numel(),
              _stream(stream)), fn_name)
    return out_idx, out_score


def indexer_topk(q, w, kc, m: int, k: int, out_idx=None, out_score=None, workspace=None, stream=None):
    """Top-k keys and scores of every query row (si_indexer_topk).

    q bf16 [B,S,H_I,d_I], w fp32 [B,S,H_I], kc bf16 [B,T,d_I] on the GPU.
    Returns (idx int32 [B,S,k], score fp32 [B,S,k]), asynchronously on
    ``stream`` (default: torch's current stream).
    """
    return _topk_call("si_indexer_topk", q, w, kc, m, k, out_idx, out_score, workspace, stream)


def indexer_topk_rows(q, w, kc, m: int, k: int, t_begin: int, t_end: int, out_idx, out_score, workspace,
                      stream=None):
    """Query rows [t_begin, t_end) of every batch (si_indexer_topk_rows): the
    whole q, w and output tensors are passed, only the window's rows are read
    and written.  t_begin is a multiple of 256, t_end a multiple of 256 or S.
    The workspace's error word is not reset (see reset_device_status)."""
    B, S, T, H, D = _dims(q, w, kc)
    _need(out_idx, "out_idx", torch.int32, 3)
    _need(out_score, "out_score", torch.float32, 3)
    _check(load_library().si_indexer_topk_rows(q.data_ptr(), w.data_ptr(), kc.data_ptr() if T > 0 else None, B, S,
                                               T, H, D, m, k, int(t_begin), int(t_end), out_idx.data_ptr(),
                                               out_score.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                               _stream(stream)), "si_indexer_topk_rows")
    return out_idx, out_score


def select_topk(q, w, kc, m: int, k: int, out_idx=None, out_score=None, workspace=None, stream=None):
    """First stage only (si_select_topk): each row's top-k set, already in
    final order where select_sorts_rows(H, D, k), else unordered."""
    return _topk_call("si_select_topk", q, w, kc, m, k, out_idx, out_score, workspace, stream)


def sort_topk(out_idx, out_score, stream=None):
    """Second stage only (si_sort_topk): order rows in place."""
    _need(out_idx, "out_idx", torch.int32, 3)
    _need(out_score, "out_score", torch.float32, 3)
    B, S, k = out_idx.shape
    _check(load_library().si_sort_topk(out_idx.data_ptr(), out_score.data_ptr(), B * S, k, _stream(stream)),
           "si_sort_topk")
    return out_idx, out_score


def indexer_scores(q, w, kc, m: int, out=None, workspace=None, stream=None):
    """Materialise path for small problems (si_indexer_scores): dense fp32
    [B,S,T] scores; entries of keys a row cannot see are left as given in
    ``out`` (default: NaN)."""
    B, S, T, H, D = _dims(q, w, kc)
    if out is None:
        out = torch.full((B, S, T), float("nan"), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, 3)
    if workspace is None:
        workspace = torch.empty(256, dtype=torch.uint8, device=q.device)
    _check(load_library().si_indexer_scores(q.data_ptr(), w.data_ptr(), kc.data_ptr() if T > 0 else None,
                                            B, S, T, H, D, m, out.data_ptr(), workspace.data_ptr(),
                                            workspace.numel(), _stream(stream)), "si_indexer_scores")
    return out


def reset_device_status(workspace, stream=None):
    """Clear the device error word (si_reset_device_status), asynchronously."""
    _check(load_library().si_reset_device_status(workspace.data_ptr(), _stream(stream)), "si_reset_device_status")


def check_device_status(workspace, stream=None) -> int:
    """Synchronise and return the device status word of the last call (0 = OK)."""
    return int(load_library().si_check_device_status(workspace.data_ptr(), _stream(stream)))


def selftest_timeout(workspace, limit_ns: int, stream=None) -> int:
    """Run the bounded-wait self-test; returns the device status it left."""
    _check(load_library().si_selftest_timeout(workspace.data_ptr(), workspace.numel(), int(limit_ns),
                                              _stream(stream)), "si_selftest_timeout")
    return check_device_status(workspace, stream)


def host_row_windows(S: int, chunks: int):
    """Row windows of si_indexer_topk_host, in row order: si_host_window_rows
    rows each (a multiple of 256), the last window ending at S."""
    step = int(load_library().si_host_window_rows(int(S), int(chunks)))
    if step <= 0:
        return []
    bounds = list(range(0, S, step)) + [S]
    return [(bounds[i], bounds[i + 1]) for i in range(len(bounds) - 1)]


def indexer_topk_host(q, w, kc, m: int, k: int, device="cuda", buffers=None, stream=None, chunks=None):
    """End-to-end call on host tensors (si_indexer_topk_host): copies q, w, kc
    to the GPU, runs the indexer and copies (idx, score) back into host
    tensors, overlapped by row windows inside the library.

    Host tensors should be pinned for the copies to overlap.  ``chunks`` sets
    the number of row windows (default: the library's, S/2048 capped at 32).
    ``buffers`` may hold preallocated device tensors ("q","w","kc","idx",
    "score","ws") and pinned host outputs ("idx_h","score_h") to reuse; they
    are created on first use.  Returns (idx_h, score_h), complete once
    ``stream`` (default: torch's current stream) is synchronised.
    """
    for t, n, dt, nd in ((q, "q", torch.bfloat16, 4), (w, "w", torch.float32, 3), (kc, "kc", torch.bfloat16, 3)):
        if not isinstance(t, torch.Tensor) or t.is_cuda or t.dtype != dt or t.dim() != nd or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous {nd}-d {dt} host tensor")
    b = {} if buffers is None else buffers
    dev = torch.device(device)
    B, S, H, D = q.shape
    T = kc.shape[1]
    if tuple(w.shape) != (B, S, H) or kc.shape[0] != B or kc.shape[2] != D:
        raise ValueError(f"shape mismatch: q {tuple(q.shape)} w {tuple(w.shape)} kc {tuple(kc.shape)}")
    if "q" not in b:
        b["q"] = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
        b["w"] = torch.empty(w.shape, dtype=torch.float32, device=dev)
        b["kc"] = torch.empty(kc.shape, dtype=torch.bfloat16, device=dev)
        b["idx"] = torch.empty((B, S, k), dtype=torch.int32, device=dev)
        b["score"] = torch.empty((B, S, k), dtype=torch.float32, device=dev)
        b["ws"] = torch.empty(workspace_bytes(B, S, T, H, D, m, k), dtype=torch.uint8, device=dev)
        b["idx_h"] = torch.empty((B, S, k), dtype=torch.int32, pin_memory=True)
        b["score_h"] = torch.empty((B, S, k), dtype=torch.float32, pin_memory=True)
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    with torch.cuda.device(dev):
        _check(load_library().si_indexer_topk_host(
            q.data_ptr(), w.data_ptr(), kc.data_ptr() if T > 0 else None, B, S, T, H, D, m, k,
            b["idx_h"].data_ptr(), b["score_h"].data_ptr(), b["q"].data_ptr(), b["w"].data_ptr(),
            b["kc"].data_ptr() if T > 0 else None, b["idx"].data_ptr(), b["score"].data_ptr(), b["ws"].data_ptr(),
            b["ws"].numel(), 0 if chunks is None else int(chunks), _stream(s)), "si_indexer_topk_host")
    return b["idx_h"], b["score_h"]


def sparse_attention(q, kcache, vcache, idx, scale: float, out=None, lse=None, status=None, stream=None):
    """CSA sparse attention over the selected keys (si_sparse_attention).

    q bf16 [B,S,128,d], kcache bf16 [B,T,d], vcache bf16 [B,T,d_v], idx int32
    [B,S,k] (entries outside [0,T) are skipped).  Returns (out bf16
    [B,S,128,d_v], lse fp32 [B,S,128], status int32 [1] device word: 0, or 6
    if a device wait expired), asynchronously on ``stream``.
    """
    _need(q, "q", torch.bfloat16, 4)
    _need(kcache, "kcache", torch.bfloat16, 3)
    _need(vcache, "vcache", torch.bfloat16, 3)
    _need(idx, "idx", torch.int32, 3)
    B, S, H, D = q.shape
    T, DV = kcache.shape[1], vcache.shape[2]
    k = idx.shape[2]
    if kcache.shape[0] != B or vcache.shape[:2] != (B, T) or kcache.shape[2] != D or tuple(idx.shape[:2]) != (B, S):
        raise ValueError("shape mismatch")
    if out is None:
        out = torch.empty((B, S, H, DV), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, S, H), dtype=torch.float32, device=q.device)
    if status is None:
        status = torch.empty(1, dtype=torch.int32, device=q.device)
    _need(out, "out", torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 3)
    _check(load_library().si_sparse_attention(q.data_ptr(), kcache.data_ptr() if T > 0 else None,
                                              vcache.data_ptr() if T > 0 else None, idx.data_ptr(), B, S, T, H, D,
                                              DV, k, float(scale), out.data_ptr(), lse.data_ptr(),
                                              status.data_ptr(), _stream(stream)), "si_sparse_attention")
    return out, lse, status


def indexer_inputs(x, w_q, w_w, w_k, H: int, D: int, m: int, q=None, w=None, kc=None, status=None, stream=None):
    """q, w and kc of the indexer from hidden states (si_indexer_inputs).

    x bf16 [B,S,d_model]; weights bf16 in [out, in] layout: w_q [H*D,
    d_model], w_w [H, d_model], w_k [D, d_model].  Returns (q bf16 [B,S,H,D],
    w fp32 [B,S,H], kc bf16 [B,S//m,D], status int32 [1] device word),
    asynchronously on ``stream``.
    """
    _need(x, "x", torch.bfloat16, 3)
    for name, t, rows in (("w_q", w_q, H * D), ("w_w", w_w, H), ("w_k", w_k, D)):
        _need(t, name, torch.bfloat16, 2)
        if tuple(t.shape) != (rows, x.shape[2]):
            raise ValueError(f"{name} must be [{rows}, d_model]")
    B, S, DM = x.shape
    T = S // m
    if q is None:
        q = torch.empty((B, S, H, D), dtype=torch.bfloat16, device=x.device)
    if w is None:
        w = torch.empty((B, S, H), dtype=torch.float32, device=x.device)
    if kc is None:
        kc = torch.empty((B, T, D), dtype=torch.bfloat16, device=x.device)
    if status is None:
        status = torch.empty(1, dtype=torch.int32, device=x.device)
    _check(load_library().si_indexer_inputs(x.data_ptr(), w_q.data_ptr(), w_w.data_ptr(), w_k.data_ptr(), B, S, DM,
                                            H, D, m, q.data_ptr(), w.data_ptr(), kc.data_ptr(), status.data_ptr(),
                                            _stream(stream)), "si_indexer_inputs")
    return q, w, kc, status
