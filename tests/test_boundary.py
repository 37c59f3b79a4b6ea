"""The C-ABI library without a GPU: it loads, exports every function the
header declares, sizes workspaces on the host and rejects bad arguments
before touching CUDA."""
import ctypes
import os
import re

import pytest

import streaming_top_indexer_b200 as si
from streaming_top_indexer_b200 import build as sbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "si.h")


@pytest.fixture(scope="module")
def lib():
    sbuild.build()
    return si.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(si_[a-z_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for need in ("si_workspace_bytes", "si_indexer_topk", "si_check_device_status", "si_status_string"):
        assert need in names


def test_every_declared_symbol_is_exported(lib):
    raw = ctypes.CDLL(si.library_path())
    for name in declared_functions():
        assert hasattr(raw, name), f"{name} not exported"


def test_only_declared_symbols_are_exported():
    out = os.popen(f"nm -D --defined-only {si.library_path()}").read()
    exported = sorted(set(re.findall(r" T (si_\w+)", out)))
    assert exported == declared_functions()


def test_status_strings(lib):
    for code, name in si.SI_STATUS.items():
        assert lib.si_status_string(code).decode() == name


def test_workspace_bytes_host_arithmetic(lib):
    # pools fit in shared memory: header only
    assert si.workspace_bytes(1, 262144, 65536, 64, 128, 4, 512) == 256
    assert si.workspace_bytes(1, 2048, 512, 8, 64, 4, 64) == 256
    # k = 1024 at H_I=64 still fits (1856-entry pools, spare room k + 768)
    assert si.workspace_bytes(1, 65536, 16384, 64, 128, 4, 1024) == 256
    # k = 600 at H_I=32 does not: 148 CTAs x 8 queries x 2400-entry (4k) pools x 8 bytes
    assert si.workspace_bytes(1, 98304, 24576, 32, 128, 4, 600) == 256 + 148 * 8 * 2400 * 8
    # k = 2048 at H_I=64: 148 CTAs x 4 queries x 8192-entry (4k) pools x 8 bytes
    assert si.workspace_bytes(4, 131072, 32768, 64, 128, 4, 2048) == 256 + 148 * 4 * 8192 * 8
    # independent of S and T (never O(S*T))
    assert si.workspace_bytes(1, 1 << 20, 1 << 18, 64, 128, 4, 2048) == si.workspace_bytes(1, 64, 16, 64, 128, 4, 2048)
    for bad in [(1, 10, 4, 12, 128, 4, 8), (1, 10, 4, 64, 96, 4, 8), (1, 10, 4, 64, 128, 4, 0),
                (1, 10, 4, 64, 128, 4, 4096), (0, 10, 4, 64, 128, 4, 8), (1, 10, 4, 64, 128, 0, 8)]:
        assert lib.si_workspace_bytes(*bad) == 0


def call_topk(lib, q=16, w=16, kc=16, B=1, S=8, T=2, H=64, D=128, m=4, k=4, oi=16, os_=16, ws=16, wsb=1 << 20):
    return lib.si_indexer_topk(q, w, kc, B, S, T, H, D, m, k, oi, os_, ws, wsb, None)


def test_argument_errors_before_any_cuda_call(lib):
    assert call_topk(lib, q=0) == 1          # null q
    assert call_topk(lib, oi=0) == 1         # null output
    assert call_topk(lib, ws=0) == 1         # null workspace
    assert call_topk(lib, B=0) == 1
    assert call_topk(lib, m=0) == 1
    assert call_topk(lib, H=12) == 2         # unsupported H_I
    assert call_topk(lib, D=96) == 2         # unsupported d_I
    assert call_topk(lib, k=4096) == 2       # k too large
    assert call_topk(lib, S=1 << 26) == 2    # S*H_I >= 2^31
    assert call_topk(lib, q=24) == 3         # q not 16-byte aligned
    assert call_topk(lib, kc=8) == 3
    assert call_topk(lib, oi=18) == 3        # out_idx not 4-byte aligned
    assert call_topk(lib, wsb=16) == 4       # workspace too small
    assert lib.si_sort_topk(16, 16, 4, 0, None) == 2
    assert lib.si_sort_topk(0, 16, 4, 8, None) == 1
    assert lib.si_indexer_scores(16, 16, 16, 1, 8, 2, 64, 128, 4, 16, 16, 8, None) == 4
    assert lib.si_selftest_timeout(0, 256, 1000, None) == 1
    assert lib.si_reset_device_status(0, None) == 1
    assert lib.si_reset_device_status(24, None) == 3


def test_python_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros((1, 8, 64, 128), dtype=torch.bfloat16)
    w = torch.zeros((1, 8, 64))
    kc = torch.zeros((1, 2, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        si.indexer_topk(q, w, kc, 4, 4)


def call_rows(lib, t0, t1, S=1000, **kw):
    a = dict(q=16, w=16, kc=16, B=1, T=250, H=64, D=128, m=4, k=4, oi=16, os_=16, ws=16, wsb=1 << 20)
    a.update(kw)
    return lib.si_indexer_topk_rows(a["q"], a["w"], a["kc"], a["B"], S, a["T"], a["H"], a["D"], a["m"], a["k"],
                                    t0, t1, a["oi"], a["os_"], a["ws"], a["wsb"], None)


def test_row_window_arguments_before_any_cuda_call(lib):
    assert call_rows(lib, 100, 512) == 1     # window start not a multiple of 256
    assert call_rows(lib, 0, 300) == 1       # window end neither a multiple of 256 nor S
    assert call_rows(lib, 512, 256) == 1     # start after end
    assert call_rows(lib, -256, 256) == 1
    assert call_rows(lib, 0, 1024) == 1      # end past S
    assert call_rows(lib, 0, 256, q=0) == 1  # the whole-problem checks still apply
    assert call_rows(lib, 0, 256, H=12) == 2


def test_host_row_windows(lib):
    for S, chunks in [(262144, 8), (65536, 8), (2048, 8), (300, 8), (100, 4), (257, 1), (4096, 3)]:
        win = si.host_row_windows(S, chunks)
        assert win[0][0] == 0 and win[-1][1] == S
        for (a, b), (c, _) in zip(win, win[1:]):
            assert b == c
        for a, b in win:
            assert a < b and a % 256 == 0 and (b % 256 == 0 or b == S)
        assert len(win) <= max(1, chunks) + 1
        # rows per window: ceil(S / chunks) rounded down to a multiple of 256, at least 256
        assert lib.si_host_window_rows(S, chunks) == max(256, -(-S // chunks) // 256 * 256)
    assert lib.si_host_window_rows(0, 4) == 0 and si.host_row_windows(0, 4) == []
    assert lib.si_host_window_rows(1000, 0) == 768  # chunks < 1 counts as one window


def call_host(lib, **kw):
    a = dict(qh=16, wh=16, kch=16, B=1, S=1000, T=250, H=64, D=128, m=4, k=4, ih=16, sh=16, q=16, w=16, kc=16,
             oi=16, os_=16, ws=16, wsb=1 << 20, chunks=0)
    a.update(kw)
    return lib.si_indexer_topk_host(a["qh"], a["wh"], a["kch"], a["B"], a["S"], a["T"], a["H"], a["D"], a["m"],
                                    a["k"], a["ih"], a["sh"], a["q"], a["w"], a["kc"], a["oi"], a["os_"], a["ws"],
                                    a["wsb"], a["chunks"], None)


def test_host_entry_arguments_before_any_cuda_call(lib):
    """si_indexer_topk_host checks its host pointers, then every device-side
    rule of si_indexer_topk, before anything is enqueued."""
    for name in ("qh", "wh", "kch", "ih", "sh"):
        assert call_host(lib, **{name: 0}) == 1, name
    assert call_host(lib, kch=0, kc=0, T=0, chunks=-1) == 1    # negative window count
    assert call_host(lib, q=0) == 1 and call_host(lib, oi=0) == 1
    assert call_host(lib, H=12) == 2 and call_host(lib, k=2049) == 2
    assert call_host(lib, w=20) == 3                              # misaligned device buffer
    assert call_host(lib, wsb=8) == 4                             # workspace below si_workspace_bytes


def test_select_sorts_rows_host_arithmetic(lib):
    """The select kernel sorts rows in place for k <= 1024 (128*E >= k keys,
    E <= 8 a power of two); larger k keeps the separate row sort."""
    for H, D in [(64, 128), (64, 64), (32, 128), (32, 64), (16, 128), (16, 64), (8, 128), (8, 64)]:
        for k in (1, 64, 128, 129, 512, 600, 1024):
            assert si.select_sorts_rows(H, D, k), (H, D, k)
        for k in (1025, 1089, 2048):  # 16 keys per thread: the separate row sort is faster
            assert not si.select_sorts_rows(H, D, k), (H, D, k)
    assert not si.select_sorts_rows(64, 128, 0) and not si.select_sorts_rows(64, 128, 2049)
    assert not si.select_sorts_rows(48, 128, 64)


def test_tuning_knob_host_side(lib):
    """si_set_tuning: pool capacity, cut slack and check interval are
    validated, change the workspace only through the pool capacity, and
    reset to the defaults with zeros."""
    base = si.workspace_bytes(1, 65536, 16384, 64, 128, 4, 512)
    try:
        si.set_tuning(pool_entries=1344)
        assert si.workspace_bytes(1, 65536, 16384, 64, 128, 4, 512) == base  # fits shared memory
        si.set_tuning(pool_entries=4096)
        assert si.workspace_bytes(1, 65536, 16384, 64, 128, 4, 512) == 256 + 148 * 4 * 4096 * 8
        si.set_tuning(check_tiles=6, cut_slack=64)
        assert si.workspace_bytes(1, 65536, 16384, 64, 128, 4, 512) == base
        for bad in [dict(pool_entries=-1), dict(check_tiles=17), dict(cut_slack=5000)]:
            with pytest.raises(si.SIError):
                si.set_tuning(**bad)
    finally:
        si.set_tuning()
    assert si.workspace_bytes(1, 65536, 16384, 64, 128, 4, 512) == base
