"""The select kernel's abort path on the GPU, without a fault or a hang.

Every device wait of the select kernel is bounded: when a wait runs out, the
kernel records SI_ERR_TIMEOUT in the workspace's error word, raises the CTA's
abort flag, lets the TMA loads and MMAs it issued complete (with bounded
waits), releases TMEM and returns.  The library built with SI_FAULT_TEST
(lib/libsi_ftest.so, a test-only variant) withholds one accumulator-ready
signal in CTA 0, so the epilogue's wait on it expires after the limit set by
si_set_timeout_ns.  The call must report SI_ERR_TIMEOUT (also through the
no-allocation entry point's out_status), return within bounded time, and
leave the CUDA context usable: the product library then gives the same rows
as before.
"""
import ctypes
import time

import pytest
import torch

import streaming_top_indexer_b200 as si
from streaming_top_indexer_b200 import build as sbuild
from streaming_top_indexer_b200 import synth

pytestmark = pytest.mark.gpu

SI_ERR_TIMEOUT = 6


@pytest.fixture(scope="module")
def ftest():
    lib = ctypes.CDLL(sbuild.build_fault_test())
    vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    lib.si_indexer_topk.restype = i32
    lib.si_indexer_topk.argtypes = [vp, vp, vp, i64, i64, i64, i32, i32, i32, i32, vp, vp, vp, sz, vp]
    lib.si_indexer_topk_noalloc.restype = i32
    lib.si_indexer_topk_noalloc.argtypes = [vp, vp, vp, i64, i64, i64, i32, i32, i32, i32, vp, vp, vp, vp]
    lib.si_check_device_status.restype = i32
    lib.si_check_device_status.argtypes = [vp, vp]
    lib.si_set_timeout_ns.restype = None
    lib.si_set_timeout_ns.argtypes = [ctypes.c_uint64]
    lib.si_workspace_bytes.restype = sz
    lib.si_workspace_bytes.argtypes = [i64, i64, i64, i32, i32, i32, i32]
    lib.si_set_timeout_ns(50_000_000)  # 50 ms
    return lib


# The longest unit (CTA 0's first) has 16 key tiles, so the withheld signal
# (the third tile's) falls in the middle of a unit.
SHAPES = [
    # B, S, T, H, D, m, k
    (1, 8192, 2048, 64, 128, 4, 64),     # shared-memory pools
    (1, 8192, 2048, 64, 128, 4, 2048),   # workspace pools
    (2, 4096, 1024, 16, 128, 4, 100),    # H_I=16, workspace pools
]


def _inputs(B, S, T, H, D, m, k):
    wl = synth.Workload("abort", B, S, m, H, D, k)
    return synth.generate(wl, seed=S + k, device="cuda", T=T)


@pytest.mark.parametrize("B,S,T,H,D,m,k", SHAPES)
def test_expired_wait_reports_timeout_and_context_survives(ftest, B, S, T, H, D, m, k):
    q, w, kc = _inputs(B, S, T, H, D, m, k)
    ref_idx, ref_sc = si.indexer_topk(q, w, kc, m, k)
    torch.cuda.synchronize()
    ws = torch.zeros(int(ftest.si_workspace_bytes(B, S, T, H, D, m, k)), dtype=torch.uint8, device="cuda")
    idx = torch.empty((B, S, k), dtype=torch.int32, device="cuda")
    sc = torch.empty((B, S, k), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    t0 = time.monotonic()
    rc = ftest.si_indexer_topk(q.data_ptr(), w.data_ptr(), kc.data_ptr(), B, S, T, H, D, m, k, idx.data_ptr(),
                               sc.data_ptr(), ws.data_ptr(), ws.numel(), stream)
    assert rc == 0
    assert ftest.si_check_device_status(ws.data_ptr(), stream) == SI_ERR_TIMEOUT
    assert time.monotonic() - t0 < 10.0
    # the context is still usable: the product library's rows are unchanged
    idx2, sc2 = si.indexer_topk(q, w, kc, m, k)
    torch.cuda.synchronize()
    assert torch.equal(idx2, ref_idx) and torch.equal(sc2, ref_sc)


def test_noalloc_out_status_receives_timeout(ftest):
    B, S, T, H, D, m, k = SHAPES[0]
    q, w, kc = _inputs(B, S, T, H, D, m, k)
    idx = torch.empty((B, S, k), dtype=torch.int32, device="cuda")
    sc = torch.empty((B, S, k), dtype=torch.float32, device="cuda")
    status = torch.full((1,), 99, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    rc = ftest.si_indexer_topk_noalloc(q.data_ptr(), w.data_ptr(), kc.data_ptr(), B, S, T, H, D, m, k,
                                       idx.data_ptr(), sc.data_ptr(), status.data_ptr(), stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert int(status.item()) == SI_ERR_TIMEOUT
    # the context is still usable
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    si.indexer_topk(q, w, kc, m, k, workspace=ws)
    assert si.check_device_status(ws) == 0
