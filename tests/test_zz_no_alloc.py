"""The workspace-free entry point, si_indexer_topk_noalloc, called through
the C ABI.  It serves callers that cannot allocate device memory themselves
(a plugin whose host application owns all device memory, a serving loop with
a frozen memory plan); it uses the library's built-in 1 MiB scratch array.
Its results must equal those of si_indexer_topk, call after call.  This file
is named to be collected last."""
import ctypes

import pytest
import torch

import streaming_top_indexer_b200 as si
from streaming_top_indexer_b200 import synth

pytestmark = pytest.mark.gpu

SI_ERR_WORKSPACE_TOO_SMALL = 4


def noalloc_fn():
    lib = si.load_library()
    fn = lib.si_indexer_topk_noalloc
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    fn.restype = ctypes.c_int
    fn.argtypes = [vp, vp, vp, i64, i64, i64, i32, i32, i32, i32, vp, vp, vp, vp]
    return fn


def call_noalloc(fn, q, w, kc, m, k, stream):
    B, S, H, D = q.shape
    T = kc.shape[1]
    idx = torch.full((B, S, k), 7, dtype=torch.int32, device=q.device)
    sc = torch.full((B, S, k), 7.0, dtype=torch.float32, device=q.device)
    status = torch.full((1,), 99, dtype=torch.int32, device=q.device)
    rc = fn(q.data_ptr(), w.data_ptr(), kc.data_ptr(), B, S, T, H, D, m, k, idx.data_ptr(), sc.data_ptr(),
            status.data_ptr(), stream)
    return rc, idx, sc, status


@pytest.mark.parametrize("B,S,T,H,D,m,k", [
    (1, 2048, 512, 8, 64, 4, 64),      # tiny workload shape
    (2, 3000, 750, 64, 128, 4, 512),   # V4-shaped heads, several tiles, ragged
])
def test_noalloc_equals_indexer_topk_on_two_calls(B, S, T, H, D, m, k):
    wl = synth.Workload("noalloc", B, S, m, H, D, k)
    q, w, kc = synth.generate(wl, seed=S + k, device="cuda", T=T)
    ref_idx, ref_sc = si.indexer_topk(q, w, kc, m, k)
    stream = torch.cuda.current_stream().cuda_stream
    fn = noalloc_fn()
    for _ in range(2):
        rc, idx, sc, status = call_noalloc(fn, q, w, kc, m, k, stream)
        assert rc == 0
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        # same kernels, same inputs: identical indices and bit-identical scores
        assert torch.equal(idx, ref_idx)
        assert torch.equal(sc, ref_sc)


@pytest.mark.parametrize("H,D,k", [
    (64, 128, 2048),  # ~39 MB of candidate pools, more than 1 MiB
    (64, 128, 1089),  # the first refused k at H_I=64, d_I=128
    (8, 128, 64),     # H_I=8, d_I=128: 32 queries per unit, pools never fit in shared memory
    (16, 64, 481),    # the first refused k at H_I=16, d_I=64
])
def test_noalloc_rejects_configurations_beyond_its_scratch(H, D, k):
    wl = synth.Workload("noalloc_big", 1, 256, 4, H, D, k)
    q, w, kc = synth.generate(wl, seed=1, device="cuda")
    rc, idx, _, status = call_noalloc(noalloc_fn(), q, w, kc, 4, k, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert rc == SI_ERR_WORKSPACE_TOO_SMALL
    assert int(status.item()) == 99 and int(idx[0, 0, 0].item()) == 7  # nothing was enqueued


def test_noalloc_first_accepted_below_the_limit():
    """k = 1088 at H_I=64, d_I=128 (one below the first refused k) runs and
    equals si_indexer_topk."""
    wl = synth.Workload("noalloc_edge", 1, 9000, 4, 64, 128, 1088)
    q, w, kc = synth.generate(wl, seed=5, device="cuda")
    ref_idx, ref_sc = si.indexer_topk(q, w, kc, wl.m, wl.k)
    rc, idx, sc, status = call_noalloc(noalloc_fn(), q, w, kc, wl.m, wl.k, torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(idx, ref_idx) and torch.equal(sc, ref_sc)


def test_noalloc_leaves_device_memory_unchanged():
    """After the first call on the device (which resolves the array's address),
    calls take no device memory: cudaMemGetInfo's free bytes do not move."""
    wl = synth.Workload("noalloc_mem", 1, 4096, 4, 64, 128, 512)
    q, w, kc = synth.generate(wl, seed=6, device="cuda")
    fn = noalloc_fn()
    stream = torch.cuda.current_stream().cuda_stream
    outs = [call_noalloc(fn, q, w, kc, wl.m, wl.k, stream)]  # first call; outputs come from torch
    torch.cuda.synchronize()
    idx = torch.empty((1, wl.S, wl.k), dtype=torch.int32, device="cuda")
    sc = torch.empty((1, wl.S, wl.k), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        rc = fn(q.data_ptr(), w.data_ptr(), kc.data_ptr(), 1, wl.S, wl.T, wl.H, wl.D, wl.m, wl.k, idx.data_ptr(),
                sc.data_ptr(), status.data_ptr(), stream)
        assert rc == 0
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert int(status.item()) == 0
    assert torch.equal(idx, outs[0][1]) and torch.equal(sc, outs[0][2])
