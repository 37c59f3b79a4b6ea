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


def test_noalloc_rejects_configurations_beyond_its_scratch():
    # k = 2048 at H_I=64 needs ~39 MB of candidate pools, more than 1 MiB
    wl = synth.Workload("noalloc_big", 1, 256, 4, 64, 128, 2048)
    q, w, kc = synth.generate(wl, seed=1, device="cuda")
    rc, idx, _, status = call_noalloc(noalloc_fn(), q, w, kc, 4, 2048, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert rc == SI_ERR_WORKSPACE_TOO_SMALL
    assert int(status.item()) == 99 and int(idx[0, 0, 0].item()) == 7  # nothing was enqueued
