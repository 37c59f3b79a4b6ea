"""Row windows (si_indexer_topk_rows) and the pipelined host entry point
built on them (si_indexer_topk_host): the same rows as the whole-problem
call, bit for bit."""
import pytest
import torch

import streaming_top_indexer_b200 as si
from streaming_top_indexer_b200 import synth

pytestmark = pytest.mark.gpu

DEV = "cuda"

SHAPES = [
    # B, S, T, H, D, m, k
    (1, 1000, 250, 64, 128, 4, 64),
    (2, 777, 300, 32, 128, 2, 100),
    (1, 2000, 500, 64, 64, 4, 600),   # k > T
    (3, 600, 40, 8, 128, 7, 5),       # T > S/m
    (1, 1500, 375, 64, 128, 4, 2048),  # workspace pools
]


def inputs(B, S, T, H, D, m, k, seed):
    wl = synth.Workload("rows", B, S, m, H, D, k)
    return synth.generate(wl, seed=seed, device=DEV, T=T)


@pytest.mark.parametrize("B,S,T,H,D,m,k", SHAPES)
def test_windows_equal_whole_call(B, S, T, H, D, m, k):
    q, w, kc = inputs(B, S, T, H, D, m, k, seed=S + 7)
    ws = torch.zeros(si.workspace_bytes(B, S, T, H, D, m, k), dtype=torch.uint8, device=DEV)
    ref_idx, ref_sc = si.indexer_topk(q, w, kc, m, k, workspace=ws)
    assert si.check_device_status(ws) == 0
    idx = torch.full((B, S, k), -7, dtype=torch.int32, device=DEV)
    sc = torch.full((B, S, k), 7.0, dtype=torch.float32, device=DEV)
    si.reset_device_status(ws)
    for t0, t1 in si.host_row_windows(S, 3)[::-1]:  # any order
        si.indexer_topk_rows(q, w, kc, m, k, t0, t1, idx, sc, ws)
    assert si.check_device_status(ws) == 0
    assert torch.equal(idx, ref_idx)
    assert torch.equal(sc.view(torch.int32), ref_sc.view(torch.int32))


def test_window_touches_only_its_rows():
    B, S, T, H, D, m, k = 2, 1024, 256, 64, 128, 4, 32
    q, w, kc = inputs(B, S, T, H, D, m, k, seed=3)
    ws = torch.zeros(si.workspace_bytes(B, S, T, H, D, m, k), dtype=torch.uint8, device=DEV)
    ref_idx, ref_sc = si.indexer_topk(q, w, kc, m, k, workspace=ws)
    idx = torch.full((B, S, k), -7, dtype=torch.int32, device=DEV)
    sc = torch.full((B, S, k), 7.0, dtype=torch.float32, device=DEV)
    si.indexer_topk_rows(q, w, kc, m, k, 256, 768, idx, sc, ws)
    assert si.check_device_status(ws) == 0
    assert torch.equal(idx[:, 256:768], ref_idx[:, 256:768])
    assert torch.equal(sc[:, 256:768], ref_sc[:, 256:768])
    assert torch.all(idx[:, :256] == -7) and torch.all(idx[:, 768:] == -7)
    assert torch.all(sc[:, :256] == 7.0) and torch.all(sc[:, 768:] == 7.0)


@pytest.mark.parametrize("chunks", [1, 4])
def test_pipelined_host_path_equals_device_call(chunks):
    B, S, T, H, D, m, k = 1, 4096, 1024, 64, 128, 4, 512
    q, w, kc = inputs(B, S, T, H, D, m, k, seed=11)
    ref_idx, ref_sc = si.indexer_topk(q, w, kc, m, k)
    qh, wh, kch = q.cpu().pin_memory(), w.cpu().pin_memory(), kc.cpu().pin_memory()
    bufs = {}
    for _ in range(2):  # buffers and streams reused on the second call
        idx_h, sc_h = si.indexer_topk_host(qh, wh, kch, m, k, device=DEV, buffers=bufs, chunks=chunks)
        torch.cuda.current_stream().synchronize()
        assert si.check_device_status(bufs["ws"]) == 0
        assert torch.equal(idx_h, ref_idx.cpu())
        assert torch.equal(sc_h.view(torch.int32), ref_sc.cpu().view(torch.int32))


@pytest.mark.parametrize("B,S,T,H,D,m,k", SHAPES)
@pytest.mark.parametrize("pinned", [True, False])
def test_host_entry_equals_device_call(B, S, T, H, D, m, k, pinned):
    """Ragged S, several batches (strided row copies), k > T, T > S/m and
    workspace pools, from page-locked and from pageable host memory."""
    q, w, kc = inputs(B, S, T, H, D, m, k, seed=S + 11)
    ref_idx, ref_sc = si.indexer_topk(q, w, kc, m, k)
    qh, wh, kch = q.cpu(), w.cpu(), kc.cpu()
    if pinned:
        qh, wh, kch = qh.pin_memory(), wh.pin_memory(), kch.pin_memory()
    bufs = {}
    idx_h, sc_h = si.indexer_topk_host(qh, wh, kch, m, k, device=DEV, buffers=bufs, chunks=3)
    torch.cuda.current_stream().synchronize()
    assert si.check_device_status(bufs["ws"]) == 0
    assert torch.equal(idx_h, ref_idx.cpu())
    assert torch.equal(sc_h.view(torch.int32), ref_sc.cpu().view(torch.int32))


def test_host_entry_with_no_keys_gives_padding():
    B, S, H, D, m, k = 2, 600, 64, 128, 4, 8
    q, w, _ = inputs(B, S, 4, H, D, m, k, seed=6)
    kc = torch.empty((B, 0, D), dtype=torch.bfloat16)
    idx_h, sc_h = si.indexer_topk_host(q.cpu().pin_memory(), w.cpu().pin_memory(), kc, m, k, device=DEV, chunks=2)
    torch.cuda.current_stream().synchronize()
    assert torch.all(idx_h == -1) and torch.all(torch.isneginf(sc_h))


def test_host_entry_waits_for_work_queued_before():
    """A second call may reuse the buffers at once: its copies in wait for the
    first call's reads of them (both queued without a synchronisation)."""
    B, S, T, H, D, m, k = 1, 2048, 512, 64, 128, 4, 64
    q1, w1, kc1 = inputs(B, S, T, H, D, m, k, seed=21)
    q2, w2, kc2 = inputs(B, S, T, H, D, m, k, seed=22)
    r1 = si.indexer_topk(q1, w1, kc1, m, k)
    r2 = si.indexer_topk(q2, w2, kc2, m, k)
    h1 = [t.cpu().pin_memory() for t in (q1, w1, kc1)]
    h2 = [t.cpu().pin_memory() for t in (q2, w2, kc2)]
    bufs = {}
    i1, s1 = si.indexer_topk_host(*h1, m, k, device=DEV, buffers=bufs, chunks=4)
    torch.cuda.current_stream().synchronize()
    assert torch.equal(i1, r1[0].cpu()) and torch.equal(s1, r1[1].cpu())
    si.indexer_topk_host(*h1, m, k, device=DEV, buffers=bufs, chunks=4)
    i2, s2 = si.indexer_topk_host(*h2, m, k, device=DEV, buffers=bufs, chunks=4)  # no synchronisation between
    torch.cuda.current_stream().synchronize()
    assert torch.equal(i2, r2[0].cpu()) and torch.equal(s2, r2[1].cpu())


def test_windows_with_no_keys_give_padding():
    B, S, T, H, D, m, k = 2, 600, 0, 64, 128, 4, 8
    q, w, _ = inputs(B, S, 4, H, D, m, k, seed=5)
    kc = torch.empty((B, 0, D), dtype=torch.bfloat16, device=DEV)
    ws = torch.zeros(si.workspace_bytes(B, S, T, H, D, m, k), dtype=torch.uint8, device=DEV)
    idx = torch.zeros((B, S, k), dtype=torch.int32, device=DEV)
    sc = torch.zeros((B, S, k), dtype=torch.float32, device=DEV)
    si.reset_device_status(ws)
    for t0, t1 in si.host_row_windows(S, 2):
        si.indexer_topk_rows(q, w, kc, m, k, t0, t1, idx, sc, ws)
    assert si.check_device_status(ws) == 0
    assert torch.all(idx == -1) and torch.all(torch.isneginf(sc))


def test_reset_clears_a_recorded_timeout():
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    assert si.selftest_timeout(ws, limit_ns=5_000_000) == 6  # SI_ERR_TIMEOUT recorded
    assert si.check_device_status(ws) == 6                    # and kept
    si.reset_device_status(ws)
    assert si.check_device_status(ws) == 0
