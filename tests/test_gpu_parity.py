"""CUDA path vs the CPU oracle on seeded inputs (needs a B200)."""
import math

import numpy as np
import pytest
import torch

import streaming_top_indexer_b200 as si
from streaming_top_indexer_b200 import synth
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu

DEV = "cuda"


def make(B, S, T, H, D, m, k, seed=0, kind="normal"):
    wl = synth.Workload("case", B, S, m, H, D, k, kind)
    return synth.generate(wl, seed=seed, device=DEV, T=T)


def test_library_loads_and_reports_version():
    assert "sm_100a" in si.version()


def test_dense_scores_match_oracle():
    """Materialise path through the same TMA + tcgen05 pipeline: every
    visible score against the fp64 oracle."""
    for (B, S, T, H, D, m) in [(1, 300, 75, 8, 64, 4), (2, 130, 130, 64, 128, 1), (1, 517, 200, 16, 128, 2)]:
        q, w, kc = make(B, S, T, H, D, m, 1, seed=S)
        dense = si.indexer_scores(q, w, kc, m).cpu().numpy()
        b_rows, t_rows = gh.all_rows(B, S)
        _, _, meta, ref = gh.oracle_rows(q, w, kc, m, 1, b_rows, t_rows)
        got = dense.reshape(B * S, T)
        vis = ~np.isnan(ref)
        assert np.array_equal(~np.isnan(got), vis), "visible pattern differs"
        tol = 1e-5 * np.maximum(meta[:, :1], 1.0) + 1e-5 * np.abs(ref)
        err = np.abs(got - ref)
        assert np.all(err[vis] <= np.broadcast_to(tol, ref.shape)[vis]), f"max err {np.nanmax(err)}"


def test_tiny_workload_all_rows():
    """tiny workload: B=1 S=2048 T=512 H_I=8 d_I=64 k=64, every row."""
    wl = synth.WORKLOADS["tiny"]
    q, w, kc = synth.generate(wl, seed=0, device=DEV)
    b_rows, t_rows = gh.all_rows(wl.B, wl.S)
    rep = gh.check_against_oracle(q, w, kc, wl.m, wl.k, b_rows, t_rows, where="tiny")
    assert rep["exact_needed"] > 100  # the exact-index rule binds on many rows here


SHAPES = [
    # B, S, T, H, D, m, k
    (1, 1000, 250, 64, 128, 4, 64),     # several tiles, ragged query block
    (2, 777, 300, 32, 128, 2, 100),     # B=2, T < S/m, ragged everything
    (1, 555, 555, 16, 64, 1, 33),       # m=1
    (3, 160, 20, 8, 128, 7, 5),         # T > S/m, tiny T
    (1, 2000, 500, 64, 64, 4, 600),     # k > T: all padding tails
    (1, 1200, 300, 8, 64, 4, 1),        # k = 1
    (1, 1500, 375, 64, 128, 4, 2048),   # largest k: pools in global memory
    (2, 1100, 275, 16, 128, 4, 300),    # H=16: pools in global memory
    (1, 5, 2, 64, 128, 4, 8),           # tiny S (single ragged block)
]


@pytest.mark.parametrize("B,S,T,H,D,m,k", SHAPES)
def test_shapes_all_rows(B, S, T, H, D, m, k):
    q, w, kc = make(B, S, T, H, D, m, k, seed=B * 1000 + S)
    b_rows, t_rows = gh.all_rows(B, S)
    gh.check_against_oracle(q, w, kc, m, k, b_rows, t_rows, where=f"{(B, S, T, H, D, m, k)}")


def test_all_keys_tied():
    """Identical kc rows: bit-identical scores on the GPU regardless of tile
    position, so each row returns keys 0..min(k,V)-1 in order."""
    B, S, T, H, D, m, k = 1, 3000, 750, 64, 128, 4, 100
    q, w, kc = make(B, S, T, H, D, m, k, seed=5)
    kc[:] = kc[0, 0]
    idx, sc = gh.gpu_topk(q, w, kc, m, k)
    idx = idx.cpu().numpy()[0]
    sc = sc.cpu().numpy()[0]
    for t in range(S):
        n = min(k, min(T, (t + 1) // m))
        assert idx[t, :n].tolist() == list(range(n)), f"row {t}"
        assert np.all(sc[t, :n] == sc[t, 0])


def test_tie_heavy_codebook_small():
    B, S, H, D, m, k = 2, 4096, 64, 128, 4, 256
    wl = synth.Workload("tie_small", B, S, m, H, D, k, "tieheavy")
    q, w, kc = synth.generate(wl, seed=3, device=DEV)
    b_rows, t_rows = gh.all_rows(B, S)
    gh.check_against_oracle(q, w, kc, m, k, b_rows, t_rows, where="tie small")


def test_planted_keys():
    wl = synth.Workload("planted", 1, 16384, 4, 64, 128, 512)
    q, w, kc = synth.generate(wl, seed=11, device=DEV)
    q, w, kc, planted = synth.plant_keys(q, w, kc, wl.k, seed=11)
    idx, _ = gh.gpu_topk(q, w, kc, wl.m, wl.k)
    idx = idx.cpu().numpy()[0]
    P = planted[0].tolist()
    T = wl.T
    for t in range(wl.S):
        V = min(T, (t + 1) // wl.m)
        if V >= T // 2:
            assert idx[t].tolist() == P, f"row {t}"
        else:
            assert set(p for p in P if p < V) <= set(idx[t].tolist()), f"row {t}"


def test_deterministic_repeat():
    q, w, kc = make(1, 4096, 1024, 64, 128, 4, 512, seed=9)
    a = gh.gpu_topk(q, w, kc, 4, 512)
    b = gh.gpu_topk(q, w, kc, 4, 512)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_select_output_is_already_sorted():
    """The select kernel sorts each row at unit end: its output alone equals
    the full call, and sorting it again changes nothing."""
    q, w, kc = make(1, 3000, 750, 64, 128, 4, 128, seed=13)
    assert si.select_sorts_rows(64, 128, 128)
    idx, sc = gh.gpu_topk(q, w, kc, 4, 128)
    i2, s2 = si.select_topk(q, w, kc, 4, 128)
    torch.cuda.synchronize()
    assert torch.equal(idx, i2) and torch.equal(sc, s2)
    si.sort_topk(i2, s2)
    torch.cuda.synchronize()
    assert torch.equal(idx, i2) and torch.equal(sc, s2)


SORT_CASES = [
    # B, S, T, H, D, m, k   (keys per thread of the unit-end sort, pools)
    (1, 1000, 250, 64, 128, 4, 100),    # E=1, shared-memory pools
    (2, 777, 300, 32, 128, 2, 200),     # E=2
    (1, 2000, 500, 64, 64, 4, 600),     # E=8 with k > T (padding inside the sorted rows)
    (1, 9000, 2250, 64, 128, 4, 512),   # E=4, several cuts per query
    (1, 5000, 1250, 64, 128, 4, 1024),  # E=8, shared-memory pools of 1856
    (1, 3000, 750, 64, 128, 4, 1050),   # k > 1024: the kernel leaves rows unordered, the row sort runs
    (1, 2000, 500, 32, 128, 4, 700),    # E=8, workspace pools (the shared-memory buffer)
    (2, 1100, 275, 16, 128, 4, 300),    # H=16: workspace pools, E=4
    (3, 160, 20, 8, 128, 7, 5),         # H=8: 16 queries per half
]


@pytest.mark.parametrize("B,S,T,H,D,m,k", SORT_CASES)
def test_in_kernel_sort_equals_separate_sort(B, S, T, H, D, m, k):
    """Rows sorted at unit end inside the select kernel are bit-identical to
    unordered rows sorted by the separate row-sort kernel."""
    q, w, kc = make(B, S, T, H, D, m, k, seed=B * 77 + S + k)
    a_idx, a_sc = gh.gpu_topk(q, w, kc, m, k)
    si.set_sort_in_select(False)
    try:
        b_idx, b_sc = gh.gpu_topk(q, w, kc, m, k)
    finally:
        si.set_sort_in_select(True)
    assert torch.equal(a_idx, b_idx)
    assert torch.equal(a_sc.view(torch.int32), b_sc.view(torch.int32))


def test_zero_keys_gives_padding():
    q, w, _ = make(1, 64, 4, 64, 128, 4, 8, seed=1)
    kc = torch.empty((1, 0, 128), dtype=torch.bfloat16, device=DEV)
    idx, sc = gh.gpu_topk(q, w, kc, 4, 8)
    assert torch.all(idx == -1) and torch.all(torch.isneginf(sc))


def test_timeout_selftest_reports_and_context_survives():
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    status = si.selftest_timeout(ws, limit_ns=20_000_000)
    assert status == 6  # SI_ERR_TIMEOUT
    q, w, kc = make(1, 256, 64, 64, 128, 4, 8, seed=2)
    idx, _ = gh.gpu_topk(q, w, kc, 4, 8)  # the context is still usable
    assert idx.shape == (1, 256, 8)


def test_workspace_pools_with_streamed_cuts():
    """k=600 at H_I=32 puts the candidate pools in the workspace (4k = 2400
    entries per query), and rows long enough that the pools are cut while
    more than 2048 entries are held: the streamed (not register-held) cut
    path, with the shared-memory exact-cut buffer."""
    wl = synth.Workload("ws_pools", 1, 98304, 4, 32, 128, 600)
    q, w, kc = synth.generate(wl, seed=21, device=DEV)
    b_rows, t_rows = gh.sampled_rows(wl.B, wl.S, wl.m, wl.k, n=256)
    gh.check_against_oracle(q, w, kc, wl.m, wl.k, b_rows, t_rows, where="ws pools")


def test_shared_memory_pools_at_k1024():
    """k=1024 at H_I=64: 1856-entry pools in shared memory, cut often."""
    wl = synth.Workload("smem_k1024", 1, 65536, 4, 64, 128, 1024)
    q, w, kc = synth.generate(wl, seed=23, device=DEV)
    b_rows, t_rows = gh.sampled_rows(wl.B, wl.S, wl.m, wl.k, n=256)
    gh.check_against_oracle(q, w, kc, wl.m, wl.k, b_rows, t_rows, where="smem k=1024")


@pytest.mark.parametrize("name", ["v4flash", "long"])
def test_full_size_sampled_rows(name):
    """Full-size workloads in the benchmark's launch configuration: 512
    seeded rows per batch plus edge rows against the oracle."""
    wl = synth.WORKLOADS[name]
    q, w, kc = synth.generate(wl, seed=0, device=DEV)
    b_rows, t_rows = gh.sampled_rows(wl.B, wl.S, wl.m, wl.k)
    rep = gh.check_against_oracle(q, w, kc, wl.m, wl.k, b_rows, t_rows, where=name)
    assert rep["rows"] >= 512


@pytest.mark.slow
@pytest.mark.parametrize("name", ["tieheavy", "tieheavy_iid", "extreme"])
def test_full_size_sampled_rows_large(name):
    wl = synth.WORKLOADS[name]
    q, w, kc = synth.generate(wl, seed=0, device=DEV)
    b_rows, t_rows = gh.sampled_rows(wl.B, wl.S, wl.m, wl.k)
    gh.check_against_oracle(q, w, kc, wl.m, wl.k, b_rows, t_rows, where=name)
