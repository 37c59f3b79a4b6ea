"""CSA sparse attention (si_sparse_attention) against the fp64 oracle on the
GPU: every checked output element within the derived fp32/bf16 error bound,
lse likewise, empty rows exactly 0 / -inf (needs a B200)."""
import numpy as np
import pytest
import torch

import streaming_top_indexer_b200 as si
from oracle import attention as att
from streaming_top_indexer_b200 import synth
from tests import checker
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu

DEV = "cuda"


def check_attention(q, kc, vc, idx, scale, b_rows=None, t_rows=None, where=""):
    out, lse, status = si.sparse_attention(q, kc, vc, idx, scale)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"{where}: device status {int(status.item())}"
    B, S = idx.shape[:2]
    if b_rows is None:
        b_rows, t_rows = gh.all_rows(B, S)
    b_rows = np.asarray(b_rows, np.int64)
    t_rows = np.asarray(t_rows, np.int64)
    bt = torch.from_numpy(b_rows).to(DEV)
    tt = torch.from_numpy(t_rows).to(DEV)
    q_rows = synth.bf16_bits(q[bt, tt])
    idx_rows = idx[bt, tt].cpu().numpy()
    kb, vb = synth.bf16_bits(kc), synth.bf16_bits(vc)
    ref, ref_lse, absw = att.sparse_attention_rows(q_rows, idx_rows, b_rows, kb, vb, scale, want_absw=True)
    got = out[bt, tt].float().cpu().numpy().astype(np.float64)
    got_lse = lse[bt, tt].cpu().numpy().astype(np.float64)
    tol, tol_lse = checker.attention_tolerance(q_rows, kb, b_rows, idx_rows, scale, absw, ref, ref_lse)
    empty = np.isneginf(ref_lse)
    assert np.all(got[empty] == 0) and np.all(np.isneginf(got_lse[empty])), f"{where}: empty rows"
    full = ~empty
    err = np.abs(got - ref)
    bad = err[full] > tol[full]
    assert not np.any(bad), f"{where}: {bad.sum()} outputs outside the bound, worst err {err[full].max():.3g}"
    lerr = np.abs(got_lse[full] - ref_lse[full])
    assert np.all(lerr <= tol_lse[full]), f"{where}: lse err {lerr.max():.3g}"
    return {"max_err": float(err[full].max()) if full.any() else 0.0,
            "max_err_over_tol": float((err[full] / tol[full]).max()) if full.any() else 0.0}


@pytest.mark.parametrize("D,DV", [(128, 128), (64, 64), (64, 128), (128, 64)])
def test_on_indexer_output_all_rows(D, DV):
    """The indexer's own top-k (with its -1 padding on early rows) feeds the
    attention; every row of a small problem is checked."""
    B, S, m, k = 2, 600, 4, 64
    wl = synth.Workload("attn", B, S, m, 64, 128, k)
    qi, wi, kci = synth.generate(wl, seed=31, device=DEV)
    idx, _ = gh.gpu_topk(qi, wi, kci, m, k)
    q, kc, vc = synth.generate_attention(B, S, wl.T, D, DV, seed=31, device=DEV)
    check_attention(q, kc, vc, idx, 1.0 / np.sqrt(D), where=f"indexer d={D} dv={DV}")


@pytest.mark.parametrize("k", [1, 63, 64, 100, 512, 2048])
def test_random_selections(k):
    """Random index rows: several chunks and a ragged last one, padding at
    random positions, repeated keys."""
    B, S, T = 2, 40, 3000
    rng = np.random.default_rng(k)
    q, kc, vc = synth.generate_attention(B, S, T, seed=k, device=DEV)
    idx = rng.integers(0, T, (B, S, k)).astype(np.int32)
    idx[rng.random((B, S, k)) < 0.1] = -1
    if k >= 4:
        idx[:, :, 1] = idx[:, :, 0]  # a repeated key counts twice
    idx[0, 3] = -1                   # an empty row
    check_attention(q, kc, vc, torch.from_numpy(idx).to(DEV), 0.0883883, where=f"k={k}")


def test_running_max_rescale():
    """Each chunk of 64 keys scores far above the previous one (by about 16
    in base-2 units), so O in TMEM is rescaled at every chunk."""
    B, S, T, k = 1, 16, 512, 512
    q, _, vc = synth.generate_attention(B, S, T, seed=5, device=DEV)
    q.zero_()
    q[..., 0] = 16.0
    a = (torch.arange(T, device=DEV) // 64).float() * 8.0
    kc = torch.zeros((B, T, 128), dtype=torch.bfloat16, device=DEV)
    kc[..., 0] = a.to(torch.bfloat16)
    kc[..., 1:] = (0.01 * torch.randn((B, T, 127), device=DEV)).to(torch.bfloat16)
    idx = torch.arange(T, dtype=torch.int32, device=DEV).repeat(B, S, 1)
    check_attention(q, kc, vc, idx, 1.0 / np.sqrt(128), where="rescale")
    # and the decreasing order: no rescale after the first chunk
    check_attention(q, kc, vc, idx.flip(-1).contiguous(), 1.0 / np.sqrt(128), where="no rescale")


def test_out_of_range_entries_are_skipped():
    """Entries >= T are skipped like -1: same output as with those entries
    replaced by -1."""
    B, S, T, k = 1, 30, 200, 96
    rng = np.random.default_rng(3)
    q, kc, vc = synth.generate_attention(B, S, T, seed=3, device=DEV)
    idx = rng.integers(0, T, (B, S, k)).astype(np.int32)
    bad = rng.random((B, S, k)) < 0.2
    idx_bad = idx.copy()
    idx_bad[bad] = T + rng.integers(0, 1000, bad.sum())
    idx[bad] = -1
    a, la, _ = si.sparse_attention(q, kc, vc, torch.from_numpy(idx_bad).to(DEV), 0.1)
    b, lb, _ = si.sparse_attention(q, kc, vc, torch.from_numpy(idx).to(DEV), 0.1)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(la, lb)


def test_no_keys_at_all():
    q, _, _ = synth.generate_attention(1, 8, 1, seed=1, device=DEV)
    kc = torch.empty((1, 0, 128), dtype=torch.bfloat16, device=DEV)
    vc = torch.empty((1, 0, 128), dtype=torch.bfloat16, device=DEV)
    idx = torch.full((1, 8, 16), -1, dtype=torch.int32, device=DEV)
    out, lse, status = si.sparse_attention(q, kc, vc, idx, 0.1)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))


def test_deterministic():
    B, S, T, k = 1, 300, 1000, 512
    rng = np.random.default_rng(9)
    q, kc, vc = synth.generate_attention(B, S, T, seed=9, device=DEV)
    idx = torch.from_numpy(rng.integers(0, T, (B, S, k)).astype(np.int32)).to(DEV)
    a = si.sparse_attention(q, kc, vc, idx, 0.0883883)
    b = si.sparse_attention(q, kc, vc, idx, 0.0883883)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_long_workload_composed_with_indexer():
    """The CSA step at the headline shape: the indexer's top-512 of
    S=262,144 queries over T=65,536 compressed keys, then the sparse
    attention (128 heads, d = d_v = 128) over them; 48 seeded rows plus edge
    rows against the oracle."""
    wl = synth.WORKLOADS["long"]
    qi, wi, kci = synth.generate(wl, seed=0, device=DEV)
    idx, _ = gh.gpu_topk(qi, wi, kci, wl.m, wl.k)
    del qi, wi
    q, kc, vc = synth.generate_attention(1, wl.S, wl.T, seed=0, device=DEV)
    samp, edges = synth.checked_rows(wl.S, wl.m, wl.k, 0, seed=0, n=48)
    t_rows = np.concatenate([samp, edges])
    rep = check_attention(q, kc, vc, idx, 1.0 / np.sqrt(128), np.zeros_like(t_rows), t_rows, where="long")
    assert rep["max_err_over_tol"] <= 1.0
