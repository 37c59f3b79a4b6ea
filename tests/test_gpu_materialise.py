"""Streaming top-k against materialise-then-select on the GPU.

The pages compare their streaming indexer with a baseline that materialises
the scores and then takes the top-k (StreamIndex: Memory-Bounded Compressed
Sparse Attention via Streaming Top-k, Abstract).  Here the dense [B,S,T]
scores come from si_indexer_scores (the same TMA + tcgen05 pipeline, no
selection), torch masks and stable-sorts them, and the result must equal
si_indexer_topk bit for bit: same indices, same score bits, same padding.
"""
import numpy as np
import pytest
import torch

import streaming_top_indexer_b200 as si
from streaming_top_indexer_b200 import synth
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu

DEV = "cuda"


def materialise_topk(q, w, kc, m, k):
    """Top-k rows from the dense scores: score descending, index ascending,
    padded with (-1, -inf) past the visible keys."""
    dense = si.indexer_scores(q, w, kc, m)  # NaN where a key is not visible
    B, S, T = dense.shape
    sc = torch.where(torch.isnan(dense), torch.full_like(dense, float("-inf")), dense)
    # a stable sort on the negated scores keeps equal scores in index order
    order = torch.sort(-sc, dim=-1, stable=True).indices.to(torch.int32)
    top_sc = torch.gather(sc, -1, order.long())
    kk = min(k, T)
    idx = torch.full((B, S, k), -1, dtype=torch.int32, device=q.device)
    score = torch.full((B, S, k), float("-inf"), dtype=torch.float32, device=q.device)
    idx[..., :kk] = order[..., :kk]
    score[..., :kk] = top_sc[..., :kk]
    t = torch.arange(S, device=q.device)
    vis = torch.clamp((t + 1) // m, max=T)  # visible keys of each query
    pad = torch.arange(k, device=q.device)[None, :] >= vis[:, None]
    idx[:, pad] = -1
    score[:, pad] = float("-inf")
    return idx, score


CASES = [
    # B, S, T, H, D, m, k
    (1, 1000, 250, 64, 128, 4, 64),
    (2, 777, 300, 32, 128, 2, 100),
    (1, 555, 555, 16, 64, 1, 33),
    (1, 2000, 500, 64, 64, 4, 600),    # k > T
    (3, 160, 20, 8, 128, 7, 5),        # T > S/m
    (1, 4096, 1024, 64, 128, 4, 512),  # several pool cuts per query
]


@pytest.mark.parametrize("B,S,T,H,D,m,k", CASES)
def test_streaming_equals_materialise(B, S, T, H, D, m, k):
    wl = synth.Workload("mat", B, S, m, H, D, k)
    q, w, kc = synth.generate(wl, seed=S + k, device=DEV, T=T)
    got_idx, got_sc = gh.gpu_topk(q, w, kc, m, k)
    ref_idx, ref_sc = materialise_topk(q, w, kc, m, k)
    assert torch.equal(got_idx, ref_idx)
    assert torch.equal(got_sc.view(torch.int32), ref_sc.view(torch.int32))


def test_streaming_equals_materialise_with_ties():
    """Tie-heavy keys (16-row codebook): many exactly equal scores, ordered by
    index on both sides."""
    wl = synth.Workload("mat_tie", 1, 2048, 4, 64, 128, 256, "tieheavy")
    q, w, kc = synth.generate(wl, seed=7, device=DEV)
    got_idx, got_sc = gh.gpu_topk(q, w, kc, wl.m, wl.k)
    ref_idx, ref_sc = materialise_topk(q, w, kc, wl.m, wl.k)
    assert torch.equal(got_idx, ref_idx)
    assert torch.equal(got_sc.view(torch.int32), ref_sc.view(torch.int32))


def materialise_topk_chunked(dense, m, k, rows=4096):
    """materialise_topk's selection on given dense scores, sorted in blocks of
    rows (the full-size cases hold a [S, T] fp32 tensor of gigabytes)."""
    B, S, T = dense.shape
    idx = torch.full((B, S, k), -1, dtype=torch.int32, device=dense.device)
    score = torch.full((B, S, k), float("-inf"), dtype=torch.float32, device=dense.device)
    kk = min(k, T)
    for b in range(B):
        for t0 in range(0, S, rows):
            t1 = min(S, t0 + rows)
            blk = dense[b, t0:t1]
            sc = torch.where(torch.isnan(blk), torch.full_like(blk, float("-inf")), blk)
            order = torch.sort(-sc, dim=-1, stable=True).indices[:, :kk]
            idx[b, t0:t1, :kk] = order.to(torch.int32)
            score[b, t0:t1, :kk] = torch.gather(sc, -1, order)
            del sc, order
    t = torch.arange(S, device=dense.device)
    vis = torch.clamp((t + 1) // m, max=T)
    pad = torch.arange(k, device=dense.device)[None, :] >= vis[:, None]
    idx[:, pad] = -1
    score[:, pad] = float("-inf")
    return idx, score


@pytest.mark.parametrize("B,S,T,H,D,m,k,kind", [
    (1, 65536, 16384, 64, 128, 4, 512, "normal"),     # the V4-Flash-like shape, every row
    (1, 32768, 8192, 64, 128, 4, 2048, "tieheavy"),   # workspace pools, many equal scores
])
def test_streaming_equals_materialise_at_full_size(B, S, T, H, D, m, k, kind):
    """Every row of a full-size problem, bit for bit: the streaming result
    against a stable sort of the dense scores (thousands of pool cuts and
    unit-end selects per launch)."""
    wl = synth.Workload("mat_full", B, S, m, H, D, k, kind)
    q, w, kc = synth.generate(wl, seed=11, device=DEV, T=T)
    got_idx, got_sc = gh.gpu_topk(q, w, kc, m, k)
    dense = si.indexer_scores(q, w, kc, m)
    del q, w, kc
    ref_idx, ref_sc = materialise_topk_chunked(dense, m, k)
    del dense
    assert torch.equal(got_idx, ref_idx)
    assert torch.equal(got_sc.view(torch.int32), ref_sc.view(torch.int32))


def per_head_materialise_topk(q, w, kc, m, k):
    """The pages' baseline in its own form (StreamIndex, Abstract: public CSA
    code materialises the [B,S,H_I,T] fp32 score tensor before the top-k):
    per-head fp32 scores by torch einsum, ReLU, times w, summed over heads,
    masked to the visible keys, then a stable descending sort (equal scores
    keep ascending key order).  Independent of this library's kernels.
    Returns (order [B,S,T], head-summed scores [B,S,T], visible count [S],
    bytes of the per-head tensor)."""
    B, S, H, D = q.shape
    T = kc.shape[1]
    per_head = torch.einsum("bshd,btd->bsht", q.float(), kc.float())          # [B,S,H,T] fp32
    nbytes = per_head.numel() * 4
    scores = (torch.relu(per_head) * w[..., None]).sum(dim=2)                # [B,S,T]
    del per_head
    t = torch.arange(S, device=q.device)
    vis = (torch.arange(T, device=q.device)[None, :] + 1) * m <= (t[:, None] + 1)
    scores = torch.where(vis[None], scores, torch.full_like(scores, float("-inf")))
    order = torch.sort(-scores, dim=-1, stable=True).indices
    n = torch.clamp((t + 1) // m, max=T)
    return order, scores, n, nbytes


@pytest.mark.parametrize("B,S,T,H,D,m,k", [
    (1, 2048, 512, 64, 128, 4, 64),
    (2, 1024, 256, 64, 128, 4, 100),
    (1, 4096, 1024, 64, 128, 4, 512),
    (1, 2048, 512, 8, 64, 4, 64),
])
def test_streaming_equals_per_head_materialise(B, S, T, H, D, m, k):
    """The streaming top-k against the per-head materialised top-k.  Both
    evaluate the same scores in fp32 in different orders, so each side's
    score of a key is within e (the kernel's first-order fp32 bound) of the
    exact one: the index sets must be equal wherever the materialised scores
    at ranks k and k+1 are more than 4e apart, returned scores within 2e of the
    materialised ones, and recall is at least 0.9995 overall."""
    torch.backends.cuda.matmul.allow_tf32 = False
    wl = synth.Workload("mat_head", B, S, m, H, D, k)
    q, w, kc = synth.generate(wl, seed=S + k + H, device=DEV, T=T)
    got_idx, got_sc = gh.gpu_topk(q, w, kc, m, k)
    order, scores, n, nbytes = per_head_materialise_topk(q, w, kc, m, k)
    assert nbytes == 4 * B * S * H * T
    qa, wa = q.float().abs(), w.abs()
    recalls, clear_rows = [], 0
    for b in range(B):
        kca = kc[b].float().abs()
        for t in range(0, S, max(1, S // 256)):
            nv = int(n[t])
            kk = min(k, nv)
            if kk == 0:
                assert torch.all(got_idx[b, t] == -1)
                continue
            g = got_idx[b, t, :kk].long()
            o = order[b, t, :kk]
            e = 1.01 * (D + H) * 2.0 ** -23 * (wa[b, t][:, None] * (qa[b, t] @ kca.T)).sum(0)   # [T]
            row = scores[b, t]
            assert torch.all((got_sc[b, t, :kk] - row[g]).abs() <= 2 * e[g]), f"row {t}: scores"
            rec = len(set(g.tolist()) & set(o.tolist())) / kk
            recalls.append(rec)
            if nv > k and float(row[order[b, t, k - 1]] - row[order[b, t, k]]) > 4 * float(e.max()):
                assert rec == 1.0, f"row {t}: index sets differ outside the rounding band"
                clear_rows += 1
            elif nv <= k:
                assert rec == 1.0
    assert clear_rows > 0
    assert np.mean(recalls) >= 0.9995 and min(recalls) >= 0.998


def test_materialise_boundary_from_free_memory():
    """The per-head materialised tensor is 4 * B * S * H_I * (S/m) bytes:
    64 * S^2 bytes at H_I = 64, m = 4 (Abstract: 256 GB at S = 65,536).  The
    largest S whose tensor fits this device's free memory, from
    cudaMemGetInfo; the pages' materialise path fails at S = 65,536 on an H200
    and fits at S = 32,768, and a 180 GB B200 falls between those."""
    free, total = torch.cuda.mem_get_info()
    s_max = int((free / 64) ** 0.5)
    print(f"free {free / 1e9:.1f} GB of {total / 1e9:.1f} GB: per-head materialise fits up to S = {s_max}")
    assert 4 * 1 * 65536 * 64 * (65536 // 4) == 256 * 2 ** 30
    assert 32768 < s_max < 65536
