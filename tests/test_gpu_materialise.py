"""Streaming top-k against materialise-then-select on the GPU.

The pages compare their streaming indexer with a baseline that materialises
the scores and then takes the top-k (StreamIndex: Memory-Bounded Compressed
Sparse Attention via Streaming Top-k, Abstract).  Here the dense [B,S,T]
scores come from si_indexer_scores (the same TMA + tcgen05 pipeline, no
selection), torch masks and stable-sorts them, and the result must equal
si_indexer_topk bit for bit: same indices, same score bits, same padding.
"""
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
