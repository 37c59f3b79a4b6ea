"""Host-side logic of bench.py that needs no GPU: the materialised top-k used
by the sweep's recall check, and the causal pair count behind the TFLOP/s."""
import numpy as np
import torch

import bench


def test_materialised_topk_rows_matches_a_plain_sort():
    rng = np.random.default_rng(0)
    S, T, m, k = 40, 10, 4, 6
    dense = torch.tensor(rng.integers(-3, 4, size=(S, T)).astype(np.float32))  # many ties
    for t in range(S):
        dense[t, min(T, (t + 1) // m):] = float("nan")  # keys the row cannot see
    rows = torch.arange(S)
    order, vis = bench.materialised_topk_rows(dense, rows, m, k)
    for t in range(S):
        V = min(T, (t + 1) // m)
        assert int(vis[t]) == V
        want = sorted(range(V), key=lambda s: (-float(dense[t, s]), s))[:min(k, V)]
        assert order[t, :len(want)].tolist() == want


def test_visible_pairs_closed_form():
    for B, S, T, m in [(1, 2048, 512, 4), (2, 777, 300, 2), (3, 160, 20, 7), (1, 262144, 65536, 4)]:
        t = np.arange(S, dtype=np.int64)
        brute = B * int(np.minimum(T, (t + 1) // m).sum())
        assert bench.visible_pairs(B, S, T, m) == brute
