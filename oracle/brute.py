"""Second, independent restatement of the oracle in numpy, for tiny inputs.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).  It recomputes the CSA
indexer top-k (StreamIndex: Memory-Bounded Compressed Sparse Attention via
Streaming Top-k, Abstract) with numpy's matmul and a lexicographic sort, so
that a stride or sort mistake in si_oracle.c shows up as a disagreement.  It
is a cross-check of the C code, not a pin of the definition.
"""
from __future__ import annotations

import numpy as np


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def topk_all_rows(q_bits, w, kc_bits, m: int, k: int, with_meta: bool = False):
    """Top-k of every query row; q_bits [B,S,H,D], w [B,S,H], kc_bits [B,T,D].

    With ``with_meta`` also returns the per-row meta [B,S,4]: max |score|
    over the visible keys (0 if none), the scores at ranks k and k+1 (NaN
    where the row has fewer keys) and the visible count."""
    q = bf16_bits_to_f64(q_bits)
    kc = bf16_bits_to_f64(kc_bits)
    w = np.asarray(w, np.float32).astype(np.float64)
    B, S, H, D = q.shape
    T = kc.shape[1]
    idx = np.full((B, S, k), -1, np.int32)
    score = np.full((B, S, k), -np.inf)
    meta = np.full((B, S, 4), np.nan)
    meta[..., 0] = 0.0
    meta[..., 3] = 0.0
    s_all = np.arange(T)
    for b in range(B):
        for t in range(S):
            vis = s_all[(s_all + 1) * m <= t + 1]
            if vis.size == 0:
                continue
            x = q[b, t] @ kc[b, vis].T                     # [H, V]
            sc = (w[b, t][:, None] * np.maximum(x, 0.0)).sum(axis=0)
            order = np.lexsort((vis, -sc))                 # score desc, idx asc
            n = min(k, vis.size)
            idx[b, t, :n] = vis[order[:n]]
            score[b, t, :n] = sc[order[:n]]
            ranked = sc[order]
            meta[b, t, 0] = np.abs(sc).max()
            meta[b, t, 1] = ranked[k - 1] if vis.size >= k else np.nan
            meta[b, t, 2] = ranked[k] if vis.size > k else np.nan
            meta[b, t, 3] = vis.size
    if with_meta:
        return idx, score, meta
    return idx, score
