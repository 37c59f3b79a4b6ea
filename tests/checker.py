"""Acceptance rules comparing the CUDA path's top-k rows with the oracle's.

Rules (the indexer step's exact top-k, StreamIndex: Memory-Bounded
Compressed Sparse Attention via Streaming Top-k, Abstract; the Abstract
measures set-overlap recall against the materialised ground truth):

1. invariants of every GPU row: indices visible and distinct, scores
   non-increasing with equal scores in ascending index order, padding
   (-1, -inf) exactly at positions >= min(k, V_t);
2. where V_t > k and the oracle's k-th and (k+1)-th scores differ by more
   than BAND * max|score| of the row, the GPU index set equals the oracle's;
   positions whose oracle score is separated from both neighbours by more
   than the band hold the same index;
3. every returned score is within SCORE_RTOL of the oracle's score of that
   key, relative to max(|oracle score|, 1e-2 * row max);
4. set-overlap recall |G & O| / min(k, V_t) over rows with V_t > 0:
   mean >= 0.9995 and min >= 0.998.
"""
from __future__ import annotations

import numpy as np

BAND = 2e-3
SCORE_RTOL = 2e-3
RECALL_MEAN = 0.9995
RECALL_MIN = 0.998


class Report(dict):
    pass


def check_rows(g_idx, g_score, o_idx, o_score, o_meta, o_scores, k, where="") -> Report:
    """Check GPU rows against oracle rows; raises AssertionError on failure.

    g_idx int32 [R,k], g_score float32 [R,k]: GPU output rows.
    o_idx, o_score, o_meta, o_scores: oracle.topk_rows(..., want_scores=True).
    """
    g_idx = np.asarray(g_idx)
    g_score = np.asarray(g_score, np.float64)
    R = g_idx.shape[0]
    recalls = []
    exact_rows = 0
    exact_needed = 0
    for r in range(R):
        V = int(o_meta[r, 3])
        rowmax = float(o_meta[r, 0])
        n = min(k, V)
        gi, gs = g_idx[r], g_score[r]
        tag = f"{where} row {r}"
        # 1. invariants
        assert np.all(gi[n:] == -1), f"{tag}: padding indices {gi[n:][:8]}"
        assert np.all(np.isneginf(gs[n:])), f"{tag}: padding scores"
        sel = gi[:n]
        assert np.all((sel >= 0) & (sel < V)), f"{tag}: index outside visible range"
        assert len(np.unique(sel)) == n, f"{tag}: duplicate indices"
        s = gs[:n]
        assert np.all(np.isfinite(s)), f"{tag}: non-finite score"
        assert np.all(s[:-1] >= s[1:]), f"{tag}: scores not non-increasing"
        eq = s[:-1] == s[1:]
        assert np.all(sel[:-1][eq] < sel[1:][eq]), f"{tag}: equal scores not in index order"
        if V == 0:
            continue
        # 3. score tolerance against the oracle's score of the same key
        ref = o_scores[r, sel]
        tol = SCORE_RTOL * np.maximum(np.abs(ref), 1e-2 * rowmax)
        bad = np.abs(s - ref) > tol
        assert not np.any(bad), (f"{tag}: score mismatch at {np.nonzero(bad)[0][:5]}: "
                                 f"gpu {s[bad][:5]} oracle {ref[bad][:5]}")
        # 2. exact index set outside the tie band
        oi = o_idx[r, :n]
        if V > k:
            gap = o_meta[r, 1] - o_meta[r, 2]
            if gap > BAND * rowmax:
                exact_needed += 1
                assert set(sel.tolist()) == set(oi.tolist()), (
                    f"{tag}: index set differs outside the tie band (gap {gap:.3g}, "
                    f"rowmax {rowmax:.3g})")
                os_ = o_score[r, :n]
                sep = np.ones(n, bool)
                d = np.diff(os_)
                sep[:-1] &= -d > BAND * rowmax
                sep[1:] &= -d > BAND * rowmax
                assert np.array_equal(sel[sep], oi[sep]), f"{tag}: order differs at separated positions"
                exact_rows += 1
        else:
            assert set(sel.tolist()) == set(range(V)), f"{tag}: rows with V<=k return every visible key"
        recalls.append(len(np.intersect1d(sel, oi)) / n)
    rec = np.asarray(recalls) if recalls else np.ones(1)
    rep = Report(rows=R, recall_mean=float(rec.mean()), recall_min=float(rec.min()),
                 exact_rows=exact_rows, exact_needed=exact_needed)
    assert rep["recall_mean"] >= RECALL_MEAN, f"{where}: mean recall {rep['recall_mean']}"
    assert rep["recall_min"] >= RECALL_MIN, f"{where}: min recall {rep['recall_min']}"
    return rep
