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
3. every returned score is within max(SCORE_RTOL * |oracle score|, e) of
   the oracle's score of that key, where e is the a-priori error bound of the
   kernel's fp32 evaluation of that score (score_error_bound): the relative
   test alone cannot hold where the head sum cancels to near zero;
4. set-overlap recall |G & O| / min(k, V_t) over rows with V_t > 0:
   mean >= 0.9995 and min >= 0.998.
"""
from __future__ import annotations

import numpy as np

BAND = 2e-3
SCORE_RTOL = 2e-3
RECALL_MEAN = 0.9995
RECALL_MIN = 0.998


# Unit roundoff allowed per fp32 addition: 2^-23 (one ulp), which also covers
# an accumulator that truncates instead of rounding to nearest.
FP32_ULP = 2.0 ** -23


class Report(dict):
    pass


def score_error_bound(q_rows_bits, w_rows, kc_bits, row_b, sel):
    """First-order bound on |fp32 score - exact score| for each selected key.

    The kernel computes acc_h = sum_d q[h,d]*kc[d] in fp32 (every bf16 x bf16
    product is exact in fp32; D-1 additions), then ReLU (exact, 1-Lipschitz)
    and score = sum_h w[h]*ReLU(acc_h) with fused multiply-adds (H-1 rounded
    additions).  With A_h = sum_d |q[h,d]*kc[d]| >= |acc_h| this gives

        |error| <= (D + H) * 2^-23 * sum_h |w[h]| * A_h      (times 1.01)

    q_rows_bits uint16 [R,H,D], w_rows float32 [R,H], kc_bits uint16 [B,T,D],
    row_b int64 [R], sel int [R,n] key indices (negative entries: padding,
    bound 0).  Returns float64 [R,n]."""
    def f64(bits):
        return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)

    qa = np.abs(f64(q_rows_bits))
    wa = np.abs(np.asarray(w_rows, np.float64))
    sel = np.asarray(sel)
    R, H, D = qa.shape
    out = np.zeros(sel.shape, np.float64)
    for r in range(R):
        ok = sel[r] >= 0
        if not ok.any():
            continue
        kca = np.abs(f64(kc_bits[row_b[r], sel[r][ok]]))   # [n, D]
        A = qa[r] @ kca.T                                    # [H, n]
        out[r, ok] = 1.01 * (D + H) * FP32_ULP * (wa[r] @ A)
    return out


def check_rows(g_idx, g_score, o_idx, o_score, o_meta, o_scores, k, bound, where="") -> Report:
    """Check GPU rows against oracle rows; raises AssertionError on failure.

    g_idx int32 [R,k], g_score float32 [R,k]: GPU output rows.
    o_idx, o_score, o_meta, o_scores: oracle.topk_rows(..., want_scores=True).
    bound float64 [R,k]: score_error_bound of the GPU's selected keys.
    """
    g_idx = np.asarray(g_idx)
    g_score = np.asarray(g_score, np.float64)
    R = g_idx.shape[0]
    recalls = []
    exact_rows = 0
    exact_needed = 0
    scores_compared = 0
    scores_on_bound = 0
    max_rel_err = 0.0
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
        rel = SCORE_RTOL * np.abs(ref)
        eb = bound[r, :n]
        tol = np.maximum(rel, eb)
        err = np.abs(s - ref)
        bad = err > tol
        scores_compared += n
        scores_on_bound += int(np.count_nonzero(eb > rel))
        nz = ref != 0
        if nz.any():
            max_rel_err = max(max_rel_err, float((err[nz] / np.abs(ref[nz])).max()))
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
                 exact_rows=exact_rows, exact_needed=exact_needed, scores_compared=scores_compared,
                 scores_on_bound=scores_on_bound, max_rel_err=max_rel_err)
    assert rep["recall_mean"] >= RECALL_MEAN, f"{where}: mean recall {rep['recall_mean']}"
    assert rep["recall_min"] >= RECALL_MIN, f"{where}: min recall {rep['recall_min']}"
    return rep


def attention_tolerance(q_rows_bits, kc_bits, row_b, idx_rows, scale, absw, ref_out, ref_lse):
    """First-order error bounds of the GPU sparse attention against the fp64
    oracle, per output element and per lse value.

    The kernel computes each score in fp32 from exact bf16 products
    (error e_j <= d * 2^-23 * scale * sum_d |q_d K_jd|), exponentiates with
    ex2.approx (relative error below 2^-21), rounds the weights to bf16 for
    the P.V product while l sums them in fp32, accumulates in fp32
    (n * 2^-23 relative of sum_j p_j |V_j|), and rounds the output to bf16.
    bf16 keeps 8 significant bits, so each of its roundings is within 2^-8
    relative.  With E = 2 * max_j e_j over the row's keys, n the number of
    keys, A = sum_j p_j |V_j| (absw) and O the exact output:

        |out - O| <= 1.1 * (2^-8 + E + n 2^-23 + 2^-20) * (A + |O|)
        |lse - L| <= 1.1 * (E + n 2^-23 + 2^-19) + 2^-22 |L|
    Returns (tol_out [R,H,DV], tol_lse [R,H])."""
    def f64(bits):
        return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)

    qa = np.abs(f64(q_rows_bits))                       # [R,H,D]
    R, H, D = qa.shape
    tol_out = np.zeros(ref_out.shape)
    tol_lse = np.zeros(ref_lse.shape)
    T = kc_bits.shape[1]
    for r in range(R):
        sel = idx_rows[r][(idx_rows[r] >= 0) & (idx_rows[r] < T)]
        n = len(sel)
        if n == 0:
            continue
        ka = np.abs(f64(kc_bits[row_b[r], sel]))        # [n, D]
        E = 2 * D * FP32_ULP * abs(scale) * (qa[r] @ ka.T).max(axis=1)   # [H]
        eps = 2.0 ** -8 + E + n * FP32_ULP + 2.0 ** -20
        tol_out[r] = 1.1 * eps[:, None] * (absw[r] + np.abs(ref_out[r]))
        tol_lse[r] = 1.1 * (E + n * FP32_ULP + 2.0 ** -19) + 2.0 ** -22 * np.abs(ref_lse[r])
    return tol_out, tol_lse
