"""The acceptance checker on the CPU: the fp32 error bound covers an fp32
evaluation of the scores, oracle rows pass, and planted mistakes (on the CPU,
in copies of the oracle's rows) are rejected."""
import numpy as np
import pytest

from oracle import oracle as orc
from tests import checker
from tests import oracle_pins as pins


def _bits_to_f32(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def _case(seed=0, S=96, m=4, H=8, D=64, k=6, B=2):
    rng = np.random.default_rng(seed)
    T = S // m
    q = pins.random_bf16(rng, (B, S, H, D), scale=1 / np.sqrt(D))
    w = (rng.standard_normal((B, S, H)) / np.sqrt(H)).astype(np.float32)
    kc = pins.random_bf16(rng, (B, T, D))
    rb = np.repeat(np.arange(B), S).astype(np.int64)
    rt = np.tile(np.arange(S), B).astype(np.int64)
    o = orc.topk_rows(q.reshape(B * S, H, D), w.reshape(B * S, H), rb, rt, kc, m, k, want_scores=True)
    return q.reshape(B * S, H, D), w.reshape(B * S, H), kc, rb, o


def test_bound_covers_fp32_evaluation():
    """Scores evaluated in fp32 (products, sequential fp32 sums, ReLU, fp32
    head sum) stay within score_error_bound of the fp64 scores."""
    q, w, kc, rb, (o_idx, o_sc, meta, scores) = _case(seed=1, H=64, D=128, S=64, B=1)
    R, H, D = q.shape
    qf = _bits_to_f32(q)
    kf = _bits_to_f32(kc)
    T = kc.shape[1]
    sel = np.tile(np.arange(T), (R, 1))
    bound = checker.score_error_bound(q, w, kc, rb, sel)
    worst = 0.0
    for r in range(R):
        V = int(meta[r, 3])
        for s in range(V):
            acc = np.zeros(H, np.float32)
            for d in range(D):  # sequential fp32 accumulation, one rounding per add
                acc = (acc + qf[r, :, d] * kf[0, s, d]).astype(np.float32)
            x = np.maximum(acc, np.float32(0))
            sc = np.float32(0)
            for h in range(H):
                sc = np.float32(sc + np.float32(w[r, h] * x[h]))
            err = abs(float(sc) - scores[r, s])
            assert err <= bound[r, s], (r, s, err, bound[r, s])
            worst = max(worst, err / bound[r, s])
    assert worst > 0


def _as_gpu(o_idx, o_sc):
    return o_idx.copy(), o_sc.astype(np.float32)


def test_oracle_rows_pass_and_report_counts():
    q, w, kc, rb, (o_idx, o_sc, meta, scores) = _case(seed=2)
    g_idx, g_sc = _as_gpu(o_idx, o_sc)
    bound = checker.score_error_bound(q, w, kc, rb, g_idx)
    rep = checker.check_rows(g_idx, g_sc, o_idx, o_sc, meta, scores, o_idx.shape[1], bound, "oracle as gpu")
    assert rep["recall_min"] == 1.0 and rep["exact_needed"] > 0
    assert rep["scores_compared"] == int((g_idx >= 0).sum())


@pytest.mark.parametrize("mistake", ["wrong_index", "score_off", "order", "padding", "duplicate"])
def test_planted_mistakes_are_rejected(mistake):
    q, w, kc, rb, (o_idx, o_sc, meta, scores) = _case(seed=3)
    k = o_idx.shape[1]
    g_idx, g_sc = _as_gpu(o_idx, o_sc)
    # a row that sees more than k keys with a clear gap at rank k
    rows = [r for r in range(len(meta)) if meta[r, 3] > k + 1 and meta[r, 1] - meta[r, 2] > 0.01 * meta[r, 0]]
    r = rows[len(rows) // 2]
    V = int(meta[r, 3])
    if mistake == "wrong_index":
        outside = [s for s in range(V) if s not in set(o_idx[r].tolist())]
        g_idx[r, k - 1] = outside[0]
        g_sc[r, k - 1] = np.float32(scores[r, outside[0]])
        g_sc[r] = np.sort(g_sc[r])[::-1]
    elif mistake == "score_off":
        g_sc[r, 0] = np.float32(g_sc[r, 0] * (1 + 5e-3))
    elif mistake == "order":
        g_idx[r, [0, 1]] = g_idx[r, [1, 0]]
        g_sc[r, [0, 1]] = g_sc[r, [1, 0]]
    elif mistake == "padding":
        short = [rr for rr in range(len(meta)) if 0 < meta[rr, 3] < k][0]
        g_idx[short, k - 1] = 0
        g_sc[short, k - 1] = np.float32(scores[short, 0])
    elif mistake == "duplicate":
        g_idx[r, 1] = g_idx[r, 0]
        g_sc[r, 1] = g_sc[r, 0]
    bound = checker.score_error_bound(q, w, kc, rb, g_idx)
    with pytest.raises(AssertionError):
        checker.check_rows(g_idx, g_sc, o_idx, o_sc, meta, scores, k, bound, mistake)
