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


def test_attention_bound_covers_kernel_arithmetic():
    """The attention tolerance covers the kernel's arithmetic simulated on the
    CPU: fp32 scores, base-2 softmax with bf16 weights for P.V and an fp32
    sum l, fp32 accumulation, bf16 output.  Rows with few keys (where one
    weight's bf16 rounding dominates) included."""
    import torch
    from oracle import attention as att
    rng = np.random.default_rng(21)
    B, T, H, D, DV = 1, 300, 16, 64, 32
    q = pins.random_bf16(rng, (40, H, D))
    K = pins.random_bf16(rng, (B, T, D))
    V = pins.random_bf16(rng, (B, T, DV))
    scale = 1 / np.sqrt(D)
    idx = np.full((40, 64), -1, np.int32)
    for r in range(40):
        n = 1 + r if r < 30 else 64
        idx[r, :n] = rng.choice(T, n, replace=False)
    rb = np.zeros(40, np.int64)
    ref, lse, absw = att.sparse_attention_rows(q, idx, rb, K, V, scale, want_absw=True)
    tol, tol_lse = checker.attention_tolerance(q, K, rb, idx, scale, absw, ref, lse)
    qf, kf, vf = _bits_to_f32(q), _bits_to_f32(K[0]), _bits_to_f32(V[0])
    c2 = np.float32(scale * np.log2(np.e))
    worst = 0.0
    for r in range(40):
        sel = idx[r][idx[r] >= 0]
        s = (qf[r].astype(np.float32) @ kf[sel].T.astype(np.float32)).astype(np.float32)   # [H, n]
        x = (s * c2).astype(np.float32)
        p = np.exp2(x - x.max(axis=1, keepdims=True)).astype(np.float32)
        l = p.sum(axis=1, dtype=np.float32)
        pb = torch.from_numpy(p).to(torch.bfloat16).float().numpy()
        o = (pb @ vf[sel]).astype(np.float32) / l[:, None]
        ob = torch.from_numpy(o.astype(np.float32)).to(torch.bfloat16).double().numpy()
        err = np.abs(ob - ref[r])
        assert np.all(err <= tol[r]), (r, float((err / tol[r]).max()))
        worst = max(worst, float((err / tol[r]).max()))
    assert worst > 0.05  # the bound is not vacuous
