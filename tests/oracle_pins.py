"""Pins of the CPU oracle to facts other than its own code.

Each ``pin_*`` function runs the oracle library ``lib`` (the real one, or a
deliberately broken copy in the mutation test) on inputs whose answer is
fixed by hand computation, a closed form, a library routine on a special
case, or a structural property of the definition, and raises AssertionError
on a mismatch.  The definition pinned is the CSA indexer step (StreamIndex:
Memory-Bounded Compressed Sparse Attention via Streaming Top-k, Abstract)
with this library's score rule sum_h w*ReLU(q.kc), visibility
(s+1)*m <= t+1, ties to the lower index and -1/-inf padding.
"""
from __future__ import annotations

import json
import os

import numpy as np

from oracle import oracle as orc

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def f32_to_bf16_bits(x) -> np.ndarray:
    """Exact bf16 bits of values that are representable in bf16."""
    u = np.asarray(x, np.float32).view(np.uint32)
    if np.any(u & 0xFFFF):
        raise ValueError("value not exactly representable in bf16")
    return (u >> 16).astype(np.uint16)


def random_bf16(rng, shape, scale=1.0, nonneg=False):
    """bf16 bit patterns of N(0, scale^2) values (rounded by truncation)."""
    x = rng.standard_normal(shape).astype(np.float32) * np.float32(scale)
    if nonneg:
        x = np.abs(x)
    u = x.view(np.uint32) & np.uint32(0xFFFF0000)
    return (u >> 16).astype(np.uint16)


def bits_to_f64(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def run_all(lib, q_bits, w, kc_bits, m, k, want_scores=False):
    return orc.topk_all_rows(q_bits, w, kc_bits, m, k, want_scores, lib=lib)


def visible_count(t, T, m):
    """Closed form of the number of keys row t sees: min(T, floor((t+1)/m))."""
    return np.minimum(T, (np.asarray(t) + 1) // m)


def check_invariants(idx, score, nvis, k):
    """Output invariants of a top-k row set (any implementation)."""
    R = idx.shape[0]
    for r in range(R):
        n = int(min(k, nvis[r]))
        row_i, row_s = idx[r], score[r]
        assert np.all(row_i[n:] == -1), f"row {r}: padding index"
        assert np.all(np.isneginf(row_s[n:])), f"row {r}: padding score"
        sel = row_i[:n]
        assert np.all((sel >= 0) & (sel < nvis[r])), f"row {r}: index not visible"
        assert len(set(sel.tolist())) == n, f"row {r}: duplicate index"
        s = row_s[:n]
        assert np.all(np.isfinite(s)), f"row {r}: non-finite score"
        assert np.all(s[:-1] >= s[1:]), f"row {r}: scores increase"
        eq = s[:-1] == s[1:]
        assert np.all(sel[:-1][eq] < sel[1:][eq]), f"row {r}: tie order"


# --------------------------------------------------------------------------
# Pins
# --------------------------------------------------------------------------

def pin_hand_cases(lib):
    """Hand-computed fixtures under tests/golden/: indices, scores and the
    per-row meta (max |score| over the visible keys, the scores at ranks k
    and k+1, the visible count) that the acceptance rule's tie band and
    score tolerance are built on."""
    for name in sorted(os.listdir(GOLDEN)):
        if not name.startswith("hand_case_"):
            continue
        with open(os.path.join(GOLDEN, name)) as f:
            case = json.load(f)
        B, S, T, m, H, D, k = (case[x] for x in "B S T m H D k".split())
        q = f32_to_bf16_bits(case["q"]).reshape(B, S, H, D)
        w = np.asarray(case["w"], np.float32).reshape(B, S, H)
        kc = f32_to_bf16_bits(case["kc"]).reshape(B, T, D)
        idx, sc, meta, _ = run_all(lib, q, w, kc, m, k)
        e_idx = np.asarray(case["expect_idx"], np.int32).reshape(B, S, k)
        e_sc = np.asarray([[float(v) for v in row] for row in case["expect_score"]]).reshape(B, S, k)
        assert np.array_equal(idx, e_idx), f"{name}: idx {idx.tolist()} != {e_idx.tolist()}"
        assert np.array_equal(sc, e_sc), f"{name}: score {sc.tolist()} != {e_sc.tolist()}"
        e_meta = np.asarray([[float(v) for v in row] for row in case["expect_meta"]]).reshape(B, S, 4)
        assert np.array_equal(meta, e_meta, equal_nan=True), f"{name}: meta {meta.tolist()} != {e_meta.tolist()}"


def pin_matmul_special_case(lib, seed=1):
    """H=1, w=1, non-negative q and kc: the indexer reduces to the causal top-k
    of the matrix product Q Kc^T, computed here with numpy matmul and a stable
    argsort (equal scores keep ascending index)."""
    rng = np.random.default_rng(seed)
    for (B, S, m, D, k) in [(2, 64, 4, 8, 5), (1, 40, 2, 16, 12), (1, 33, 1, 4, 40)]:
        T = S // m
        q = random_bf16(rng, (B, S, 1, D), nonneg=True)
        kc = random_bf16(rng, (B, T, D), nonneg=True)
        w = np.ones((B, S, 1), np.float32)
        idx, sc, meta, _ = run_all(lib, q, w, kc, m, k)
        prod = np.einsum("bsd,btd->bst", bits_to_f64(q[:, :, 0, :]), bits_to_f64(kc))
        for b in range(B):
            for t in range(S):
                v = int(visible_count(t, T, m))
                row = prod[b, t, :v]
                order = np.argsort(-row, kind="stable")[:k]
                n = len(order)
                assert np.array_equal(idx[b, t, :n], order), f"matmul case b={b} t={t}"
                assert np.allclose(sc[b, t, :n], row[order], rtol=1e-12, atol=0)
                assert np.all(idx[b, t, n:] == -1)


def pin_relu_head_sum_closed_form(lib, seed=2):
    """Heads that are scaled copies of one vector v, q_h = c_h v: with
    y_s = v.kc_s the score is max(y,0)*sum_{c_h>0} w_h c_h
    + min(y,0)*sum_{c_h<0} w_h c_h (ReLU per head, w after ReLU)."""
    rng = np.random.default_rng(seed)
    B, S, m, D, k = 1, 48, 3, 8, 6
    T = S // m
    c = np.array([1.0, -1.0, 2.0, -0.5, 0.5, -2.0], np.float32)
    H = len(c)
    v = bits_to_f64(random_bf16(rng, (B, S, D))).astype(np.float32)
    q = f32_to_bf16_bits(v[:, :, None, :] * c[None, None, :, None])
    w = rng.uniform(-1, 1, (B, S, H)).astype(np.float32)
    kc = random_bf16(rng, (B, T, D))
    _, _, _, scores = run_all(lib, q, w, kc, m, k, want_scores=True)
    y = np.einsum("bsd,btd->bst", v.astype(np.float64), bits_to_f64(kc))
    wd = w.astype(np.float64)
    cd = c.astype(np.float64)
    A = (wd * np.where(cd > 0, cd, 0.0)).sum(-1)[..., None]
    C = (wd * np.where(cd < 0, cd, 0.0)).sum(-1)[..., None]
    expect = np.maximum(y, 0.0) * A + np.minimum(y, 0.0) * C
    for t in range(S):
        nv = int(visible_count(t, T, m))
        got = scores[0, t, :nv]
        assert np.allclose(got, expect[0, t, :nv], rtol=1e-12, atol=1e-12), f"closed form t={t}"
        assert np.all(np.isnan(scores[0, t, nv:])), "invisible key scored"


def pin_visible_count(lib):
    """Number of returned keys = min(k, min(T, floor((t+1)/m))), for T both
    below and above S/m."""
    rng = np.random.default_rng(3)
    for (S, T, m, k) in [(37, 9, 4, 3), (37, 20, 4, 30), (16, 16, 1, 7), (50, 5, 7, 2), (12, 40, 2, 64)]:
        q = random_bf16(rng, (1, S, 2, 4))
        w = rng.standard_normal((1, S, 2)).astype(np.float32)
        kc = random_bf16(rng, (1, T, 4))
        idx, _, meta, _ = run_all(lib, q, w, kc, m, k)
        nv = visible_count(np.arange(S), T, m)
        assert np.array_equal(meta[0, :, 3].astype(np.int64), nv), "visible count"
        got_n = (idx[0] >= 0).sum(-1)
        assert np.array_equal(got_n, np.minimum(k, nv)), "returned count"
        # with k >= T every visible key comes back
        if k >= T:
            for t in range(S):
                assert sorted(idx[0, t, : nv[t]].tolist()) == list(range(nv[t]))


def pin_all_tied(lib):
    """All kc rows identical: every visible key has the same score, so the
    top-k is keys 0..k-1 in ascending order."""
    rng = np.random.default_rng(4)
    S, m, k, D, H = 40, 2, 7, 4, 3
    T = S // m
    row = random_bf16(rng, (D,))
    kc = np.broadcast_to(row, (1, T, D)).copy()
    q = random_bf16(rng, (1, S, H, D))
    w = rng.standard_normal((1, S, H)).astype(np.float32)
    idx, sc, _, _ = run_all(lib, q, w, kc, m, k)
    for t in range(S):
        n = int(min(k, visible_count(t, T, m)))
        assert idx[0, t, :n].tolist() == list(range(n)), f"tie order t={t}"
        assert np.all(sc[0, t, :n] == sc[0, t, 0])


def pin_planted(lib):
    """Planted dominant keys: rows that see all of them return exactly them
    (tied, so in ascending index order); other rows contain every planted
    key they can see."""
    rng = np.random.default_rng(5)
    B, S, m, H, D, k = 2, 96, 4, 4, 8, 5
    T = S // m
    q = bits_to_f64(random_bf16(rng, (B, S, H, D), scale=1 / np.sqrt(D))).astype(np.float32)
    q[..., 0] += 0.5
    q = (q.view(np.uint32) >> 16).astype(np.uint16)  # truncate to bf16
    w = np.abs(rng.standard_normal((B, S, H))).astype(np.float32)
    kc = random_bf16(rng, (B, T, D))
    planted = [np.sort(rng.choice(T // 2, size=k, replace=False)) for _ in range(B)]
    for b in range(B):
        kc[b, planted[b]] = 0
        kc[b, planted[b], 0] = f32_to_bf16_bits([16.0])[0]
    idx, _, _, _ = run_all(lib, q, w, kc, m, k)
    for b in range(B):
        for t in range(S):
            nv = int(visible_count(t, T, m))
            vis_p = [p for p in planted[b].tolist() if p < nv]
            if nv >= T // 2:
                assert idx[b, t].tolist() == planted[b].tolist(), f"planted b={b} t={t}"
            else:
                assert set(vis_p) <= set(idx[b, t].tolist())


def pin_scaling_and_causality(lib):
    """Doubling w, q or kc doubles every score (exact in binary floating
    point) and keeps the indices; changing keys a row cannot see, or adding
    keys past T, leaves that row unchanged."""
    rng = np.random.default_rng(6)
    B, S, m, H, D, k = 1, 32, 2, 3, 4, 4
    T = S // m
    q = random_bf16(rng, (B, S, H, D))
    w = rng.standard_normal((B, S, H)).astype(np.float32)
    kc = random_bf16(rng, (B, T, D))
    idx0, sc0, _, _ = run_all(lib, q, w, kc, m, k)
    dbl = lambda bits: f32_to_bf16_bits(bits_to_f64(bits).astype(np.float32) * 2)
    for (qq, ww, kk) in [(q, w * 2, kc), (dbl(q), w, kc), (q, w, dbl(kc))]:
        idx1, sc1, _, _ = run_all(lib, qq, ww, kk, m, k)
        assert np.array_equal(idx1, idx0), "scaling changed indices"
        fin = np.isfinite(sc0)
        assert np.array_equal(sc1[fin], 2 * sc0[fin]), "scaling law"
    t = 13
    nv = int(visible_count(t, T, m))
    kc2 = kc.copy()
    kc2[:, nv:] = random_bf16(rng, (B, T - nv, D), scale=50.0)
    idx2, sc2, _, _ = run_all(lib, q, w, kc2, m, k)
    assert np.array_equal(idx2[0, t], idx0[0, t]) and np.array_equal(sc2[0, t], sc0[0, t])
    kc3 = np.concatenate([kc, random_bf16(rng, (B, 8, D), scale=50.0)], axis=1)
    idx3, sc3, _, _ = run_all(lib, q, w, kc3, m, k)
    for tt in range(S):
        if visible_count(tt, T, m) < T:
            assert np.array_equal(idx3[0, tt], idx0[0, tt]), "keys past T leaked"


def pin_invariants_random(lib):
    """Output invariants on random inputs, including k larger than T."""
    rng = np.random.default_rng(7)
    for (B, S, m, H, D, k) in [(2, 64, 4, 8, 16, 6), (1, 30, 1, 2, 8, 40), (1, 70, 3, 4, 4, 9)]:
        T = S // m
        q = random_bf16(rng, (B, S, H, D))
        w = rng.standard_normal((B, S, H)).astype(np.float32)
        kc = random_bf16(rng, (B, T, D))
        idx, sc, meta, _ = run_all(lib, q, w, kc, m, k)
        check_invariants(idx.reshape(-1, k), sc.reshape(-1, k), meta.reshape(-1, 4)[:, 3], k)


ALL_PINS = [pin_hand_cases, pin_matmul_special_case, pin_relu_head_sum_closed_form,
            pin_visible_count, pin_all_tied, pin_planted, pin_scaling_and_causality,
            pin_invariants_random]
