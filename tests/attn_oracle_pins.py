"""Pins of the sparse-attention oracle to facts other than its own code.

Each ``pin_*`` runs the oracle library ``lib`` (the real one, or a broken
copy in the mutation test) on inputs whose answer is fixed by hand
computation, a closed form, a library routine on a special case, or an
invariance of the definition, and raises AssertionError on a mismatch.  The
definition pinned is CSA's sparse attention stage (StreamIndex:
Memory-Bounded Compressed Sparse Attention via Streaming Top-k, Abstract)
with this library's reading: per-head softmax over the selected shared
key/value entries, padding (< 0) skipped, an empty row giving 0 and -inf.
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch

from oracle import attention as att
from tests import oracle_pins as ipins

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _f64(bits):
    return ipins.bits_to_f64(bits)


def pin_hand_case(lib):
    """tests/golden/attn_hand_case_1.json: outputs, log-sum-exp and the
    |V|-weighted sums, evaluated from closed forms."""
    with open(os.path.join(GOLDEN, "attn_hand_case_1.json")) as f:
        c = json.load(f)
    B, T, H, D, DV = c["B"], c["T"], c["H"], c["D"], c["DV"]
    R = len(c["q"])
    q = ipins.f32_to_bf16_bits(c["q"]).reshape(R, H, D)
    idx = np.asarray(c["idx"], np.int32)
    K = ipins.f32_to_bf16_bits(c["K"]).reshape(B, T, D)
    V = ipins.f32_to_bf16_bits(c["V"]).reshape(B, T, DV)
    out, lse, absw = att.sparse_attention_rows(q, idx, np.zeros(R, np.int64), K, V, c["scale"], True, lib=lib)
    e_out = np.asarray(c["expect_out"], np.float64)
    e_lse = np.asarray([[float(x) for x in row] for row in c["expect_lse"]])
    e_abs = np.asarray(c["expect_absw"], np.float64)
    assert np.allclose(out, e_out, rtol=1e-13, atol=1e-13), f"out {out.tolist()}"
    assert np.array_equal(np.isneginf(lse), np.isneginf(e_lse)), f"lse {lse.tolist()}"
    fin = np.isfinite(e_lse)
    assert np.allclose(lse[fin], e_lse[fin], rtol=1e-13, atol=1e-13), f"lse {lse.tolist()}"
    assert np.allclose(absw, e_abs, rtol=1e-13, atol=1e-13), f"absw {absw.tolist()}"


def pin_uniform_scores(lib, seed=11):
    """Identical K rows: every selected key scores the same, so the output is
    the plain mean of the selected V rows and lse = s + ln(n)."""
    rng = np.random.default_rng(seed)
    B, T, H, D, DV, k = 2, 20, 3, 8, 6, 7
    krow = ipins.random_bf16(rng, (D,))
    K = np.broadcast_to(krow, (B, T, D)).copy()
    V = ipins.random_bf16(rng, (B, T, DV))
    R = 6
    q = ipins.random_bf16(rng, (R, H, D))
    rb = rng.integers(0, B, R).astype(np.int64)
    idx = np.stack([rng.choice(T, k, replace=False) for _ in range(R)]).astype(np.int32)
    idx[1, 3:] = -1
    out, lse, _ = att.sparse_attention_rows(q, idx, rb, K, V, 0.25, lib=lib)
    for r in range(R):
        sel = idx[r][idx[r] >= 0]
        mean = _f64(V[rb[r], sel]).mean(axis=0)
        s = 0.25 * (_f64(q[r]) @ _f64(krow))
        for h in range(H):
            assert np.allclose(out[r, h], mean, rtol=1e-12, atol=1e-12), f"uniform r={r} h={h}"
            assert np.isclose(lse[r, h], s[h] + np.log(len(sel)), rtol=1e-12, atol=1e-12)


def pin_dense_causal_sdpa(lib, seed=12):
    """Selecting every key a row can see ((s+1)*m <= t+1) is dense causal
    attention over the compressed keys: torch's scaled_dot_product_attention
    in fp64 with that boolean mask gives the same output."""
    rng = np.random.default_rng(seed)
    B, S, m, H, D, DV = 2, 24, 3, 4, 8, 5
    T = S // m
    q = ipins.random_bf16(rng, (B, S, H, D), scale=0.5)
    K = ipins.random_bf16(rng, (B, T, D))
    V = ipins.random_bf16(rng, (B, T, DV))
    scale = 1 / np.sqrt(D)
    vis = ((np.arange(T)[None, :] + 1) * m <= np.arange(S)[:, None] + 1)  # [S, T]
    idx = np.where(vis, np.arange(T)[None, :], -1).astype(np.int32)       # every visible key, k = T
    rows_b = np.repeat(np.arange(B), S).astype(np.int64)
    out, lse, _ = att.sparse_attention_rows(q.reshape(B * S, H, D), np.tile(idx, (B, 1)), rows_b, K, V, scale,
                                            lib=lib)
    qt = torch.from_numpy(_f64(q)).permute(0, 2, 1, 3)                    # [B,H,S,D]
    kt = torch.from_numpy(_f64(K))[:, None].expand(B, H, T, D)
    vt = torch.from_numpy(_f64(V))[:, None].expand(B, H, T, DV)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=torch.from_numpy(vis), scale=scale)
    ref = ref.permute(0, 2, 1, 3).reshape(B * S, H, DV).numpy()
    has = np.tile(vis.any(axis=1), B)
    assert np.allclose(out[has], ref[has], rtol=1e-10, atol=1e-12), "dense causal special case"
    assert np.all(out[~has] == 0) and np.all(np.isneginf(lse[~has]))


def pin_dominant_key(lib, seed=13):
    """One selected key whose score exceeds every other by g: the output is
    that key's V row within exp(-g) * (sum of the others' |V|)."""
    rng = np.random.default_rng(seed)
    B, T, H, D, DV, k = 1, 16, 2, 4, 3, 6
    K = ipins.random_bf16(rng, (B, T, D), scale=0.1)
    V = ipins.random_bf16(rng, (B, T, DV))
    K[0, 5] = ipins.f32_to_bf16_bits([8.0, 0, 0, 0])
    q = ipins.f32_to_bf16_bits(np.tile(np.array([4.0, 0, 0, 0], np.float32), (1, H, 1)))  # [1,H,D]
    idx = np.array([[3, 5, 9, 11, 0, 14]], np.int32)
    out, _, _ = att.sparse_attention_rows(q, idx, np.zeros(1, np.int64), K, V, 1.0, lib=lib)
    s = _f64(q[0]) @ _f64(K[0, idx[0]]).T
    gap = s[:, 1] - np.delete(s, 1, axis=1).max(axis=1)
    bound = np.exp(-gap)[:, None] * 2 * np.abs(_f64(V[0])).sum(axis=0).max()
    assert np.all(gap > 20)
    assert np.all(np.abs(out[0] - _f64(V[0, 5])) <= bound)


def pin_permutation_and_padding(lib, seed=14):
    """The output does not depend on the order of the selected indices, and
    padding entries (-1) anywhere in the row are skipped."""
    rng = np.random.default_rng(seed)
    B, T, H, D, DV, k = 2, 40, 3, 8, 8, 10
    K = ipins.random_bf16(rng, (B, T, D))
    V = ipins.random_bf16(rng, (B, T, DV))
    R = 5
    q = ipins.random_bf16(rng, (R, H, D), scale=0.4)
    rb = np.array([0, 1, 1, 0, 1], np.int64)
    idx = np.stack([rng.choice(T, k, replace=False) for _ in range(R)]).astype(np.int32)
    out, lse, _ = att.sparse_attention_rows(q, idx, rb, K, V, 0.3, lib=lib)
    perm = np.stack([rng.permutation(row) for row in idx])
    padded = np.full((R, k + 6), -1, np.int32)
    for r in range(R):
        pos = np.sort(rng.choice(k + 6, k, replace=False))
        padded[r, pos] = perm[r]
    out2, lse2, _ = att.sparse_attention_rows(q, padded, rb, K, V, 0.3, lib=lib)
    assert np.allclose(out, out2, rtol=1e-12, atol=1e-12)
    assert np.allclose(lse, lse2, rtol=1e-12, atol=1e-12)


ALL_PINS = [pin_hand_case, pin_uniform_scores, pin_dense_causal_sdpa, pin_dominant_key, pin_permutation_and_padding]
