"""Pins of the producers' oracle (oracle/producers.py) to facts other than its
own code: brute force on tiny inputs, one-hot inputs that select weight
columns, the mean of identical tokens, and linearity."""
import numpy as np

from oracle import producers as pr
from tests import oracle_pins as pins


def test_brute_force_tiny():
    """A 3-token, 4-wide projection and a 2:1 compression written out by hand
    loops (sums of products over the input width)."""
    rng = np.random.default_rng(1)
    x = pins.random_bf16(rng, (1, 4, 5))
    wq = pins.random_bf16(rng, (3, 5))
    wk = pins.random_bf16(rng, (2, 5))
    xf, wqf, wkf = pins.bits_to_f64(x), pins.bits_to_f64(wq), pins.bits_to_f64(wk)
    q = pr.project(x, wq)
    for t in range(4):
        for o in range(3):
            assert abs(q[0, t, o] - sum(xf[0, t, i] * wqf[o, i] for i in range(5))) < 1e-12
    kc = pr.compress_keys(x, wk, 2)
    assert kc.shape == (1, 2, 2)
    for s in range(2):
        for o in range(2):
            want = sum((xf[0, 2 * s, i] + xf[0, 2 * s + 1, i]) / 2 * wkf[o, i] for i in range(5))
            assert abs(kc[0, s, o] - want) < 1e-12


def test_one_hot_tokens_select_weight_columns():
    """x = e_i gives column i of W (the [out, in] layout, not its transpose)."""
    rng = np.random.default_rng(2)
    Din, Dout = 16, 6
    w = pins.random_bf16(rng, (Dout, Din))
    eye = pins.f32_to_bf16_bits(np.eye(Din, dtype=np.float32))
    got = pr.project(eye, w)
    assert np.array_equal(got, pins.bits_to_f64(w).T)


def test_compression_of_identical_tokens_and_ragged_tail():
    """m identical tokens compress to the projection of that token; tokens
    past T*m are not covered; the ratio m=1 is the plain projection."""
    rng = np.random.default_rng(3)
    B, T, m, Din, d = 2, 5, 4, 8, 3
    tok = pins.random_bf16(rng, (B, T, 1, Din))
    x = np.repeat(tok, m, axis=2).reshape(B, T * m, Din)
    x = np.concatenate([x, pins.random_bf16(rng, (B, 3, Din), scale=100.0)], axis=1)  # ragged tail
    wk = pins.random_bf16(rng, (d, Din))
    kc = pr.compress_keys(x, wk, m)
    assert kc.shape == (B, T, d)
    assert np.allclose(kc, pr.project(tok[:, :, 0], wk), rtol=1e-13, atol=1e-13)
    assert np.allclose(pr.compress_keys(x, wk, 1), pr.project(x, wk), rtol=1e-13, atol=1e-13)


def test_linearity():
    """Projection of a token sum is the sum of projections (exact bf16 sums
    of small integers)."""
    rng = np.random.default_rng(4)
    a = rng.integers(-4, 5, (6, 10)).astype(np.float32)
    b = rng.integers(-4, 5, (6, 10)).astype(np.float32)
    w = pins.random_bf16(rng, (7, 10))
    pa, pb = pr.project(pins.f32_to_bf16_bits(a), w), pr.project(pins.f32_to_bf16_bits(b), w)
    pab = pr.project(pins.f32_to_bf16_bits(a + b), w)
    assert np.allclose(pab, pa + pb, rtol=1e-13, atol=1e-12)
