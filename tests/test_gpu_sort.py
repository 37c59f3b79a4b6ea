"""The row sort (si_sort_topk) on long rows against an independent order
(needs a B200).

Each row is ordered by score descending, then key index ascending, with
padding (-1, -inf) last.  The expected order is computed on the host from
64-bit keys, (order-preserving map of the fp32 score) << 32 | (2^32 - 1 -
index), sorted descending with numpy, which is that order exactly.
"""
import numpy as np
import pytest
import torch

import streaming_top_indexer_b200 as si

pytestmark = pytest.mark.gpu

DEV = "cuda"


def host_keys(idx, score):
    u = (score.astype(np.float32) + np.float32(0.0)).view(np.uint32).astype(np.uint64)  # -0.0 -> +0.0
    neg = (u >> np.uint64(31)) & np.uint64(1)
    ordv = np.where(neg == 1, (~u) & np.uint64(0xFFFFFFFF), u | np.uint64(0x80000000))
    low = (~idx.astype(np.int64).astype(np.uint64)) & np.uint64(0xFFFFFFFF)
    return (ordv << np.uint64(32)) | low


def expected_rows(idx, score):
    keys = host_keys(idx, score)
    order = np.argsort(keys, axis=1, kind="stable")[:, ::-1]
    return np.take_along_axis(idx, order, 1), np.take_along_axis(score, order, 1)


def random_rows(rows, k, seed, ties):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.choice(1 << 20, size=k, replace=False) for _ in range(rows)]).astype(np.int32)
    if ties:
        score = rng.integers(-8, 8, size=(rows, k)).astype(np.float32) / 4  # 16 levels: many equal scores
    else:
        score = rng.standard_normal((rows, k)).astype(np.float32)
    # padding entries (index -1, score -inf) at random places in some rows
    pad = rng.random((rows, k)) < np.where(np.arange(rows)[:, None] % 3 == 0, 0.3, 0.0)
    idx[pad] = -1
    score[pad] = -np.inf
    score[0, :5] = 0.0
    score[0, 5:10] = -0.0  # both zeros pack alike
    return idx, score


@pytest.mark.parametrize("k", [1025, 1500, 2047, 2048])
@pytest.mark.parametrize("ties", [False, True])
def test_long_row_sort_equals_host_order(k, ties):
    rows = 1537
    idx, score = random_rows(rows, k, seed=k + (7 if ties else 0), ties=ties)
    ti = torch.from_numpy(idx).to(DEV)[None]  # [1, rows, k]
    ts = torch.from_numpy(score).to(DEV)[None]
    si.sort_topk(ti, ts)
    torch.cuda.synchronize()
    want_i, want_s = expected_rows(idx, score)
    got_i, got_s = ti[0].cpu().numpy(), ts[0].cpu().numpy()
    assert np.array_equal(got_i, want_i)
    # scores as bits, except that -0.0 comes back as +0.0 (the two are one key)
    assert np.array_equal((got_s + np.float32(0.0)).view(np.uint32), (want_s + np.float32(0.0)).view(np.uint32))


def test_long_row_sort_misaligned_rows():
    """k = 1027: rows start at 4-byte but not 16-byte boundaries (the scalar
    load and store path)."""
    idx, score = random_rows(64, 1027, seed=3, ties=True)
    ti = torch.from_numpy(idx).to(DEV)[None]  # [1, rows, k]
    ts = torch.from_numpy(score).to(DEV)[None]
    si.sort_topk(ti, ts)
    torch.cuda.synchronize()
    want_i, _ = expected_rows(idx, score)
    assert np.array_equal(ti[0].cpu().numpy(), want_i)
