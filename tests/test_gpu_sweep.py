"""Design-space sweeps with recall against the oracle (needs a B200).

The pages sweep three parameters of their driver over five points each --
chunk size, key-tile size and top-k -- and report mean recall rounding to
1.0000 and min recall >= 0.9980 in every cell (StreamIndex: Memory-Bounded
Compressed Sparse Attention via Streaming Top-k, Abstract).  This design's
counterparts (si_set_tuning):
  pool capacity P   candidates a query holds before a partition-merge (the
                    chunk of scores merged at once);
  check interval    128-key tiles streamed between two checks of the pools
                    (the key tiles a merge decision covers);
  cut slack         entries above k an intermediate merge keeps;
and k itself.  Each cell runs the full V4-Flash-like shape (S = 65,536,
T = 16,384, H_I = 64, d_I = 128) and checks 512 seeded rows plus edge rows
against the fp64 oracle with the acceptance rules of tests/checker.py.  With
$SI_SWEEP_OUT set, the cells are also written there as JSON lines.
"""
import json
import os

import numpy as np
import pytest
import torch

import streaming_top_indexer_b200 as si
from streaming_top_indexer_b200 import synth
from tests import checker
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu

DEV = "cuda"

SWEEPS = {
    "k": [("k", v) for v in (128, 256, 512, 1024, 2048)],
    "pool": [("pool_entries", v) for v in (800, 1056, 1344, 1600, 1856)],
    "check": [("check_tiles", v) for v in (1, 2, 3, 4, 6)],
    "slack": [("cut_slack", v) for v in (32, 64, 128, 256, 512)],
}


@pytest.fixture(scope="module")
def inputs():
    wl = synth.WORKLOADS["v4flash"]
    q, w, kc = synth.generate(wl, seed=0, device=DEV)
    b_rows, t_rows = gh.sampled_rows(wl.B, wl.S, wl.m, 2048)
    return wl, q, w, kc, b_rows, t_rows


_oracle_cache = {}


def _oracle(wl, q, w, kc, b_rows, t_rows, k):
    if k not in _oracle_cache:
        _oracle_cache[k] = gh.oracle_rows(q, w, kc, wl.m, k, b_rows, t_rows)
    return _oracle_cache[k]


@pytest.mark.parametrize("sweep", sorted(SWEEPS))
def test_design_sweep_recall_against_oracle(inputs, sweep):
    wl, q, w, kc, b_rows, t_rows = inputs
    out = os.environ.get("SI_SWEEP_OUT")
    cells = []
    try:
        for name, value in SWEEPS[sweep]:
            k = value if name == "k" else wl.k
            si.set_tuning(**({} if name == "k" else {name: value}))
            ws = torch.zeros(si.workspace_bytes(wl.B, wl.S, wl.T, wl.H, wl.D, wl.m, k), dtype=torch.uint8,
                             device=DEV)
            idx, sc = si.indexer_topk(q, w, kc, wl.m, k, workspace=ws)
            assert si.check_device_status(ws) == 0
            bt = torch.from_numpy(b_rows).to(DEV)
            tt = torch.from_numpy(t_rows).to(DEV)
            gi = idx[bt, tt].cpu().numpy()
            gs = sc[bt, tt].cpu().numpy()
            o_idx, o_sc, o_meta, o_scores = _oracle(wl, q, w, kc, b_rows, t_rows, k)
            bound = checker.score_error_bound(synth.bf16_bits(q[bt, tt]), w[bt, tt].cpu().numpy(),
                                              synth.bf16_bits(kc), b_rows, gi)
            rep = checker.check_rows(gi, gs, o_idx, o_sc, o_meta, o_scores, k, bound, f"{sweep} {name}={value}")
            cell = {"sweep": sweep, "parameter": name, "value": value, "k": k, "rows": int(rep["rows"]),
                    "recall_mean": rep["recall_mean"], "recall_min": rep["recall_min"],
                    "exact_rows": rep["exact_rows"], "exact_needed": rep["exact_needed"],
                    "max_rel_err": rep["max_rel_err"]}
            cells.append(cell)
            assert rep["recall_mean"] >= 0.9995 and rep["recall_min"] >= 0.998
    finally:
        si.set_tuning()
    if out:
        with open(out, "a") as f:
            for c in cells:
                f.write(json.dumps(c) + "\n")
    assert len(cells) == 5
