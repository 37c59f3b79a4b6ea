"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
binding and the CPU oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

import streaming_top_indexer_b200 as si
from oracle import oracle as orc
from streaming_top_indexer_b200 import synth
from tests import checker


def gpu_topk(q, w, kc, m, k):
    """si_indexer_topk on device tensors; returns host (idx, score)."""
    B, S, H, D = q.shape
    T = kc.shape[1]
    ws = torch.zeros(si.workspace_bytes(B, S, T, H, D, m, k), dtype=torch.uint8, device=q.device)
    idx, sc = si.indexer_topk(q, w, kc, m, k, workspace=ws)
    status = si.check_device_status(ws)
    assert status == 0, f"device status {status}"
    return idx, sc


def oracle_rows(q, w, kc, m, k, b_rows, t_rows):
    """Oracle top-k (with all scores) of the given (b, t) rows."""
    b_rows = np.asarray(b_rows, np.int64)
    t_rows = np.asarray(t_rows, np.int64)
    bt = torch.from_numpy(b_rows).to(q.device)
    tt = torch.from_numpy(t_rows).to(q.device)
    q_rows = synth.bf16_bits(q[bt, tt])
    w_rows = w[bt, tt].cpu().numpy()
    kc_bits = synth.bf16_bits(kc)
    return orc.topk_rows(q_rows, w_rows, b_rows, t_rows, kc_bits, m, k, want_scores=True)


def check_against_oracle(q, w, kc, m, k, b_rows, t_rows, g_idx=None, g_score=None, where=""):
    if g_idx is None:
        g_idx, g_score = gpu_topk(q, w, kc, m, k)
    b_rows = np.asarray(b_rows, np.int64)
    t_rows = np.asarray(t_rows, np.int64)
    bt = torch.from_numpy(b_rows).to(g_idx.device)
    tt = torch.from_numpy(t_rows).to(g_idx.device)
    gi = g_idx[bt, tt].cpu().numpy()
    gs = g_score[bt, tt].cpu().numpy()
    o_idx, o_score, o_meta, o_scores = oracle_rows(q, w, kc, m, k, b_rows, t_rows)
    bound = checker.score_error_bound(synth.bf16_bits(q[bt.to(q.device), tt.to(q.device)]),
                                      w[bt.to(w.device), tt.to(w.device)].cpu().numpy(), synth.bf16_bits(kc),
                                      b_rows, gi)
    return checker.check_rows(gi, gs, o_idx, o_score, o_meta, o_scores, k, bound, where)


def all_rows(B, S):
    return np.repeat(np.arange(B), S), np.tile(np.arange(S), B)


def sampled_rows(B, S, m, k, seed=0, n=512):
    bs, ts = [], []
    for b in range(B):
        samp, edges = synth.checked_rows(S, m, k, b, seed, n)
        t = np.concatenate([samp, edges])
        bs.append(np.full(t.shape, b))
        ts.append(t)
    return np.concatenate(bs), np.concatenate(ts)
