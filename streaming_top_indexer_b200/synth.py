"""Seeded synthetic inputs for the CSA indexer step.

This module is the one piece shared by the CUDA path's tests/benchmark and
the CPU oracle: it draws q, w and kc with the shapes and value distributions
of the workloads, and it holds none of the indexer's arithmetic (no scores,
no visibility rule, no selection).

Workloads (StreamIndex: Memory-Bounded Compressed Sparse Attention via
Streaming Top-k, Abstract: synthetic V4-shaped inputs, H_I=64 indexer heads,
compression ratio m=4):

  tiny      B=1 S=2048      T=512     H_I=8  d_I=64  k=64
  v4flash   B=1 S=65536     T=16384   H_I=64 d_I=128 k=512
  long      B=1 S=262144    T=65536   H_I=64 d_I=128 k=512   (headline shape)
  extreme   B=1 S=1048576   T=262144  H_I=64 d_I=128 k=512
  tieheavy  B=4 S=131072    T=32768   H_I=64 d_I=128 k=2048  (16-level keys)

q is N(0,1) scaled by 1/sqrt(d_I) in fp32 and then rounded once to bf16
(drawn in fixed blocks of rows, so generation needs no full fp32 copy); kc
is N(0,1) rounded to bf16; w is fp32 N(0,1)/sqrt(H_I).  The tie-heavy
workload draws a 16-row codebook per batch whose entries come from the 16
bf16-exact levels (i-7.5)/4, i=0..15, and copies a uniformly chosen codebook
row into every kc row; its w is uniform in [0,1].  q, w and kc are drawn in
that order from one seeded torch generator on the requested device.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    S: int
    m: int
    H: int
    D: int
    k: int
    kind: str = "normal"  # "normal" | "tieheavy" | "tieheavy_iid"

    @property
    def T(self) -> int:
        return self.S // self.m


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2048, 4, 8, 64, 64),
    "v4flash": Workload("v4flash", 1, 65536, 4, 64, 128, 512),
    "long": Workload("long", 1, 262144, 4, 64, 128, 512),
    "extreme": Workload("extreme", 1, 1048576, 4, 64, 128, 512),
    "tieheavy": Workload("tieheavy", 4, 131072, 4, 64, 128, 2048, "tieheavy"),
    # the literal reading of the tie-heavy keys: i.i.d. entries from the 16 levels
    "tieheavy_iid": Workload("tieheavy_iid", 4, 131072, 4, 64, 128, 2048, "tieheavy_iid"),
}

TIE_LEVELS = [(i - 7.5) / 4.0 for i in range(16)]

# fp32 values of q drawn per block (256 MiB); fixed, so that a seed names the
# same inputs on every run.
Q_BLOCK_ELEMS = 1 << 26


def generate(wl: Workload, seed: int = 0, device="cpu", T: int | None = None):
    """Draw (q bf16 [B,S,H,D], w fp32 [B,S,H], kc bf16 [B,T,D]) for a workload.

    ``T`` overrides S//m (used by tests of ragged key counts).
    """
    T = wl.T if T is None else T
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    # q is drawn in fp32 blocks of at most Q_BLOCK_ELEMS values, each scaled
    # and rounded to bf16 in place, so no full-size fp32 copy ever exists
    # (at S=1,048,576 that copy alone would be 34 GB).
    q = torch.empty((wl.B, wl.S, wl.H, wl.D), dtype=torch.bfloat16, device=dev)
    rows = max(1, Q_BLOCK_ELEMS // (wl.H * wl.D))
    for b in range(wl.B):
        for s0 in range(0, wl.S, rows):
            s1 = min(wl.S, s0 + rows)
            blk = torch.randn((s1 - s0, wl.H, wl.D), generator=g, device=dev, dtype=torch.float32)
            blk.mul_(1.0 / math.sqrt(wl.D))
            q[b, s0:s1].copy_(blk)
            del blk
    if wl.kind.startswith("tieheavy"):
        w = torch.rand((wl.B, wl.S, wl.H), generator=g, device=dev,
                       dtype=torch.float32)
    else:
        w = torch.randn((wl.B, wl.S, wl.H), generator=g, device=dev,
                        dtype=torch.float32)
        w.mul_(1.0 / math.sqrt(wl.H))
    levels = torch.tensor(TIE_LEVELS, dtype=torch.float32, device=dev)
    if wl.kind == "tieheavy":
        book_lv = torch.randint(0, 16, (wl.B, 16, wl.D), generator=g, device=dev)
        book = levels[book_lv]  # [B,16,D]
        pick = torch.randint(0, 16, (wl.B, T), generator=g, device=dev)
        kc = torch.gather(book, 1, pick[:, :, None].expand(wl.B, T, wl.D))
        kc = kc.to(torch.bfloat16)
    elif wl.kind == "tieheavy_iid":
        lv = torch.randint(0, 16, (wl.B, T, wl.D), generator=g, device=dev)
        kc = levels[lv].to(torch.bfloat16)
    else:
        kc = torch.randn((wl.B, T, wl.D), generator=g, device=dev,
                         dtype=torch.float32).to(torch.bfloat16)
    return q, w, kc


def plant_keys(q, w, kc, k: int, seed: int = 0, scale: float = 16.0):
    """Planted-key variant: k keys made dominant for every query that sees them.

    Picks, per batch, a random set P of k keys in [0, T/2) and sets their kc
    rows to ``scale * e_0``; adds 0.5 to coordinate 0 of every q head vector
    and replaces w by |w|.  Every planted key then out-scores every other key
    by a wide margin, and all planted keys of a batch tie exactly with one
    another.  Returns (q, w, kc, planted) with planted int64 [B, k] sorted.
    """
    B, T, D = kc.shape
    if 2 * k > T:
        raise ValueError("plant_keys needs k <= T/2")
    rng = np.random.default_rng(seed + 7919)
    planted = np.stack([np.sort(rng.choice(T // 2, size=k, replace=False))
                        for _ in range(B)]).astype(np.int64)
    q = q.float().clone()
    q[..., 0] += 0.5
    q = q.to(torch.bfloat16)
    w = w.abs()
    kc = kc.clone()
    row = torch.zeros(D, dtype=torch.bfloat16, device=kc.device)
    row[0] = scale
    for b in range(B):
        kc[b, torch.from_numpy(planted[b]).to(kc.device)] = row
    return q, w, kc, planted


def checked_rows(S: int, m: int, k: int, b: int, seed: int = 0, n: int = 512):
    """Query rows the large workloads check: n seeded rows plus edge rows.

    Returns (sampled int64 [n], edges int64 [<=5]); the edge rows
    t in {0, m-1, m*k-2, m*k-1, S-1} are extra and not among the n.
    """
    rng = np.random.default_rng(seed + 1 + b)
    sampled = np.sort(rng.choice(S, size=min(n, S), replace=False)).astype(np.int64)
    edges = sorted({t for t in (0, m - 1, m * k - 2, m * k - 1, S - 1) if 0 <= t < S})
    edges = np.array([t for t in edges if t not in set(sampled.tolist())], np.int64)
    return sampled, edges


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw bf16 bit patterns of a tensor as a host uint16 array."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


ATTN_HEADS = 128


def generate_attention(B: int, S: int, T: int, D: int = 128, DV: int = 128, seed: int = 0, device="cpu"):
    """Draw the sparse attention's inputs: q bf16 [B,S,128,D], kcache bf16
    [B,T,D] and vcache bf16 [B,T,DV], N(0,1) values rounded to bf16 (q drawn
    in fixed row blocks like generate), from one seeded generator."""
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(seed + 7777)
    q = torch.empty((B, S, ATTN_HEADS, D), dtype=torch.bfloat16, device=dev)
    rows = max(1, Q_BLOCK_ELEMS // (ATTN_HEADS * D))
    for b in range(B):
        for s0 in range(0, S, rows):
            s1 = min(S, s0 + rows)
            q[b, s0:s1].copy_(torch.randn((s1 - s0, ATTN_HEADS, D), generator=g, device=dev, dtype=torch.float32))
    kc = torch.randn((B, T, D), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    vc = torch.randn((B, T, DV), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    return q, kc, vc


def generate_hidden(B: int, S: int, d_model: int, H: int, D: int, m: int, seed: int = 0, device="cpu"):
    """Draw hidden states and random producer weights (no trained weights exist):
    x bf16 [B,S,d_model] ~ N(0,1); W_q bf16 [H*D, d_model] ~ N(0, 1/(d_model*D)),
    W_w bf16 [H, d_model] ~ N(0, 1/(d_model*H)), W_k bf16 [D, d_model]
    ~ N(0, m/d_model), so that the projected q, w and kc have the spreads of
    generate()'s inputs (N(0,1/D), N(0,1/H), N(0,1))."""
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(seed + 31337)
    x = torch.empty((B, S, d_model), dtype=torch.bfloat16, device=dev)
    rows = max(1, Q_BLOCK_ELEMS // d_model)
    for b in range(B):
        for s0 in range(0, S, rows):
            s1 = min(S, s0 + rows)
            x[b, s0:s1].copy_(torch.randn((s1 - s0, d_model), generator=g, device=dev, dtype=torch.float32))

    def weight(rows_, std):
        return (torch.randn((rows_, d_model), generator=g, device=dev, dtype=torch.float32) * std).to(torch.bfloat16)

    w_q = weight(H * D, 1.0 / math.sqrt(d_model * D))
    w_w = weight(H, 1.0 / math.sqrt(d_model * H))
    w_k = weight(D, math.sqrt(m / d_model))
    return x, w_q, w_w, w_k
