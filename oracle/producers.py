"""Plain fp64 CPU oracle of the CSA indexer's upstream producers.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module; the product path
never does.  It shares no code with the CUDA library.

What it computes (StreamIndex: Memory-Bounded Compressed Sparse Attention via
Streaming Top-k, Abstract): the lightning indexer scores the queries against
keys compressed at ratio m; the Abstract calls the score a learned projection
and gives neither the projections nor the compressor.  This library takes the
plainest reading, with the weights in the usual [out, in] layout:

    q[b,t,h,:]  = x[b,t,:] . W_q[h*d_I:(h+1)*d_I, :]^T      (bf16 output)
    w[b,t,h]    = x[b,t,:] . W_w[h, :]^T                    (fp32 output)
    kc[b,s,:]   = (1/m) sum_{j<m} x[b, s*m + j, :] . W_k^T  (bf16 output)

for s < T = floor(S/m): each compressed key averages the m consecutive
tokens it covers and projects the average.  Every value here is the exact
fp64 result from the bf16 inputs (numpy matmul as the library step).
"""
from __future__ import annotations

import numpy as np


def bf16_to_f64(bits) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def project(x_bits, w_bits) -> np.ndarray:
    """x [..., Din] (bf16 bits) times W [Dout, Din]^T (bf16 bits), in fp64."""
    return bf16_to_f64(x_bits) @ bf16_to_f64(w_bits).T


def compress_keys(x_bits, wk_bits, m: int) -> np.ndarray:
    """kc [B, T, d_I] from x [B, S, Din]: the mean of each group of m
    consecutive tokens (the last S - T*m tokens, if any, are not covered),
    projected by W_k [d_I, Din], in fp64."""
    x = bf16_to_f64(x_bits)
    B, S, Din = x.shape
    T = S // m
    pooled = x[:, :T * m].reshape(B, T, m, Din).mean(axis=2)
    return pooled @ bf16_to_f64(wk_bits).T
