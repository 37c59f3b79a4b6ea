"""The indexer's upstream producers (si_indexer_inputs) against the fp64
oracle (oracle/producers.py) on the GPU, and the whole CSA step composed
from hidden states (needs a B200)."""
import numpy as np
import pytest
import torch

import streaming_top_indexer_b200 as si
from oracle import producers as pr
from streaming_top_indexer_b200 import synth
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu

DEV = "cuda"


def check_output(got, ref, absdot, K, bf16_out, scale_err=0.0, where=""):
    """|got - ref| <= 1.01 * K * 2^-23 * sum|x||W| (fp32 accumulation of exact
    bf16 products) + 2^-8 |ref| if rounded to bf16 (8 significant bits) +
    scale_err |ref| (a rounded 1/m)."""
    tol = 1.01 * K * 2.0 ** -23 * absdot + (2.0 ** -8 if bf16_out else 0.0) * np.abs(ref) + scale_err * np.abs(ref)
    err = np.abs(got - ref)
    assert np.all(err <= tol + 1e-300), f"{where}: {np.count_nonzero(err > tol)} outside, worst {err.max():.3g}"


def bits(t):
    return synth.bf16_bits(t)


@pytest.mark.parametrize("B,S,DM,H,D,m", [
    (2, 300, 128, 8, 64, 4),       # ragged S (300 = 75*4), two batches
    (1, 1000, 256, 64, 128, 4),    # V4-shaped heads, several row tiles
    (1, 259, 192, 16, 64, 3),      # m = 3 (1/m rounded), ragged tail of 1 token
])
def test_producers_match_oracle(B, S, DM, H, D, m):
    x, w_q, w_w, w_k = synth.generate_hidden(B, S, DM, H, D, m, seed=S, device=DEV)
    q, w, kc, st = si.indexer_inputs(x, w_q, w_w, w_k, H, D, m)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    xb, wqb, wwb, wkb = bits(x), bits(w_q), bits(w_w), bits(w_k)
    xa = np.abs(pr.bf16_to_f64(xb))
    ref_q = pr.project(xb, wqb).reshape(B, S, H, D)
    check_output(q.float().cpu().numpy(), ref_q, (xa @ np.abs(pr.bf16_to_f64(wqb)).T).reshape(B, S, H, D), DM, True,
                 where="q")
    ref_w = pr.project(xb, wwb)
    check_output(w.cpu().numpy(), ref_w, xa @ np.abs(pr.bf16_to_f64(wwb)).T, DM, False, where="w")
    T = S // m
    ref_kc = pr.compress_keys(xb, wkb, m)
    pooled_abs = xa[:, :T * m].reshape(B, T, m, DM).sum(axis=2) / m
    check_output(kc.float().cpu().numpy(), ref_kc, pooled_abs @ np.abs(pr.bf16_to_f64(wkb)).T, m * DM, True,
                 scale_err=0.0 if m in (1, 2, 4, 8) else 2.0 ** -23, where="kc")


def test_csa_step_from_hidden_states():
    """x -> producers -> indexer top-k -> sparse attention, at S = 16,384 with
    the V4-shaped heads: the indexer's rows against the oracle on the
    produced inputs, and the attention output finite with lse set wherever a
    key is visible."""
    B, S, DM, H, D, m, k = 1, 16384, 1024, 64, 128, 4, 512
    x, w_q, w_w, w_k = synth.generate_hidden(B, S, DM, H, D, m, seed=1, device=DEV)
    q, w, kc, st = si.indexer_inputs(x, w_q, w_w, w_k, H, D, m)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    b_rows, t_rows = gh.sampled_rows(B, S, m, k, n=128)
    rep = gh.check_against_oracle(q, w, kc, m, k, b_rows, t_rows, where="produced inputs")
    assert rep["recall_min"] >= 0.998
    idx, _ = gh.gpu_topk(q, w, kc, m, k)
    qa, ka, va = synth.generate_attention(B, S, S // m, seed=1, device=DEV)
    out, lse, ast = si.sparse_attention(qa, ka, va, idx, 1.0 / np.sqrt(128))
    torch.cuda.synchronize()
    assert int(ast.item()) == 0
    vis = torch.clamp((torch.arange(S, device=DEV) + 1) // m, max=S // m) > 0
    assert torch.all(torch.isfinite(lse[0, vis])) and torch.all(torch.isneginf(lse[0, ~vis]))
    assert torch.all(torch.isfinite(out.float()))


def test_long_shape_sampled_rows():
    """The headline shape's producers (S = 262,144, d_model = 4096, H_I = 64,
    d_I = 128, m = 4): sampled rows of q and w and sampled compressed keys
    against the oracle."""
    B, S, DM, H, D, m = 1, 262144, 4096, 64, 128, 4
    x, w_q, w_w, w_k = synth.generate_hidden(B, S, DM, H, D, m, seed=2, device=DEV)
    q, w, kc, st = si.indexer_inputs(x, w_q, w_w, w_k, H, D, m)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rng = np.random.default_rng(5)
    rows = np.sort(rng.choice(S, 64, replace=False))
    keys = np.sort(rng.choice(S // m, 64, replace=False))
    tr = torch.from_numpy(rows).to(DEV)
    xb = bits(x[0, tr])
    xa = np.abs(pr.bf16_to_f64(xb))
    wqb, wwb, wkb = bits(w_q), bits(w_w), bits(w_k)
    check_output(q[0, tr].float().cpu().numpy().reshape(64, -1), pr.project(xb, wqb),
                 xa @ np.abs(pr.bf16_to_f64(wqb)).T, DM, True, where="q long")
    check_output(w[0, tr].cpu().numpy(), pr.project(xb, wwb), xa @ np.abs(pr.bf16_to_f64(wwb)).T, DM, False,
                 where="w long")
    tok = torch.from_numpy((keys[:, None] * m + np.arange(m)[None]).reshape(-1)).to(DEV)
    xk = bits(x[0, tok]).reshape(64, m, DM)
    ref = pr.compress_keys(xk.reshape(1, 64 * m, DM), wkb, m)[0]
    pooled_abs = np.abs(pr.bf16_to_f64(xk)).sum(axis=1) / m
    check_output(kc[0, torch.from_numpy(keys).to(DEV)].float().cpu().numpy(), ref,
                 pooled_abs @ np.abs(pr.bf16_to_f64(wkb)).T, m * DM, True, where="kc long")
