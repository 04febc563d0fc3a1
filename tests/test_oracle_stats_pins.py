"""Pins of the oracle's per-row softmax statistics (m, l).

The statistics follow the BPT page, section "The backward pass" (the forward
keeps (m, l) per row so that the backward recomputes each block's softmax
exactly).  Pinned against library routines (torch max / logsumexp over
scores built with torch ops), a pure-Python brute force, a closed form and
an invariant.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from blockwise_attn_ffn_b200.inputs import LayerShape, make_inputs, sample_rows


def tiny(N=24, d=16, h=2, d_ff=40, causal=True, seed=7, B=2):
    cfg = LayerShape("t", B=B, N=N, d=d, h=h, d_ff=d_ff, causal=causal, dtype="f32", block=8,
                     seed=seed, ln_scale=0.2, bias_scale=0.3)
    return cfg, make_inputs(cfg)


def all_rows(B, N):
    return np.array([(b, i) for b in range(B) for i in range(N)], dtype=np.int64)


def torch_stats(inp, h, causal):
    """max and logsumexp of each row's scores, from torch library routines."""
    T = lambda k: torch.from_numpy(np.asarray(inp[k], np.float64))
    X = T("x")
    B, N, d = X.shape
    d_k = d // h
    U = F.layer_norm(X, (d,), T("gamma1"), T("beta1"), eps=1e-5)
    Q, K = U @ T("W_Q"), U @ T("W_K")
    Qh = Q.view(B, N, h, d_k).transpose(1, 2)
    Kh = K.view(B, N, h, d_k).transpose(1, 2)
    S = Qh @ Kh.transpose(-1, -2) / math.sqrt(d_k)
    if causal:
        S = S.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
    return S.amax(-1).numpy(), torch.logsumexp(S, -1).numpy()  # [B, h, N]


@pytest.mark.parametrize("causal", [False, True])
def test_stats_vs_torch_max_and_logsumexp(causal):
    cfg, inp = tiny(N=37, d=32, h=4, causal=causal)
    m, l = oracle.attention_stats_rows(inp, cfg.h, causal, all_rows(cfg.B, cfg.N))
    mx, lse = torch_stats(inp, cfg.h, causal)
    m = m.reshape(cfg.B, cfg.N, cfg.h).transpose(0, 2, 1)
    l = l.reshape(cfg.B, cfg.N, cfg.h).transpose(0, 2, 1)
    np.testing.assert_allclose(m, mx, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(m + np.log(l), lse, rtol=1e-12, atol=1e-12)


def scalar_stats(inp, h, causal):
    """Pure-Python loops: (m, l) per (batch, row, head)."""
    L = lambda k: np.asarray(inp[k], np.float64).tolist()
    X = L("x")
    WQ, WK = L("W_Q"), L("W_K")
    g1, be1 = L("gamma1"), L("beta1")
    d = len(WQ)
    d_k = d // h

    def ln(row):
        mu = sum(row) / len(row)
        var = sum((a - mu) ** 2 for a in row) / len(row)
        return [(a - mu) / math.sqrt(var + 1e-5) * g1[k] + be1[k] for k, a in enumerate(row)]

    def vecmat(v, W):
        return [sum(v[i] * W[i][j] for i in range(len(v))) for j in range(len(W[0]))]

    out = {}
    for b, Xb in enumerate(X):
        N = len(Xb)
        U = [ln(r) for r in Xb]
        Q = [vecmat(u, WQ) for u in U]
        K = [vecmat(u, WK) for u in U]
        for i in range(N):
            for t in range(h):
                cols = range(t * d_k, (t + 1) * d_k)
                keys = range(i + 1) if causal else range(N)
                sc = [sum(Q[i][c] * K[j][c] for c in cols) / math.sqrt(d_k) for j in keys]
                mx = max(sc)
                out[(b, i, t)] = (mx, sum(math.exp(s - mx) for s in sc))
    return out


@pytest.mark.parametrize("causal", [False, True])
def test_stats_vs_scalar_brute_force(causal):
    cfg, inp = tiny(N=7, d=8, h=2, d_ff=12, causal=causal)
    rows = all_rows(cfg.B, cfg.N)
    m, l = oracle.attention_stats_rows(inp, cfg.h, causal, rows)
    ref = scalar_stats(inp, cfg.h, causal)
    for k, (b, i) in enumerate(rows):
        for t in range(cfg.h):
            assert m[k, t] == pytest.approx(ref[(b, i, t)][0], rel=1e-12, abs=1e-12)
            assert l[k, t] == pytest.approx(ref[(b, i, t)][1], rel=1e-12, abs=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_zero_WQ_gives_zero_max_and_key_count(causal):
    """All scores are 0: m = 0 and l = the number of keys the row sees."""
    cfg, inp = tiny(N=19, causal=causal)
    inp = dict(inp)
    inp["W_Q"] = np.zeros_like(inp["W_Q"])
    rows = all_rows(cfg.B, cfg.N)
    m, l = oracle.attention_stats_rows(inp, cfg.h, causal, rows)
    seen = (rows[:, 1] + 1) if causal else np.full(len(rows), cfg.N)
    np.testing.assert_array_equal(m, 0.0)
    np.testing.assert_allclose(l, np.repeat(seen[:, None], cfg.h, axis=1), rtol=1e-15)


def test_stats_invariant_bounds_on_a_workload_shape():
    """1 <= l <= (keys seen): the maximum's own term is exp(0) = 1 and every
    term is at most 1."""
    cfg = LayerShape("s", B=1, N=700, d=256, h=4, d_ff=512, causal=True, dtype="bf16",
                     block=128, seed=3, ln_scale=0.1)
    inp = make_inputs(cfg)
    rows = sample_rows(cfg, 40, B=1)
    m, l = oracle.attention_stats_rows(inp, cfg.h, True, rows)
    seen = rows[:, 1] + 1
    assert np.all(np.isfinite(m))
    assert np.all(l >= 1.0 - 1e-12)
    assert np.all(l <= seen[:, None] + 1e-9)
