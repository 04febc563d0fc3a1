"""Pins of the gated-attention oracle (``oracle.bsfa``).

"Block Sparse Flash Attention", sections "Methodology and Mechanism" and
"Gating Mechanism and Threshold Calibration".  Pinned against things the
oracle does not compute itself: the ungated oracle and torch's scaled
dot-product attention (thresholds -inf: nothing pruned), torch attention
under a block-diagonal boolean mask (thresholds +inf: only the diagonal),
a pure-Python brute force of the block maxima and the gate on a tiny ragged
case followed by torch attention under the brute-force mask, and the
calibration's counting property (exactly k blocks pass on the sample it was
fitted to).
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from blockwise_attn_ffn_b200.inputs import LayerShape, make_inputs


def qkv(seed=3, N=23, d=16, h=2):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((N, d)), rng.standard_normal((N, d)),
            rng.standard_normal((N, d)))


def torch_masked_attention(Q, K, V, h, mask):
    """softmax(q.k / sqrt(d_k)) V per head under a boolean [N, N] mask (True
    = may attend), by torch's library routine."""
    N, d = Q.shape
    dk = d // h
    heads = lambda A: torch.from_numpy(A).reshape(N, h, dk).transpose(0, 1)[None]
    o = F.scaled_dot_product_attention(heads(Q), heads(K), heads(V),
                                       attn_mask=torch.from_numpy(mask)[None, None])
    return o[0].transpose(0, 1).reshape(N, d).numpy()


@pytest.mark.parametrize("causal", [False, True])
def test_no_threshold_is_exact_attention(causal):
    Q, K, V = qkv()
    h, b, N = 2, 5, Q.shape[0]
    nb = (N + b - 1) // b
    O, keep, _ = oracle.attention_gated(Q, K, V, h, causal, np.full((h, nb), -np.inf), b)
    want = oracle.attention_rows(Q, K, V, h, causal, np.arange(N))
    np.testing.assert_allclose(O, want, rtol=1e-12, atol=1e-12)
    mask = np.tril(np.ones((N, N), bool)) if causal else np.ones((N, N), bool)
    np.testing.assert_allclose(O, torch_masked_attention(Q, K, V, h, mask), rtol=1e-10,
                               atol=1e-12)
    for t in range(h):
        vis = np.tril(np.ones((nb, nb), bool)) if causal else np.ones((nb, nb), bool)
        np.testing.assert_array_equal(keep[t], vis)


@pytest.mark.parametrize("causal", [False, True])
def test_infinite_threshold_keeps_only_the_diagonal_block(causal):
    Q, K, V = qkv(seed=4)
    h, b, N = 2, 6, Q.shape[0]
    nb = (N + b - 1) // b
    O, keep, _ = oracle.attention_gated(Q, K, V, h, causal, np.full((h, nb), np.inf), b)
    blk = np.arange(N) // b
    mask = blk[:, None] == blk[None, :]
    if causal:
        mask &= np.tril(np.ones((N, N), bool))
    np.testing.assert_allclose(O, torch_masked_attention(Q, K, V, h, mask), rtol=1e-10,
                               atol=1e-12)
    for t in range(h):
        np.testing.assert_array_equal(keep[t], np.eye(nb, dtype=bool))


@pytest.mark.parametrize("causal", [False, True])
def test_brute_force_gate_on_a_ragged_case(causal):
    """Block maxima by explicit loops over (query, key) pairs, thresholds that
    differ per head and per query block (a transposed index or a wrong head
    would change the kept set), then torch attention under that mask."""
    N, d, h, b = 17, 8, 2, 4          # 5 blocks, the last one row long
    Q, K, V = qkv(seed=9, N=N, d=d, h=h)
    nb = (N + b - 1) // b
    dk = d // h
    rng = np.random.default_rng(1)
    T = rng.uniform(-0.5, 1.5, size=(h, nb))
    O, keep, bmax = oracle.attention_gated(Q, K, V, h, causal, T, b)
    mask = np.zeros((h, N, N), bool)
    for t in range(h):
        for i in range(nb):
            for j in range(nb):
                best = -math.inf
                for p in range(i * b, min(N, i * b + b)):
                    for q in range(j * b, min(N, j * b + b)):
                        if causal and q > p:
                            continue
                        s = sum(Q[p, t * dk + c] * K[q, t * dk + c] for c in range(dk))
                        best = max(best, s / math.sqrt(dk))
                assert bmax[t, i, j] == pytest.approx(best, rel=1e-12, abs=1e-12)
                kept = best > -math.inf and (i == j or best >= T[t, i])
                assert keep[t, i, j] == kept, (t, i, j)
                if kept:
                    mask[t, i * b:min(N, i * b + b), j * b:min(N, j * b + b)] = True
        if causal:
            mask[t] &= np.tril(np.ones((N, N), bool))
    assert 0 < keep.sum() < keep.size  # the thresholds prune some blocks, not all
    for t in range(h):
        c = slice(t * dk, (t + 1) * dk)
        want = torch_masked_attention(Q[:, c], K[:, c], V[:, c], 1, mask[t])
        np.testing.assert_allclose(O[:, c], want, rtol=1e-10, atol=1e-12)


def test_layer_gated_without_pruning_is_the_layer():
    cfg = LayerShape("t", B=2, N=19, d=16, h=2, d_ff=40, causal=True, dtype="f32", block=8,
                     seed=5, ln_scale=0.2, bias_scale=0.3)
    inp = make_inputs(cfg)
    nb = (cfg.N + 7) // 8
    Z, keep, _ = oracle.layer_gated(inp, cfg.h, True, np.full((cfg.h, nb), -np.inf), b=8)
    np.testing.assert_allclose(Z, oracle.layer_unfused(inp, cfg.h, True), rtol=1e-12,
                               atol=1e-12)
    assert keep.sum() == cfg.B * cfg.h * nb * (nb + 1) // 2


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("k", [0, 1, 3])
def test_calibration_keeps_exactly_k_blocks_on_its_sample(causal, k):
    Q, K, _ = qkv(seed=12, N=40, d=16, h=2)
    h, b = 2, 5
    nb = 8
    bm = np.stack([oracle.block_max(oracle.head_scores(Q, K, h, t), causal, b)
                   for t in range(h)])
    T = oracle.calibrate_thresholds([bm], k, causal)
    for t in range(h):
        keep = oracle.keep_mask(bm[t], T[t], causal)
        for i in range(nb):
            cands = i if causal else nb - 1
            off = int(keep[i].sum()) - 1  # minus the diagonal
            assert off == min(k, cands), (t, i)
    # averaging identical samples changes nothing; more blocks kept -> lower T
    np.testing.assert_array_equal(oracle.calibrate_thresholds([bm, bm], k, causal), T)
    T_more = oracle.calibrate_thresholds([bm], k + 1, causal)
    assert np.all(T_more <= T)
