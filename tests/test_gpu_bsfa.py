"""bpt_layer_forward_bsfa (block-gated attention) against the fp64 gated oracle.

"Block Sparse Flash Attention", sections "Methodology and Mechanism" and
"Gating Mechanism and Threshold Calibration".  The gate is a floating-point
comparison, so the thresholds used for the element-wise checks are placed in
gaps between the oracle's block maxima wider than the score tolerance: the
kept set is then unique and compared exactly, and the outputs within the
layer tolerance.  The block maxima themselves are compared with the score
tolerance of the statistics test (fp16 Q and K, fp32 accumulation).
"""
import numpy as np
import pytest
import torch

import blockwise_attn_ffn_b200 as bpt
import oracle
from blockwise_attn_ffn_b200.inputs import make_inputs
from gpu_util import compare, tol_for
from test_gpu_parity import small

pytestmark = pytest.mark.gpu

CASES = [
    small("bsfa_dk128_causal", 2, 1000, 256, 2, 512, True, seed=51),
    small("bsfa_dk64_causal_ragged", 1, 900, 256, 4, 512, True, seed=52),
    small("bsfa_dk64_noncausal", 1, 700, 256, 4, 512, False, seed=53),
]


def smax_tol(s):
    return 3e-2 + 3e-3 * np.abs(s)


def gap_thresholds(bmax, causal, rng):
    """T [h, nb]: per (head, query block) a value in a gap of the off-diagonal
    block maxima (all batch elements) wider than twice the tolerance, chosen
    near a random quantile; +inf (prune all) where no gap qualifies."""
    B, h, nb, _ = bmax.shape
    T = np.full((h, nb), np.inf)
    for t in range(h):
        for i in range(nb):
            vals = [bmax[b, t, i, j] for b in range(B) for j in range(nb)
                    if j != i and (j < i or not causal)]
            if not vals:
                T[t, i] = -np.inf
                continue
            v = np.sort(np.array(vals))
            gaps = [(v[k] + v[k + 1]) / 2 for k in range(len(v) - 1)
                    if v[k + 1] - v[k] > 2 * smax_tol(max(abs(v[k]), abs(v[k + 1])))]
            if gaps:
                T[t, i] = gaps[int(rng.integers(len(gaps)))]
    return T


def run_bsfa(cfg, dev, T, opts=None):
    out, bm, kp, ws = bpt.layer_forward_bsfa(dev["x"], dev, cfg.h, cfg.causal,
                                             torch.from_numpy(T.astype(np.float32)).cuda(),
                                             block_max=True, kept=True, opts=opts)
    st, site = bpt.bpt_read_device_error(ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == bpt.BPT_OK, f"device error {bpt.status_string(st)} at site {site}"
    return out.cpu().numpy(), bm.cpu().numpy(), kp.cpu().numpy().astype(bool)


def visited(cfg, nb):
    v = np.tril(np.ones((nb, nb), bool)) if cfg.causal else np.ones((nb, nb), bool)
    return np.broadcast_to(v, (cfg.B, cfg.h, nb, nb))


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_no_pruning_is_bitwise_the_plain_forward(cfg):
    inp = make_inputs(cfg)
    dev = bpt.to_device(inp, cfg.dtype)
    nb = (cfg.N + 127) // 128
    got, bm, kp = run_bsfa(cfg, dev, np.full((cfg.h, nb), -np.inf))
    plain, _ = bpt.layer_forward(dev["x"], dev, cfg.h, cfg.causal)
    np.testing.assert_array_equal(got, plain.cpu().numpy())
    np.testing.assert_array_equal(kp, visited(cfg, nb))
    want = oracle.layer_block_max(inp, cfg.h, cfg.causal)
    vis = visited(cfg, nb)
    err = np.abs(bm[vis] - want[vis])
    assert np.all(err <= smax_tol(want[vis])), f"block max error {err.max():.3e}"
    assert np.all(bm[~vis] == -np.inf)  # unvisited pairs untouched


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_gated_layer_matches_oracle(cfg):
    inp = make_inputs(cfg)
    dev = bpt.to_device(inp, cfg.dtype)
    rng = np.random.default_rng(cfg.seed)
    T = gap_thresholds(oracle.layer_block_max(inp, cfg.h, cfg.causal), cfg.causal, rng)
    want, keep, _ = oracle.layer_gated(inp, cfg.h, cfg.causal, T)
    got, _, kp = run_bsfa(cfg, dev, T)
    np.testing.assert_array_equal(kp, keep)
    nb = keep.shape[-1]
    off = visited(cfg, nb) & ~np.eye(nb, dtype=bool)
    assert 0 < keep[off].sum() < off.sum(), "thresholds must prune some blocks, not all"
    compare(got, want, tol_for(cfg))


@pytest.mark.parametrize("cfg", CASES[:2], ids=lambda c: c.name)
def test_infinite_threshold_keeps_only_diagonal_blocks(cfg):
    inp = make_inputs(cfg)
    dev = bpt.to_device(inp, cfg.dtype)
    nb = (cfg.N + 127) // 128
    T = np.full((cfg.h, nb), np.inf)
    want, keep, _ = oracle.layer_gated(inp, cfg.h, cfg.causal, T)
    got, _, kp = run_bsfa(cfg, dev, T)
    np.testing.assert_array_equal(kp, keep)
    assert kp.sum() == cfg.B * cfg.h * nb
    compare(got, want, tol_for(cfg))


def test_gate_is_independent_of_pairing_and_waves():
    """Single-block CTAs and a sequence split over waves give bitwise the
    same output and kept set as the default launch."""
    cfg = CASES[1]
    inp = make_inputs(cfg)
    dev = bpt.to_device(inp, cfg.dtype)
    rng = np.random.default_rng(7)
    T = gap_thresholds(oracle.layer_block_max(inp, cfg.h, cfg.causal), cfg.causal, rng)
    base, _, kp0 = run_bsfa(cfg, dev, T)
    one, _, kp1 = run_bsfa(cfg, dev, T, opts={"attn_block": 128})
    waves, _, kp2 = run_bsfa(cfg, dev, T, opts={"schedule": "waves", "max_wave": 3})
    np.testing.assert_array_equal(one, base)
    np.testing.assert_array_equal(kp1, kp0)
    np.testing.assert_array_equal(kp2, kp0)
    compare(waves, oracle.layer_gated(inp, cfg.h, cfg.causal, T)[0], tol_for(cfg))
