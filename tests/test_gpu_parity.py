"""CUDA path vs the fp64 oracle, through the C ABI (needs a B200).

Small cases are compared element by element; they span several query blocks,
several GEMM tiles and a ragged last block.  The full-size workloads run in the
same launch configuration as the bench and are compared on every row (GPT-2
and mid-context shapes) or on 256 seeded sampled rows (long-context shapes),
which is exact by the token-wise property of everything after attention.
"""
import numpy as np
import pytest
import torch

import oracle
from blockwise_attn_ffn_b200.inputs import LayerShape, WORKLOADS, make_inputs, sample_rows

from gpu_util import compare, run_cuda, tol_for, workspace_qkv

pytestmark = pytest.mark.gpu


def small(name, B, N, d, h, d_ff, causal, dtype="bf16", seed=11, bias=0.0, ln=0.1):
    return LayerShape(name, B=B, N=N, d=d, h=h, d_ff=d_ff, causal=causal, dtype=dtype,
                      block=128 if dtype == "bf16" else 64, seed=seed, ln_scale=ln,
                      bias_scale=bias)


SMALL = [
    small("dk128_causal", 2, 384, 256, 2, 512, True),
    small("dk128_noncausal", 2, 384, 256, 2, 512, False),
    small("dk64_causal_ragged", 2, 300, 256, 4, 512, True),
    small("dk64_noncausal_ragged", 1, 200, 256, 4, 512, False),
    small("dk128_bias_ragged", 1, 520, 384, 3, 768, True, bias=0.5),
    small("one_block", 1, 128, 128, 1, 256, True),
    small("single_token", 1, 1, 128, 2, 256, True),
    # d and d_ff = 64 (mod 128): a GEMM CTA's 128 B columns straddle W_Q | W_K
    # | W_V, every K leaves the last 128-deep stage half empty, and W_1's last
    # column span is half past the end.
    small("d192_straddle", 1, 260, 192, 3, 448, True, seed=13),
    small("f32_causal_ragged", 2, 150, 64, 2, 192, True, dtype="f32"),
    small("f32_noncausal_bias", 1, 100, 96, 3, 160, False, dtype="f32", bias=0.5),
]


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_small_layers_elementwise(cfg):
    inp = make_inputs(cfg)
    got, _, _ = run_cuda(cfg, inp)
    want = oracle.layer_unfused(inp, cfg.h, cfg.causal)
    compare(got, want, tol_for(cfg))


def test_tiny_f32_workload():
    cfg = WORKLOADS["tiny_f32"]
    inp = make_inputs(cfg)
    got, _, _ = run_cuda(cfg, inp)
    compare(got, oracle.layer_unfused(inp, cfg.h, cfg.causal), tol_for(cfg))


@pytest.mark.parametrize("cfg", [SMALL[0], SMALL[2], SMALL[7], SMALL[8]], ids=lambda c: c.name)
def test_qkv_projection_in_workspace(cfg):
    """Step a2 alone: the Q/K/V rows the prologue GEMM wrote."""
    inp = make_inputs(cfg)
    _, _, ws = run_cuda(cfg, inp)
    qkv = workspace_qkv(ws, cfg, cfg.B)
    for b in range(cfg.B):
        it = oracle.layer_intermediates(inp, cfg.h, cfg.causal, b=b)
        want = np.concatenate([it["Q"], it["K"], it["V"]], axis=1)
        tol = (1e-4, None) if cfg.dtype == "f32" else (2e-2, 2e-3)
        compare(qkv[b], want, tol)


def test_deterministic():
    cfg = SMALL[0]
    inp = make_inputs(cfg)
    a, _, _ = run_cuda(cfg, inp)
    b, _, _ = run_cuda(cfg, inp)
    np.testing.assert_array_equal(a, b)


def test_several_waves_in_one_sequence():
    """nb > BPT_WAVE_BLOCKS: the sequence is processed in several waves."""
    cfg = small("waves", 1, 128 * 300, 128, 2, 256, True, seed=5)
    inp = make_inputs(cfg)
    got, _, _ = run_cuda(cfg, inp)
    rows = sample_rows(cfg, 96)
    want = oracle.layer_rows(inp, cfg.h, cfg.causal, rows)
    compare(got[rows[:, 0], rows[:, 1]], want, tol_for(cfg))


def test_several_waves_of_whole_sequences():
    cfg = small("seqwaves", 5, 128 * 100, 128, 2, 256, True, seed=6)
    inp = make_inputs(cfg)
    got, _, _ = run_cuda(cfg, inp)
    rows = sample_rows(cfg, 96)
    want = oracle.layer_rows(inp, cfg.h, cfg.causal, rows)
    compare(got[rows[:, 0], rows[:, 1]], want, tol_for(cfg))


@pytest.mark.parametrize("name", ["gpt2s_n2k", "mid_n16k"])
def test_workload_all_rows(name):
    cfg = WORKLOADS[name]
    inp = make_inputs(cfg)
    got, _, _ = run_cuda(cfg, inp)
    compare(got, oracle.layer_unfused(inp, cfg.h, cfg.causal), tol_for(cfg))


@pytest.mark.parametrize("name", ["long_n64k", "wide_n128k"])
def test_workload_sampled_rows(name):
    cfg = WORKLOADS[name]
    inp = make_inputs(cfg)
    got, _, _ = run_cuda(cfg, inp)
    rows = sample_rows(cfg, 256)
    want = oracle.layer_rows(inp, cfg.h, cfg.causal, rows)
    del inp
    compare(got[rows[:, 0], rows[:, 1]], want, tol_for(cfg))
