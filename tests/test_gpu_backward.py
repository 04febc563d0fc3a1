"""bpt_layer_backward against the fp64 backward oracle.

BPT page, section "The backward pass".  The CUDA path recomputes each wave
of query blocks from x and the saved (m, l) (bpt_layer_forward_train) and
accumulates the gradients; the oracle is the chain rule through the unfused
layer (``oracle.layer_backward``, pinned against torch autograd).

Tolerance (bf16 layers).  Every GEMM operand on the backward path is rounded to fp16
(relative error <= 2^-11 ~ 4.9e-4, ~2.8e-4 rms for a uniformly distributed
rounding error) and the longest chain (dZ -> dH -> dHpre -> dVn -> dY -> dO
-> dS -> dQ, dK, dV -> dU -> dx) passes about ten such roundings, each
product accumulated in fp32: independent roundings give a relative rms error
near sqrt(10) x 2.8e-4 ~ 9e-4.  Each gradient tensor is held to a relative L2
error of 3e-3 (3x that) and a largest elementwise error of 1 % of the
tensor's largest magnitude (a few rms).  Measured: <= 7.7e-4 and <= 1.2e-3.
"""
import numpy as np
import pytest
import torch

import blockwise_attn_ffn_b200 as bpt
import oracle
from blockwise_attn_ffn_b200.inputs import WORKLOADS, LayerShape, make_inputs
from test_gpu_parity import small

pytestmark = pytest.mark.gpu

NAMES = {"x": "x", "W_Q": "W_Q", "W_K": "W_K", "W_V": "W_V", "W_O": "W_O", "W_1": "W_1",
         "b_1": "b_1", "W_2": "W_2", "b_2": "b_2"}

CASES = [
    small("bwd_dk128_causal", 2, 384, 256, 2, 512, True, seed=21),
    small("bwd_dk64_noncausal_ragged", 1, 200, 256, 4, 512, False, seed=22),
    small("bwd_dk128_ragged_bias", 1, 300, 384, 3, 768, True, seed=23, bias=0.5),
    small("bwd_d192_straddle", 1, 260, 192, 3, 448, True, seed=24),
]


def upstream(cfg, seed=77):
    return np.random.default_rng(seed).standard_normal((cfg.B, cfg.N, cfg.d)).astype(np.float32)


def run_backward(cfg, inp, dZ, max_wave=0):
    dev = bpt.to_device(inp, cfg.dtype)
    x = dev["x"]
    fwd_opts = {"schedule": "waves", "max_wave": max_wave} if max_wave else None
    _, stats, ws = bpt.layer_forward_train(x, dev, cfg.h, cfg.causal, opts=fwd_opts)
    grads, bws = bpt.layer_backward(x, dev, cfg.h, cfg.causal, stats,
                                    torch.from_numpy(dZ).cuda(),
                                    opts={"max_wave": max_wave} if max_wave else None)
    for w in (ws, bws):
        st, site = bpt.bpt_read_device_error(w.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert st == bpt.BPT_OK, f"device error {bpt.status_string(st)} at site {site}"
    return {k: v.cpu().numpy().astype(np.float64) for k, v in grads.items()}


def check(name, got, want):
    assert np.all(np.isfinite(got)), f"{name}: non-finite gradient"
    scale = np.abs(want).max()
    rel_l2 = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
    mx = np.abs(got - want).max()
    print(f"  {name:12s} rel L2 {rel_l2:.2e}  max {mx / max(scale, 1e-30):.2e} of scale")
    assert rel_l2 <= 3e-3, f"{name}: relative L2 error {rel_l2:.3e}"
    assert mx <= 1e-2 * scale, f"{name}: max abs error {mx:.3e} vs scale {scale:.3e}"
    return rel_l2


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_backward_matches_oracle(cfg):
    inp = make_inputs(cfg)
    dZ = upstream(cfg)
    got = run_backward(cfg, inp, dZ)
    want = oracle.layer_backward(inp, cfg.h, cfg.causal, dZ.astype(np.float64))
    for k in NAMES:
        check(k, got[k], want[k])
    for k, (g, b) in {"ln1": ("gamma1", "beta1"), "ln2": ("gamma2", "beta2")}.items():
        check(k + ".gamma", got[k][0], want[g])
        check(k + ".beta", got[k][1], want[b])


# Multi-wave schedules on small layers (bpt_options.max_wave): a sequence
# split over three waves, and one whole sequence per wave.
WAVE_CASES = [
    (small("bwd_split_sequence", 1, 700, 256, 2, 512, True, seed=25), 2),
    (small("bwd_split_sequence_dk64", 1, 650, 256, 4, 512, True, seed=26), 2),
    (small("bwd_one_sequence_per_wave", 3, 256, 256, 4, 512, False, seed=27), 2),
]


@pytest.mark.parametrize("cfg,blocks", WAVE_CASES, ids=lambda c: getattr(c, "name", str(c)))
def test_backward_multi_wave(cfg, blocks):
    inp = make_inputs(cfg)
    dZ = upstream(cfg)
    got = run_backward(cfg, inp, dZ, max_wave=blocks)
    want = oracle.layer_backward(inp, cfg.h, cfg.causal, dZ.astype(np.float64))
    for k in NAMES:
        check(k, got[k], want[k])
    for k, (g, b) in {"ln1": ("gamma1", "beta1"), "ln2": ("gamma2", "beta2")}.items():
        check(k + ".gamma", got[k][0], want[g])
        check(k + ".beta", got[k][1], want[b])


def test_backward_is_deterministic():
    cfg = CASES[0]
    inp = make_inputs(cfg)
    dZ = upstream(cfg)
    a = run_backward(cfg, inp, dZ)
    b = run_backward(cfg, inp, dZ)
    for k in a:
        np.testing.assert_array_equal(a[k], b[k], err_msg=k)


# fp32 layers: the same schedule on the CUDA cores, every product in fp32.
# Errors are fp32 rounding along the same chain (unit roundoff 6e-8, sums of
# a few hundred terms): held to relative L2 1e-4 and elementwise 1e-3 of the
# tensor's largest magnitude.
F32_CASES = [
    small("bwd_f32_causal_ragged", 2, 150, 64, 2, 192, True, dtype="f32", seed=31, bias=0.5),
    small("bwd_f32_noncausal", 1, 100, 96, 3, 160, False, dtype="f32", seed=32),
    small("bwd_f32_dk128_multiblock", 1, 200, 256, 2, 256, True, dtype="f32", seed=33),
]


def check_f32(name, got, want):
    assert np.all(np.isfinite(got)), f"{name}: non-finite gradient"
    scale = np.abs(want).max()
    rel_l2 = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
    mx = np.abs(got - want).max()
    print(f"  {name:12s} rel L2 {rel_l2:.2e}  max {mx / max(scale, 1e-30):.2e} of scale")
    assert rel_l2 <= 1e-4, f"{name}: relative L2 error {rel_l2:.3e}"
    assert mx <= 1e-3 * scale, f"{name}: max abs error {mx:.3e} vs scale {scale:.3e}"


@pytest.mark.parametrize("cfg", F32_CASES, ids=lambda c: c.name)
def test_f32_backward_matches_oracle(cfg):
    inp = make_inputs(cfg)
    dZ = upstream(cfg)
    got = run_backward(cfg, inp, dZ)
    want = oracle.layer_backward(inp, cfg.h, cfg.causal, dZ.astype(np.float64))
    for k in NAMES:
        check_f32(k, got[k], want[k])
    for k, (g, b) in {"ln1": ("gamma1", "beta1"), "ln2": ("gamma2", "beta2")}.items():
        check_f32(k + ".gamma", got[k][0], want[g])
        check_f32(k + ".beta", got[k][1], want[b])


def test_f32_backward_multi_wave():
    cfg = small("bwd_f32_split", 1, 300, 64, 2, 192, True, dtype="f32", seed=34)
    inp = make_inputs(cfg)
    dZ = upstream(cfg)
    got = run_backward(cfg, inp, dZ, max_wave=2)
    want = oracle.layer_backward(inp, cfg.h, cfg.causal, dZ.astype(np.float64))
    for k in NAMES:
        check_f32(k, got[k], want[k])



def test_backward_full_gpt2_small_workload():
    """Every gradient of the whole GPT-2-small-shaped workload (B 8, N 2048,
    d 768, 12 heads, d_ff 3072, causal) against the fp64 backward oracle:
    the full-size check of the block recomputation at the shape it runs in
    production, every element compared."""
    cfg = WORKLOADS["gpt2s_n2k"]
    inp = make_inputs(cfg)
    dZ = upstream(cfg)
    got = run_backward(cfg, inp, dZ)
    want = oracle.layer_backward(inp, cfg.h, cfg.causal, dZ.astype(np.float64))
    for k in NAMES:
        check(k, got[k], want[k])
    for k, (g, b) in {"ln1": ("gamma1", "beta1"), "ln2": ("gamma2", "beta2")}.items():
        check(k + ".gamma", got[k][0], want[g])
        check(k + ".beta", got[k][1], want[b])


KEEP_O_CASES = [
    (CASES[0], "fused", 0),                 # two sequences, one wave
    (CASES[2], "fused", 0),                 # ragged N (padded rows in the last block)
    (CASES[1], "waves", 1),                 # waves forward, one block per wave
    (small("keep_o_dk128_split", 1, 900, 256, 2, 512, True, seed=25), "waves", 3),
]


@pytest.mark.parametrize("cfg,schedule,wave", KEEP_O_CASES,
                         ids=lambda c: getattr(c, "name", str(c)))
def test_backward_with_kept_attention_output(cfg, schedule, wave):
    """bpt_layer_forward_train_keep_o writes the attention output it fed to
    W_O (checked against the oracle's O), with out and stats bitwise those
    of bpt_layer_forward_train; bpt_layer_backward_keep_o, which reads it
    instead of recomputing the attention, gives bitwise the gradients of
    bpt_layer_backward."""
    inp = make_inputs(cfg)
    dev = bpt.to_device(inp, cfg.dtype)
    x = dev["x"]
    opts = {"schedule": schedule, "max_wave": wave}
    out0, stats0, _ = bpt.layer_forward_train(x, dev, cfg.h, cfg.causal, opts=opts)
    o = torch.full((cfg.B, cfg.N, cfg.d), float("nan"), dtype=torch.float16, device="cuda")
    out1, stats1, ws = bpt.layer_forward_train(x, dev, cfg.h, cfg.causal, opts=opts, keep_o=o)
    st, site = bpt.bpt_read_device_error(ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == bpt.BPT_OK, f"device error {bpt.status_string(st)} at site {site}"
    assert torch.equal(out0, out1) and torch.equal(stats0, stats1)
    got_o = o.float().cpu().numpy()
    assert np.all(np.isfinite(got_o))
    for b in range(cfg.B):
        want_o = oracle.layer_intermediates(inp, cfg.h, cfg.causal, b)["O"]
        err = np.abs(got_o[b] - want_o)
        # fp16 scores / P / V and an fp16 output: a few fp16 roundings of values <= ~3
        assert err.max() < 2e-2 and err.mean() < 2e-3, (b, err.max(), err.mean())
    dZ = torch.from_numpy(upstream(cfg)).cuda()
    bopts = {"max_wave": wave} if wave else None
    g_rec, _ = bpt.layer_backward(x, dev, cfg.h, cfg.causal, stats1, dZ, opts=bopts)
    g_kept, bws = bpt.layer_backward(x, dev, cfg.h, cfg.causal, stats1, dZ, opts=bopts, o=o)
    st, site = bpt.bpt_read_device_error(bws.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == bpt.BPT_OK, f"device error {bpt.status_string(st)} at site {site}"
    for k in g_rec:
        assert torch.equal(g_rec[k], g_kept[k]), k
