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

import blockwise_attn_ffn_b200 as bpt
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


@pytest.mark.parametrize("schedule", ["fused", "waves"])
@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_small_layers_elementwise(cfg, schedule):
    if cfg.dtype == "f32" and schedule == "fused":
        pytest.skip("fp32 layers always run the waves schedule")
    inp = make_inputs(cfg)
    got, _, _ = run_cuda(cfg, inp, opts={"schedule": schedule})
    want = oracle.layer_unfused(inp, cfg.h, cfg.causal)
    compare(got, want, tol_for(cfg))


# The fused layer body (one persistent kernel, two query blocks per CTA pair)
# against the wave kernels: the same per-element arithmetic, so bitwise equal.
# Cases: an odd block count (a pair item with one block), ragged sequences in a
# batch (an item whose two blocks belong to different sequences), d and d_ff
# = 64 (mod 128), and more items than CTA pairs (each pair runs several items,
# so every hand-off barrier goes through both phases).
FUSED_CASES = [
    small("fz_odd_blocks", 1, 640, 256, 2, 512, True, seed=51),
    small("fz_ragged_batch", 3, 300, 256, 4, 512, False, seed=52, bias=0.5),
    small("fz_straddle", 1, 260, 192, 3, 448, True, seed=53),
    small("fz_many_items", 1, 128 * 301, 128, 2, 256, True, seed=54),
    small("fz_many_items_batch", 7, 128 * 45 - 3, 256, 2, 320, True, seed=55),
]


@pytest.mark.parametrize("cfg", FUSED_CASES, ids=lambda c: c.name)
def test_fused_schedule_is_bitwise_the_waves_schedule(cfg):
    inp = make_inputs(cfg)
    fused, _, _ = run_cuda(cfg, inp)
    waves, _, _ = run_cuda(cfg, inp, opts={"schedule": "waves"})
    assert np.all(np.isfinite(fused))
    np.testing.assert_array_equal(fused, waves)
    if cfg.B * cfg.N <= 4096:
        compare(fused, oracle.layer_unfused(inp, cfg.h, cfg.causal), tol_for(cfg))
    else:
        rows = sample_rows(cfg, 64)
        compare(fused[rows[:, 0], rows[:, 1]], oracle.layer_rows(inp, cfg.h, cfg.causal, rows),
                tol_for(cfg))


# Items left over after the whole rounds of CTA pairs are shared by two pairs
# when at most half of the pairs would work in the last round (d % 1024 == 0,
# d_ff % 512 == 0): each pair computes half of the item's columns and reads
# the other pair's y and FFN hidden through global memory.  168 blocks = 84
# items on 74 pairs: 10 shared, the last block ragged; 149 blocks: one shared
# item holding a single block; 6 ragged sequences of 37 blocks: 37 shared
# items (the most: every pair works in the last round), one of them (blocks
# 184, 185) across two sequences, d_k = 64.  Bitwise equal to the waves schedule, and held to the oracle on rows of
# the shared items.
SHARED_CASES = [
    small("fz_shared_ragged", 1, 128 * 167 + 78, 1024, 8, 1024, True, seed=56),
    small("fz_shared_one_block", 1, 128 * 149, 1024, 8, 1536, True, seed=57),
    small("fz_shared_most", 6, 128 * 37 - 5, 1024, 16, 1536, False, seed=58, bias=0.5),
]


def shared_item_rows(cfg, pairs=74):
    """(batch, row) pairs in the items past the last whole round of `pairs`
    CTA pairs: the first, a middle and the last row of each of their blocks."""
    nb = (cfg.N + 127) // 128
    blocks = cfg.B * nb
    items = (blocks + 1) // 2
    rows = set()
    for it in range(items // pairs * pairs, items):
        for blk in (2 * it, 2 * it + 1):
            if blk >= blocks:
                continue
            b, pos = divmod(blk, nb)
            lo, hi = pos * 128, min(cfg.N, pos * 128 + 128) - 1
            rows.update((b, r) for r in (lo, (lo + hi) // 2, hi))
    return np.array(sorted(rows), dtype=np.int64)


@pytest.mark.parametrize("cfg", SHARED_CASES, ids=lambda c: c.name)
def test_shared_items_are_bitwise_the_waves_schedule(cfg):
    inp = make_inputs(cfg)
    fused, _, _ = run_cuda(cfg, inp)
    waves, _, _ = run_cuda(cfg, inp, opts={"schedule": "waves"})
    assert np.all(np.isfinite(fused))
    np.testing.assert_array_equal(fused, waves)
    rows = np.unique(np.concatenate([shared_item_rows(cfg), sample_rows(cfg, 16)]), axis=0)
    assert len(rows) > 16
    compare(fused[rows[:, 0], rows[:, 1]], oracle.layer_rows(inp, cfg.h, cfg.causal, rows),
            tol_for(cfg))


@pytest.mark.parametrize("cfg,shared", [(SHARED_CASES[0], 10), (SHARED_CASES[2], 37),
                                        (FUSED_CASES[3], 0)],
                         ids=["10_shared", "37_shared", "none_shared"])
def test_shared_items_hand_over_through_the_header(cfg, shared):
    """The hand-over counters (workspace header bytes [256, 1440), include/bpt.h:
    [kind][pair][CTA rank] uint32, kinds y and H) after a forward: each CTA of
    the 2 * shared pairs that share an item counted its eight epilogue warps
    for both hand-overs, every other entry stayed zero.  So the shared order
    really ran (a refused cooperative launch would leave all zeros)."""
    dev = bpt.to_device(make_inputs(cfg), cfg.dtype)
    _, ws = bpt.layer_forward(dev["x"], dev, cfg.h, cfg.causal)
    st, site = bpt.bpt_read_device_error(ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == bpt.BPT_OK, f"device error {bpt.status_string(st)} at site {site}"
    pairs = bpt.BPT_TAIL_MAX_PAIRS
    flags = ws[256:256 + 2 * pairs * 2 * 4].view(torch.int32).cpu().numpy().reshape(2, pairs, 2)
    want = np.zeros_like(flags)
    want[:, :2 * shared, :] = 8
    np.testing.assert_array_equal(flags, want)


def test_fused_forward_replays_from_a_cuda_graph():
    """A whole forward recorded by stream capture into a CUDA graph (its
    memsets and every launch) replays bitwise equal to the eager call, twice.
    The shape shares left-over items when run eagerly; under capture the layer
    body runs unshared (a plain launch), which gives the same bits."""
    cfg = SHARED_CASES[0]
    dev = bpt.to_device(make_inputs(cfg), cfg.dtype)
    want, ws = bpt.layer_forward(dev["x"], dev, cfg.h, cfg.causal)
    want = want.clone()
    out = torch.empty_like(want)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # first call on this stream outside the capture
        bpt.layer_forward(dev["x"], dev, cfg.h, cfg.causal, out=out, workspace=ws)
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        bpt.layer_forward(dev["x"], dev, cfg.h, cfg.causal, out=out, workspace=ws)
    for _ in range(2):
        out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        st, site = bpt.bpt_read_device_error(ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert st == bpt.BPT_OK, f"device error {bpt.status_string(st)} at site {site}"
        assert torch.equal(out, want)
    del graph


def test_tiny_f32_workload():
    cfg = WORKLOADS["tiny_f32"]
    inp = make_inputs(cfg)
    got, _, _ = run_cuda(cfg, inp)
    compare(got, oracle.layer_unfused(inp, cfg.h, cfg.causal), tol_for(cfg))


@pytest.mark.parametrize("cfg", [SMALL[0], SMALL[2], SMALL[7], SMALL[8]], ids=lambda c: c.name)
def test_qkv_projection_in_workspace(cfg):
    """Step a2 alone: the Q/K/V rows the prologue GEMM wrote (waves schedule,
    which keeps Q)."""
    inp = make_inputs(cfg)
    _, _, ws = run_cuda(cfg, inp, opts={"schedule": "waves"})
    qkv = workspace_qkv(ws, cfg, cfg.B)
    for b in range(cfg.B):
        it = oracle.layer_intermediates(inp, cfg.h, cfg.causal, b=b)
        want = np.concatenate([it["Q"], it["K"], it["V"]], axis=1)
        tol = (1e-4, None) if cfg.dtype == "f32" else (2e-2, 2e-3)
        compare(qkv[b], want, tol)


@pytest.mark.parametrize("cfg", [SMALL[0], SMALL[2], SMALL[7]], ids=lambda c: c.name)
def test_attention_output_over_queries(cfg):
    """Steps a3-a5 alone, fused schedule: each row's attention output o (heads
    concatenated) stands where its Q was; K and V are untouched."""
    inp = make_inputs(cfg)
    _, _, ws = run_cuda(cfg, inp)
    qkv = workspace_qkv(ws, cfg, cfg.B)
    for b in range(cfg.B):
        it = oracle.layer_intermediates(inp, cfg.h, cfg.causal, b=b)
        compare(qkv[b, :, :cfg.d], it["O"], (2e-2, 2e-3))
        compare(qkv[b, :, cfg.d:], np.concatenate([it["K"], it["V"]], axis=1), (2e-2, 2e-3))


@pytest.mark.parametrize("schedule", ["fused", "waves"])
def test_deterministic(schedule):
    cfg = SMALL[0]
    inp = make_inputs(cfg)
    a, _, _ = run_cuda(cfg, inp, opts={"schedule": schedule})
    b, _, _ = run_cuda(cfg, inp, opts={"schedule": schedule})
    np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("schedule", ["fused", "waves"])
def test_several_waves_in_one_sequence(schedule):
    """nb > BPT_WAVE_BLOCKS: the sequence is processed in several waves (or,
    fused, several items per CTA pair)."""
    cfg = small("waves", 1, 128 * 300, 128, 2, 256, True, seed=5)
    inp = make_inputs(cfg)
    got, _, _ = run_cuda(cfg, inp, opts={"schedule": schedule})
    rows = sample_rows(cfg, 96)
    want = oracle.layer_rows(inp, cfg.h, cfg.causal, rows)
    compare(got[rows[:, 0], rows[:, 1]], want, tol_for(cfg))


@pytest.mark.parametrize("schedule", ["fused", "waves"])
def test_several_waves_of_whole_sequences(schedule):
    cfg = small("seqwaves", 5, 128 * 100, 128, 2, 256, True, seed=6)
    inp = make_inputs(cfg)
    got, _, _ = run_cuda(cfg, inp, opts={"schedule": schedule})
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
