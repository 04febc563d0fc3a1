"""Query rows sharing each K/V tile (bpt_options.attn_block = b): one 64-row
block per CTA, two CTAs per SM (b = 64), one 128-row block per CTA
(b = 128), two blocks per CTA (b = 256, the default) and a cluster of two
such CTAs that exchange K/V halves over DSMEM (b = 512).

"Blockwise Parallel Transformer — BPT", section "Choosing the block size:
arithmetic intensity": the work done per byte re-read grows with the rows
that share it.  Pairing changes only which CTA computes a query block, not
its arithmetic, so the two settings must give bitwise equal layer outputs and
softmax statistics; the paired output is itself held to the oracle by the
parity tests.  Cases cover odd block counts (a pair without its second
block), ragged tails, both wave layouts (part of one sequence, whole
sequences) and both head widths.
"""
import numpy as np
import pytest
import torch

import blockwise_attn_ffn_b200 as bpt
from blockwise_attn_ffn_b200.inputs import make_inputs
from test_gpu_parity import small

pytestmark = pytest.mark.gpu

CASES = [
    (small("qpc_dk128_causal_odd", 1, 640, 256, 2, 512, True, seed=41), 0),
    (small("qpc_dk64_noncausal_ragged", 2, 300, 256, 4, 512, False, seed=42), 0),
    (small("qpc_dk128_split_sequence", 1, 900, 256, 2, 512, True, seed=43), 3),
    (small("qpc_dk64_whole_sequences", 3, 256, 256, 4, 512, True, seed=44), 2),
    (small("qpc_dk64_causal_ragged_half", 2, 700, 256, 4, 512, True, seed=45), 0),
    (small("qpc_dk128_noncausal_short", 2, 60, 256, 2, 512, False, seed=46), 0),
]


def forward_train(cfg, dev, opts):
    out, stats, ws = bpt.layer_forward_train(dev["x"], dev, cfg.h, cfg.causal, opts=opts)
    st, site = bpt.bpt_read_device_error(ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == bpt.BPT_OK, f"device error {bpt.status_string(st)} at site {site}"
    return out.cpu().numpy(), stats.cpu().numpy()


@pytest.mark.parametrize("schedule", ["fused", "waves"])
@pytest.mark.parametrize("cfg,wave", CASES, ids=lambda c: getattr(c, "name", str(c)))
def test_block_sharing_is_bitwise_neutral(cfg, wave, schedule):
    """b = 64, 128, 256 (default) and 512: the same layer output and softmax
    statistics, bit for bit."""
    dev = bpt.to_device(make_inputs(cfg), cfg.dtype)
    base = {"schedule": schedule, "max_wave": wave if schedule == "waves" else 0}
    out_ref, st_ref = forward_train(cfg, dev, dict(base, attn_block=256))
    assert np.all(np.isfinite(out_ref))
    for b in (64, 128, 512):
        out, st = forward_train(cfg, dev, dict(base, attn_block=b))
        np.testing.assert_array_equal(out, out_ref, err_msg=f"b = {b}")
        np.testing.assert_array_equal(st, st_ref, err_msg=f"b = {b}")


@pytest.mark.parametrize("b", [64, 512])
def test_backward_recomputation_matches(b):
    """The backward's forward recomputation through the b = 64 and b = 512
    attention kernels gives the same gradients as through the default one."""
    cfg = CASES[0][0]
    inp = make_inputs(cfg)
    dev = bpt.to_device(inp, cfg.dtype)
    _, stats, _ = bpt.layer_forward_train(dev["x"], dev, cfg.h, cfg.causal)
    dZ = torch.from_numpy(np.random.default_rng(3).standard_normal(
        (cfg.B, cfg.N, cfg.d)).astype(np.float32)).cuda()
    g_ref, _ = bpt.layer_backward(dev["x"], dev, cfg.h, cfg.causal, stats, dZ)
    g, _ = bpt.layer_backward(dev["x"], dev, cfg.h, cfg.causal, stats, dZ,
                              opts={"attn_block": b})
    for k in g_ref:
        assert torch.equal(g_ref[k], g[k]), k


@pytest.mark.parametrize("b", [64, 512])
def test_dense_only_block_sizes_reject_gating(b):
    cfg = CASES[0][0]
    dev = bpt.to_device(make_inputs(cfg), cfg.dtype)
    nb = (cfg.N + 127) // 128
    T = torch.full((cfg.h, nb), float("-inf"), dtype=torch.float32, device="cuda")
    with pytest.raises(bpt.BptError):
        bpt.layer_forward_bsfa(dev["x"], dev, cfg.h, cfg.causal, T, opts={"attn_block": b})


def test_attn_block_rejects_other_values():
    for bad in (1, 2, 4, 32, 192, 1024, -1):
        st, _ = bpt.bpt_layer_workspace_size_opt(1, 256, 256, 2, 512, True, bpt.BPT_BF16,
                                                 {"attn_block": bad})
        assert st == bpt.BPT_ERR_INVALID_ARG


@pytest.mark.parametrize("cfg,wave", [CASES[0], CASES[1], CASES[3]],
                         ids=lambda c: getattr(c, "name", str(c)))
def test_kept_attention_output_is_block_size_neutral(cfg, wave):
    """bpt_layer_forward_train_keep_o with every block size: the same output,
    statistics and kept attention output, bit for bit (each kernel writes o
    to the caller's buffer through the same row-stride override)."""
    dev = bpt.to_device(make_inputs(cfg), cfg.dtype)
    got = {}
    for b in (256, 64, 128, 512):
        o = torch.full((cfg.B, cfg.N, cfg.d), float("nan"), dtype=torch.float16, device="cuda")
        out, stats, ws = bpt.layer_forward_train(dev["x"], dev, cfg.h, cfg.causal,
                                                 opts={"attn_block": b}, keep_o=o)
        st, site = bpt.bpt_read_device_error(ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert st == bpt.BPT_OK, f"b = {b}: {bpt.status_string(st)} at site {site}"
        got[b] = (out.cpu().numpy(), stats.cpu().numpy(), o.float().cpu().numpy())
    assert np.all(np.isfinite(got[256][2]))
    for b in (64, 128, 512):
        for k, name in enumerate(("out", "stats", "o")):
            np.testing.assert_array_equal(got[b][k], got[256][k], err_msg=f"b = {b}: {name}")
