"""Query rows sharing each K/V tile: one 128-row block per CTA (b = 128), two
blocks per CTA (b = 256, the default) and a cluster of two such CTAs that
exchange K/V halves over DSMEM (b = 512) (bpt_options.attn_qpc = 1, 2, 4).

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
]


def forward_train(cfg, dev, opts):
    out, stats, ws = bpt.layer_forward_train(dev["x"], dev, cfg.h, cfg.causal, opts=opts)
    st, site = bpt.bpt_read_device_error(ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == bpt.BPT_OK, f"device error {bpt.status_string(st)} at site {site}"
    return out.cpu().numpy(), stats.cpu().numpy()


@pytest.mark.parametrize("schedule", ["fused", "waves"])
@pytest.mark.parametrize("cfg,wave", CASES, ids=lambda c: getattr(c, "name", str(c)))
def test_block_sharing_is_bitwise_neutral(cfg, wave, schedule):
    """One 128-row block per CTA (b = 128), two (b = 256, default) and a
    cluster of two CTAs sharing each K/V tile over DSMEM (b = 512): the same
    layer output and statistics, bit for bit."""
    dev = bpt.to_device(make_inputs(cfg), cfg.dtype)
    base = {"schedule": schedule, "max_wave": wave if schedule == "waves" else 0}
    out2, st2 = forward_train(cfg, dev, dict(base, attn_qpc=2))
    out1, st1 = forward_train(cfg, dev, dict(base, attn_qpc=1))
    out4, st4 = forward_train(cfg, dev, dict(base, attn_qpc=4))
    assert np.all(np.isfinite(out2))
    np.testing.assert_array_equal(out1, out2)
    np.testing.assert_array_equal(st1, st2)
    np.testing.assert_array_equal(out4, out2)
    np.testing.assert_array_equal(st4, st2)


def test_b512_backward_recomputation_matches():
    """The backward's forward recomputation through the b = 512 attention
    gives the same gradients as through the default one."""
    cfg = CASES[0][0]
    inp = make_inputs(cfg)
    dev = bpt.to_device(inp, cfg.dtype)
    _, stats, _ = bpt.layer_forward_train(dev["x"], dev, cfg.h, cfg.causal)
    dZ = torch.from_numpy(np.random.default_rng(3).standard_normal(
        (cfg.B, cfg.N, cfg.d)).astype(np.float32)).cuda()
    g2, _ = bpt.layer_backward(dev["x"], dev, cfg.h, cfg.causal, stats, dZ)
    g4, _ = bpt.layer_backward(dev["x"], dev, cfg.h, cfg.causal, stats, dZ,
                               opts={"attn_qpc": 4})
    for k in g2:
        assert torch.equal(g2[k], g4[k]), k


def test_b512_rejects_gating():
    cfg = CASES[0][0]
    dev = bpt.to_device(make_inputs(cfg), cfg.dtype)
    nb = (cfg.N + 127) // 128
    T = torch.full((cfg.h, nb), float("-inf"), dtype=torch.float32, device="cuda")
    with pytest.raises(bpt.BptError):
        bpt.layer_forward_bsfa(dev["x"], dev, cfg.h, cfg.causal, T, opts={"attn_qpc": 4})


def test_qpc_rejects_other_values():
    for bad in (3, 5, -1):
        st, _ = bpt.bpt_layer_workspace_size_opt(1, 256, 256, 2, 512, True, bpt.BPT_BF16,
                                                 {"attn_qpc": bad})
        assert st == bpt.BPT_ERR_INVALID_ARG
