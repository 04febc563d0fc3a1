"""Full-size checks of the widened rows, by properties that hold at any size.

At the long-context layer (B=1, N=65536, d=2048, h=16, d_ff=8192, causal)
in the launch configuration bench.py times:

* backward ("Blockwise Parallel Transformer — BPT", section "The backward
  pass"): Z = Y + H W_2 + b_2, so d b_2 is the column sum of dZ over every
  row of every wave, whatever the layer's weights; the accumulation over the
  two waves is checked against an fp64 sum of the same dZ.  Every gradient
  is finite, and two calls agree bitwise.
* pairing (one or two query blocks per attention CTA): bitwise equal outputs.
* block gating ("Block Sparse Flash Attention"): thresholds -inf give
  bitwise the dense forward and every visited block pair kept.
"""
import numpy as np
import pytest
import torch

import blockwise_attn_ffn_b200 as bpt
from blockwise_attn_ffn_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

CFG = WORKLOADS["long_n64k"]


@pytest.fixture(scope="module")
def dev():
    return bpt.to_device(make_inputs(CFG), CFG.dtype)


def test_backward_bias_gradient_is_the_upstream_column_sum(dev):
    x = dev["x"]
    _, stats, _ = bpt.layer_forward_train(x, dev, CFG.h, CFG.causal)
    gen = torch.Generator(device="cuda").manual_seed(123)
    dZ = torch.randn(x.shape, generator=gen, device="cuda", dtype=torch.float32)
    g1, ws = bpt.layer_backward(x, dev, CFG.h, CFG.causal, stats, dZ)
    g1 = {k: v.clone() for k, v in g1.items()}
    g2, _ = bpt.layer_backward(x, dev, CFG.h, CFG.causal, stats, dZ, workspace=ws)
    st, site = bpt.bpt_read_device_error(ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == bpt.BPT_OK, f"device error {bpt.status_string(st)} at site {site}"
    for k in g1:
        assert torch.isfinite(g1[k]).all(), k
        assert torch.equal(g1[k], g2[k]), f"{k}: two calls differ"
    want = dZ.double().reshape(-1, CFG.d).sum(0)
    err = (g1["b_2"].double() - want).abs().max().item()
    assert err <= 1e-3 + 1e-5 * want.abs().max().item(), f"d b_2 error {err:.3e}"


def test_pairing_is_bitwise_neutral_at_full_size(dev):
    x = dev["x"]
    out2, ws = bpt.layer_forward(x, dev, CFG.h, CFG.causal)
    out2 = out2.clone()
    out1, _ = bpt.layer_forward(x, dev, CFG.h, CFG.causal, workspace=ws, opts={"attn_block": 128})
    assert torch.equal(out1, out2)


def test_fused_schedule_is_bitwise_the_waves_schedule_at_full_size(dev):
    """The persistent per-block tail and the wave-level kernels run the same
    per-element arithmetic: bitwise equal layer outputs on the workload."""
    x = dev["x"]
    fused, _ = bpt.layer_forward(x, dev, CFG.h, CFG.causal)
    fused = fused.clone()
    waves, _ = bpt.layer_forward(x, dev, CFG.h, CFG.causal, opts={"schedule": "waves"})
    assert torch.isfinite(fused).all()
    assert torch.equal(fused, waves)


def test_gating_without_thresholds_is_the_dense_forward_at_full_size(dev):
    x = dev["x"]
    nb = (CFG.N + 127) // 128
    dense, ws = bpt.layer_forward(x, dev, CFG.h, CFG.causal)
    dense = dense.clone()
    T = torch.full((CFG.h, nb), float("-inf"), dtype=torch.float32, device="cuda")
    out, _, kept, _ = bpt.layer_forward_bsfa(x, dev, CFG.h, CFG.causal, T, kept=True,
                                             workspace=ws)
    assert torch.equal(out, dense)
    vis = torch.tril(torch.ones(nb, nb, dtype=torch.uint8, device="cuda"))
    assert torch.equal(kept[0], vis.expand(CFG.h, nb, nb))
