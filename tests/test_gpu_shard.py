"""Sequence sharding on the GPU: G ranks run one after another on one GPU
(every call here has a single GPU; the all-gather is replaced by stacking
the ranks' K | V in rank order, which is what the collective produces).

"Blockwise Parallel Transformer — BPT", section "BPT and Ring Attention".
Each rank's rows go through bpt_layer_shard_project and
bpt_layer_shard_forward; the reassembled output must equal bitwise the
unsharded bpt_layer_forward (the same per-element arithmetic: LN1 and the
projection act per row, every query block sees the same K/V tiles in the
same order, the layer body acts per row), and the oracle within the layer
tolerance.
"""
import numpy as np
import pytest
import torch

import blockwise_attn_ffn_b200 as bpt
import oracle
from blockwise_attn_ffn_b200 import shard
from blockwise_attn_ffn_b200.inputs import make_inputs, sample_rows
from gpu_util import compare, tol_for
from test_gpu_parity import small

pytestmark = pytest.mark.gpu

CASES = [
    (small("shard_g2_dk128_causal", 1, 1024, 256, 2, 512, True, seed=61), 2),
    (small("shard_g4_dk64_causal_batch", 2, 2048, 256, 4, 512, True, seed=62, bias=0.5), 4),
    (small("shard_g2_noncausal", 1, 1024, 256, 2, 512, False, seed=63), 2),
    (small("shard_g8_long", 1, 128 * 96, 256, 2, 512, True, seed=64), 8),
    (small("shard_g1", 1, 512, 192, 3, 448, True, seed=65), 1),
]


def run_sharded(cfg, dev, G):
    x = dev["x"]
    B, N, d = x.shape
    parts = []
    for r in range(G):
        rows = torch.from_numpy(shard.token_rows(N, G, r)).cuda()
        x_loc = x[:, rows].contiguous()
        kv_loc, out, ws = shard.project(x_loc, dev, cfg.h, cfg.causal, N, G, r)
        parts.append((rows, x_loc, kv_loc.clone(), out, ws))
    kv_all = torch.stack([p[2] for p in parts])       # the all-gather's result
    z = torch.empty((B, N, d), dtype=torch.float32, device="cuda")
    for r, (rows, x_loc, _, out, ws) in enumerate(parts):
        shard.forward(x_loc, dev, cfg.h, cfg.causal, N, G, r, kv_all, out, ws)
        st, site = bpt.bpt_read_device_error(ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert st == bpt.BPT_OK, f"rank {r}: {bpt.status_string(st)} at site {site}"
        z[:, rows] = out
    return z


@pytest.mark.parametrize("cfg,G", CASES, ids=lambda c: getattr(c, "name", str(c)))
def test_sharded_forward_is_bitwise_the_single_gpu_forward(cfg, G):
    inp = make_inputs(cfg)
    dev = bpt.to_device(inp, cfg.dtype)
    full, _ = bpt.layer_forward(dev["x"], dev, cfg.h, cfg.causal)
    z = run_sharded(cfg, dev, G)
    assert torch.isfinite(z).all()
    assert torch.equal(z, full)
    got = z.cpu().numpy()
    if cfg.B * cfg.N <= 4096:
        compare(got, oracle.layer_unfused(inp, cfg.h, cfg.causal), tol_for(cfg))
    else:
        rows = sample_rows(cfg, 64)
        compare(got[rows[:, 0], rows[:, 1]], oracle.layer_rows(inp, cfg.h, cfg.causal, rows),
                tol_for(cfg))


def test_shard_kv_is_the_projection_of_the_rank_rows():
    """Step 1 alone: kv_loc holds K | V of the rank's own rows."""
    cfg, G = CASES[0]
    inp = make_inputs(cfg)
    dev = bpt.to_device(inp, cfg.dtype)
    it = oracle.layer_intermediates(inp, cfg.h, cfg.causal)
    for r in range(G):
        rows = shard.token_rows(cfg.N, G, r)
        x_loc = dev["x"][:, torch.from_numpy(rows).cuda()].contiguous()
        kv_loc, _, _ = shard.project(x_loc, dev, cfg.h, cfg.causal, cfg.N, G, r)
        want = np.concatenate([it["K"], it["V"]], axis=1)[rows]
        compare(kv_loc[0].float().cpu().numpy(), want, (2e-2, 2e-3))


def test_shard_rejects_bad_arguments():
    cfg, G = CASES[0]
    dev = bpt.to_device(make_inputs(cfg), cfg.dtype)
    x_loc = dev["x"][:, :cfg.N // G].contiguous()
    ptrs = [x_loc.data_ptr()] + [dev[k].data_ptr() for k in bpt.PARAM_NAMES]
    kv = torch.empty((1, cfg.N // G, 2 * cfg.d), dtype=torch.float16, device="cuda")
    out = torch.empty((1, cfg.N // G, cfg.d), dtype=torch.float32, device="cuda")
    ws = shard.workspace_for(1, cfg.N, G, cfg.d, cfg.h, cfg.d_ff, True, "cuda")
    args = lambda N, G_, r: (*ptrs, 1, N, G_, r, cfg.d, cfg.h, cfg.d_ff, 1, bpt.BPT_BF16,
                             kv.data_ptr(), out.data_ptr(), ws.data_ptr(), ws.numel(), None)
    assert bpt.bpt_layer_shard_project(*args(cfg.N, G, G)) == bpt.BPT_ERR_INVALID_ARG
    assert bpt.bpt_layer_shard_project(*args(cfg.N, 0, 0)) == bpt.BPT_ERR_INVALID_ARG
    assert bpt.bpt_layer_shard_project(*args(cfg.N + 128, G, 0)) == bpt.BPT_ERR_UNSUPPORTED
    bad = list(args(cfg.N, G, 0))
    bad[20] = out.data_ptr()                          # kv over out
    assert bpt.bpt_layer_shard_project(*bad) == bpt.BPT_ERR_INVALID_ARG
