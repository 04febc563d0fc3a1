"""bpt_layer_forward_static: the layer for callers that cannot allocate.

Some callers may not allocate device memory at all: plug-ins whose host
framework owns every device buffer and hands out only a call's tensors,
deployments that reserve memory once at start-up, latency-critical loops.
The library gives them one entry point that uses its own fixed-size device
array as the workspace.  These tests call it through the C ABI and check it
against bpt_layer_forward, which takes a caller-allocated workspace and runs
the same kernels: two calls in a row must both give bitwise the same output
(the layer is deterministic), since the second call finds the first call's
leftovers in the shared array.  Device errors recorded in the array's header
are read with bpt_read_device_error(NULL, ...).

This file is collected last on purpose (its name sorts after the others), so a
run that stops at the first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

import blockwise_attn_ffn_b200 as bpt
from blockwise_attn_ffn_b200.inputs import LayerShape, make_inputs


def cfgs():
    return [
        LayerShape("static_bf16", B=2, N=300, d=256, h=2, d_ff=512, causal=True, dtype="bf16",
                   block=128, seed=31, ln_scale=0.1, bias_scale=0.2),
        LayerShape("static_f32", B=1, N=200, d=64, h=1, d_ff=256, causal=False, dtype="f32",
                   block=64, seed=32, ln_scale=0.1),
    ]


def ptrs(dev):
    return [dev[k].data_ptr() for k in ["x"] + bpt.PARAM_NAMES]


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", cfgs(), ids=lambda c: c.name)
def test_static_workspace_matches_caller_workspace(cfg):
    inp = make_inputs(cfg)
    dev = bpt.to_device(inp, cfg.dtype)
    code = bpt.BPT_BF16 if cfg.dtype == "bf16" else bpt.BPT_F32
    stream = torch.cuda.current_stream().cuda_stream
    ref, ws = bpt.layer_forward(dev["x"], dev, cfg.h, cfg.causal)
    torch.cuda.synchronize()
    st, _ = bpt.bpt_read_device_error(ws.data_ptr(), stream)
    assert st == bpt.BPT_OK
    ref = ref.cpu().numpy()
    for call in range(2):
        out = torch.full((cfg.B, cfg.N, cfg.d), float("nan"), dtype=torch.float32, device="cuda")
        st = bpt.bpt_layer_forward_static(*ptrs(dev), cfg.B, cfg.N, cfg.d, cfg.h, cfg.d_ff,
                                          cfg.causal, code, out.data_ptr(), stream)
        assert st == bpt.BPT_OK, bpt.status_string(st)
        st, site = bpt.bpt_read_device_error(None, stream)
        assert st == bpt.BPT_OK, f"call {call}: {bpt.status_string(st)} at site {site}"
        got = out.cpu().numpy()
        assert np.all(np.isfinite(got)), f"call {call}: non-finite output"
        np.testing.assert_array_equal(got, ref, err_msg=f"call {call}")


@pytest.mark.gpu
def test_static_range_error_is_readable_and_the_next_call_is_clean():
    """An input beyond the fp16 range of the tensor-core operands is reported
    through the array's header; the following clean call matches again."""
    cfg = cfgs()[0]
    inp = make_inputs(cfg)
    dev = bpt.to_device(inp, cfg.dtype)
    stream = torch.cuda.current_stream().cuda_stream
    ref, _ = bpt.layer_forward(dev["x"], dev, cfg.h, cfg.causal)
    ref = ref.cpu().numpy()
    big = dict(dev)
    big["W_Q"] = dev["W_Q"].clone()
    big["W_Q"][0, 0] = 1e5          # a bf16 weight no fp16 operand can hold
    out = torch.empty((cfg.B, cfg.N, cfg.d), dtype=torch.float32, device="cuda")
    st = bpt.bpt_layer_forward_static(*ptrs(big), cfg.B, cfg.N, cfg.d, cfg.h, cfg.d_ff,
                                      cfg.causal, bpt.BPT_BF16, out.data_ptr(), stream)
    assert st == bpt.BPT_OK
    st, site = bpt.bpt_read_device_error(None, stream)
    assert st == bpt.BPT_ERR_RANGE, bpt.status_string(st)
    assert site != 0
    st = bpt.bpt_layer_forward_static(*ptrs(dev), cfg.B, cfg.N, cfg.d, cfg.h, cfg.d_ff,
                                      cfg.causal, bpt.BPT_BF16, out.data_ptr(), stream)
    assert st == bpt.BPT_OK
    assert bpt.bpt_read_device_error(None, stream)[0] == bpt.BPT_OK
    np.testing.assert_array_equal(out.cpu().numpy(), ref)


def test_static_workspace_rejects_layers_too_large():
    """Checked on the host before anything is enqueued (no GPU needed)."""
    fake = [0x10000000 + i * 0x1000000 for i in range(12)]
    st = bpt.bpt_layer_forward_static(*fake[:11], 1, 65536, 2048, 16, 8192, 1, bpt.BPT_BF16,
                                      fake[11], None)
    assert st == bpt.BPT_ERR_WORKSPACE
    st_ws, need = bpt.bpt_layer_workspace_size(1, 2048, 768, 12, 3072, 1, bpt.BPT_BF16)
    assert st_ws == bpt.BPT_OK and need <= bpt.BPT_STATIC_WORKSPACE_BYTES


def test_static_workspace_rejects_bad_pointers():
    fake = [0x10000000 + i * 0x1000000 for i in range(12)]
    bad = list(fake)
    bad[3] = None
    assert bpt.bpt_layer_forward_static(*bad[:11], 1, 256, 256, 2, 512, 1, bpt.BPT_BF16,
                                        bad[11], None) == bpt.BPT_ERR_INVALID_ARG
