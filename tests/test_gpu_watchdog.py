"""Failure detection on the GPU without a GPU fault.

A test hook makes one CTA skip one TMA load, so the consumer's bounded wait
runs out (about 2 s) instead of completing.  The kernel must record
BPT_ERR_TIMEOUT in the device error word, drain what it issued, free its
tensor memory and exit; the host reads the status, and the next forward on
the same context is correct again.
"""
import numpy as np
import pytest
import torch

import blockwise_attn_ffn_b200 as bpt
import oracle
from blockwise_attn_ffn_b200.inputs import LayerShape, make_inputs

from gpu_util import compare, run_cuda, tol_for

pytestmark = pytest.mark.gpu

CFG = LayerShape("watchdog", B=1, N=512, d=256, h=2, d_ff=512, causal=True, dtype="bf16",
                 block=128, seed=41, ln_scale=0.1)


@pytest.mark.parametrize("code,schedule", [(1, "fused"), (2, "fused"), (3, "fused"),
                                           (2, "waves")],
                         ids=["gemm_lost_stage", "attention_lost_v", "tail_lost_stage",
                              "waves_attention_lost_v"])
def test_lost_arrive_reports_timeout_and_context_survives(code, schedule):
    inp = make_inputs(CFG)
    dev = bpt.to_device(inp, CFG.dtype)
    stream = torch.cuda.current_stream().cuda_stream
    opts = {"schedule": schedule, "fault": code}
    out, ws = bpt.layer_forward(dev["x"], dev, CFG.h, CFG.causal, opts=opts)
    st, site = bpt.bpt_read_device_error(ws.data_ptr(), stream)
    assert st == bpt.BPT_ERR_TIMEOUT, bpt.status_string(st)
    assert site != 0
    # the same context keeps working: a clean forward matches the oracle
    got, _, _ = run_cuda(CFG, inp)
    compare(got, oracle.layer_unfused(inp, CFG.h, CFG.causal), tol_for(CFG))


def test_fault_hook_rejects_unknown_codes():
    for bad in (7, -1):
        st, _ = bpt.bpt_layer_workspace_size_opt(1, 512, 256, 2, 512, True, bpt.BPT_BF16,
                                                 {"fault": bad})
        assert st == bpt.BPT_ERR_INVALID_ARG
