"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
and compare with the fp64 oracle."""
from __future__ import annotations

import json
import os

import numpy as np
import torch

import blockwise_attn_ffn_b200 as bpt
from blockwise_attn_ffn_b200.inputs import LayerShape, make_inputs

# Tolerances (max abs, mean abs) against the fp64 oracle.
TOL_F32 = (1e-4, None)
TOL_BF16 = (2e-2, 2e-3)


def tol_for(cfg: LayerShape):
    return TOL_F32 if cfg.dtype == "f32" else TOL_BF16


def run_cuda(cfg: LayerShape, inp=None, B=None, opts=None):
    """One forward through bpt_layer_forward (bpt_layer_forward_opt with
    ``opts``); returns (Z float32 numpy, dev, ws)."""
    if inp is None:
        inp = make_inputs(cfg, B=B)
    dev = bpt.to_device(inp, cfg.dtype)
    x = dev["x"]
    out, ws = bpt.layer_forward(x, dev, cfg.h, cfg.causal, opts=opts)
    st, site = bpt.bpt_read_device_error(ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == bpt.BPT_OK, f"device error {bpt.status_string(st)} at site {site}"
    return out.float().cpu().numpy(), dev, ws


def compare(got: np.ndarray, want: np.ndarray, tol):
    err = np.abs(got.astype(np.float64) - want)
    assert np.all(np.isfinite(got)), "non-finite values in the CUDA result"
    mx, mean = float(err.max()), float(err.mean())
    msg = f"max abs {mx:.3e} (tol {tol[0]}), mean abs {mean:.3e} (tol {tol[1]})"
    log = os.environ.get("BPT_PARITY_LOG")
    if log:
        with open(log, "a") as f:
            f.write(json.dumps({"test": os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0],
                                "n": int(err.size), "max_abs": mx, "mean_abs": mean,
                                "tol": list(tol)}) + "\n")
    assert mx <= tol[0], msg
    if tol[1] is not None:
        assert mean <= tol[1], msg
    return mx, mean


def workspace_qkv(ws: torch.Tensor, cfg: LayerShape, B: int) -> np.ndarray:
    """The QKV projection the library leaves in its workspace ([B*N, 3d]).

    Layout (include/bpt.h): a 2048-byte header region (error word, hand-over
    counters), then for bf16 layers the fp16 weight copies, then QKV in the
    operand type (fp16 / fp32).
    """
    off = 2048
    n = B * cfg.N * 3 * cfg.d
    if cfg.dtype == "bf16":
        w16 = (4 * cfg.d * cfg.d + 2 * cfg.d * cfg.d_ff) * 2
        off += (w16 + 1023) // 1024 * 1024
        t = ws[off:off + 2 * n].view(torch.float16)
    else:
        t = ws[off:off + 4 * n].view(torch.float32)
    return t.float().cpu().numpy().reshape(B, cfg.N, 3 * cfg.d)
