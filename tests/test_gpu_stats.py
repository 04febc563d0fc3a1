"""Per-row softmax statistics of bpt_layer_forward_train against the oracle.

BPT page, section "The backward pass": the forward keeps (m, l) per row.  The
CUDA path writes stats[b, t, i] = (m, l) with m the row's maximum score
q.k/sqrt(d_k) over its allowed keys and l = sum exp(s - m).

Tolerances.  fp32 layers: 1e-4 like the layer output.  bf16 layers: Q and K
reach the tensor cores as fp16 values after two fp16 roundings (LN output and
projection result, relative 2^-11 each), so a score carries
|ds| <~ 2 * 2^-10 * |q||k| / sqrt(d_k) ~ 0.02 for unit-scale q, k at
d_k <= 128: m and m + log l are held to 3e-2 (+ 0.3 % of |m| for large
scores); l = sum exp(s_j - m) inherits a relative error of at most twice that
of the scores, held to 5e-2.
"""
import numpy as np
import pytest
import torch

import blockwise_attn_ffn_b200 as bpt
import oracle
from blockwise_attn_ffn_b200.inputs import WORKLOADS, make_inputs, sample_rows
from gpu_util import run_cuda
from test_gpu_parity import SMALL

pytestmark = pytest.mark.gpu


def run_train(cfg, inp):
    dev = bpt.to_device(inp, cfg.dtype)
    out, stats, ws = bpt.layer_forward_train(dev["x"], dev, cfg.h, cfg.causal)
    st, site = bpt.bpt_read_device_error(ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == bpt.BPT_OK, f"device error {bpt.status_string(st)} at site {site}"
    return out.cpu().numpy(), stats.cpu().numpy()


def check_stats(cfg, stats, inp, rows):
    """stats [B, h, N, 2] from the GPU at the given (batch, row) pairs."""
    m_ref, l_ref = oracle.attention_stats_rows(inp, cfg.h, cfg.causal, rows)
    got = stats[rows[:, 0], :, rows[:, 1], :]          # [len(rows), h, 2]
    m, l = got[..., 0].astype(np.float64), got[..., 1].astype(np.float64)
    assert np.all(np.isfinite(m)) and np.all(np.isfinite(l))
    if cfg.dtype == "f32":
        a_m, r_m, r_l = 1e-4, 0.0, 1e-4
    else:
        a_m, r_m, r_l = 3e-2, 3e-3, 5e-2
    dm = np.abs(m - m_ref)
    assert np.all(dm <= a_m + r_m * np.abs(m_ref)), f"m: max abs err {dm.max():.3e}"
    dl = np.abs(l - l_ref) / l_ref
    assert np.all(dl <= r_l), f"l: max rel err {dl.max():.3e}"
    lse, lse_ref = m + np.log(l), m_ref + np.log(l_ref)
    dlse = np.abs(lse - lse_ref)
    assert np.all(dlse <= a_m + r_m * np.abs(lse_ref)), f"lse: max abs err {dlse.max():.3e}"
    return float(dm.max()), float(dl.max()), float(dlse.max())


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_small_layers_stats_all_rows(cfg):
    inp = make_inputs(cfg)
    out_t, stats = run_train(cfg, inp)
    rows = np.array([(b, i) for b in range(cfg.B) for i in range(cfg.N)], dtype=np.int64)
    check_stats(cfg, stats, inp, rows)
    # the training entry point returns the same layer output, bit for bit
    out_f, _, _ = run_cuda(cfg, inp)
    np.testing.assert_array_equal(out_t, out_f)


@pytest.mark.parametrize("name", ["gpt2s_n2k", "mid_n16k", "long_n64k"])
def test_workload_stats_sampled_rows(name):
    cfg = WORKLOADS[name]
    inp = make_inputs(cfg)
    _, stats = run_train(cfg, inp)
    rows = sample_rows(cfg, 64)
    check_stats(cfg, stats, inp, rows)


def test_train_entry_rejects_null_and_overlapping_stats():
    cfg = SMALL[0]
    inp = make_inputs(cfg)
    dev = bpt.to_device(inp, cfg.dtype)
    B, N, d = dev["x"].shape
    out = torch.empty((B, N, d), dtype=torch.float32, device="cuda")
    ws = bpt.workspace_for(B, N, d, cfg.h, cfg.d_ff, cfg.causal, dev["x"].dtype, dev["x"].device)
    ptrs = [dev["x"].data_ptr()] + [dev[k].data_ptr() for k in bpt.PARAM_NAMES]
    s = torch.cuda.current_stream().cuda_stream
    code = bpt.BPT_BF16 if cfg.dtype == "bf16" else bpt.BPT_F32
    args = ptrs + [B, N, d, cfg.h, cfg.d_ff, cfg.causal, code, out.data_ptr()]
    st = bpt.bpt_layer_forward_train(*args, 0, ws.data_ptr(), ws.numel(), s)
    assert st == bpt.BPT_ERR_INVALID_ARG
    st = bpt.bpt_layer_forward_train(*args, out.data_ptr(), ws.data_ptr(), ws.numel(), s)
    assert st == bpt.BPT_ERR_INVALID_ARG
