"""torch-tensor front end of ``bpt_layer_forward`` (marshalling only).

PyTorch provides device memory and the stream; the layer itself runs in
libbpt's kernels.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch

from . import _lib

# Parameter tensors in C-ABI order, with their shapes in terms of (d, d_ff).
PARAM_NAMES = ["ln1", "W_Q", "W_K", "W_V", "W_O", "ln2", "W_1", "b_1", "W_2", "b_2"]


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return _lib.BPT_BF16
    if t.dtype == torch.float32:
        return _lib.BPT_F32
    raise TypeError(f"x must be bfloat16 or float32, got {t.dtype}")


def to_device(inp: Dict[str, np.ndarray], dtype: str, device="cuda",
              pin_x: bool = False) -> Dict[str, torch.Tensor]:
    """Moves generator output (``inputs.make_inputs``) to device tensors.

    bf16 tensors are rebuilt from their exact bit patterns.  LN parameters
    are packed as [2, d] (gamma; beta).  With ``pin_x`` the input x stays in
    pinned host memory (for end-to-end timing, which copies it each step).
    """
    def conv(name):
        if dtype == "bf16":
            a = torch.from_numpy(np.ascontiguousarray(inp[name + "_bits"]).view(np.int16))
            return a.view(torch.bfloat16)
        return torch.from_numpy(np.ascontiguousarray(inp[name], dtype=np.float32))

    out = {}
    x = conv("x")
    out["x"] = x.pin_memory() if pin_x else x.to(device)
    for k in ("W_Q", "W_K", "W_V", "W_O", "W_1", "b_1", "W_2", "b_2"):
        out[k] = conv(k).to(device)
    out["ln1"] = torch.stack([conv("gamma1"), conv("beta1")]).to(device)
    out["ln2"] = torch.stack([conv("gamma2"), conv("beta2")]).to(device)
    return out


def workspace_for(B: int, N: int, d: int, h: int, d_ff: int, causal: bool,
                  dtype: torch.dtype, device="cuda", opts=None) -> torch.Tensor:
    """Allocates (through torch) a workspace of the size the library asks for
    (``opts``: None, an ``Options`` or a dict of its fields)."""
    code = _lib.BPT_BF16 if dtype == torch.bfloat16 else _lib.BPT_F32
    st, nbytes = _lib.bpt_layer_workspace_size_opt(B, N, d, h, d_ff, causal, code, opts)
    if st != _lib.BPT_OK:
        raise _lib.BptError(st, "bpt_layer_workspace_size")
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def layer_forward(x: torch.Tensor, p: Dict[str, torch.Tensor], h: int, causal: bool,
                  out: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None,
                  stream: Optional[torch.cuda.Stream] = None, opts=None):
    """Z = BPT layer(x) via ``bpt_layer_forward`` (``bpt_layer_forward_opt``
    when ``opts`` is given); returns (out, workspace).

    x: [B, N, d] bf16 or fp32 on the GPU; p: ``PARAM_NAMES`` tensors of the
    same dtype (ln1/ln2 as [2, d]); out: [B, N, d] fp32; opts: None, an
    ``Options`` or a dict of its fields (schedule, attn_block, max_wave, fault).
    """
    if x.dim() != 3:
        raise ValueError("x must be [B, N, d]")
    B, N, d = x.shape
    d_ff = p["W_1"].shape[1]
    code = _dtype_code(x)
    tensors = [x] + [p[k] for k in PARAM_NAMES]
    for t in tensors:
        if not t.is_cuda or not t.is_contiguous() or t.dtype != x.dtype:
            raise ValueError("inputs must be contiguous CUDA tensors of one dtype")
    if out is None:
        out = torch.empty((B, N, d), dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = workspace_for(B, N, d, h, d_ff, causal, x.dtype, x.device, opts)
    s = stream if stream is not None else torch.cuda.current_stream(x.device)
    if opts is None:
        st = _lib.bpt_layer_forward(*[t.data_ptr() for t in tensors], B, N, d, h, d_ff, causal,
                                    code, out.data_ptr(), workspace.data_ptr(),
                                    workspace.numel(), s.cuda_stream)
    else:
        st = _lib.bpt_layer_forward_opt(*[t.data_ptr() for t in tensors], B, N, d, h, d_ff,
                                        causal, code, out.data_ptr(), None,
                                        workspace.data_ptr(), workspace.numel(), opts,
                                        s.cuda_stream)
    if st != _lib.BPT_OK:
        raise _lib.BptError(st, "bpt_layer_forward")
    return out, workspace


def layer_forward_train(x: torch.Tensor, p: Dict[str, torch.Tensor], h: int, causal: bool,
                        out: Optional[torch.Tensor] = None,
                        stats: Optional[torch.Tensor] = None,
                        workspace: Optional[torch.Tensor] = None,
                        stream: Optional[torch.cuda.Stream] = None, opts=None,
                        keep_o: Optional[torch.Tensor] = None):
    """``layer_forward`` that also returns the per-row softmax statistics via
    ``bpt_layer_forward_train``: (out, stats, workspace), stats [B, h, N, 2]
    fp32 holding (m, l) per (batch, head, query row).  With ``keep_o`` (an
    fp16 [B, N, d] tensor, bf16 layers) the attention output is kept there
    too (``bpt_layer_forward_train_keep_o``), for ``layer_backward(o=...)``."""
    if x.dim() != 3:
        raise ValueError("x must be [B, N, d]")
    B, N, d = x.shape
    d_ff = p["W_1"].shape[1]
    code = _dtype_code(x)
    tensors = [x] + [p[k] for k in PARAM_NAMES]
    for t in tensors:
        if not t.is_cuda or not t.is_contiguous() or t.dtype != x.dtype:
            raise ValueError("inputs must be contiguous CUDA tensors of one dtype")
    if out is None:
        out = torch.empty((B, N, d), dtype=torch.float32, device=x.device)
    if stats is None:
        stats = torch.empty((B, h, N, 2), dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = workspace_for(B, N, d, h, d_ff, causal, x.dtype, x.device, opts)
    s = stream if stream is not None else torch.cuda.current_stream(x.device)
    if keep_o is not None:
        if (keep_o.dtype != torch.float16 or tuple(keep_o.shape) != (B, N, d)
                or not keep_o.is_contiguous()):
            raise ValueError(f"keep_o must be a contiguous fp16 [{B}, {N}, {d}] tensor")
        st = _lib.bpt_layer_forward_train_keep_o(*[t.data_ptr() for t in tensors], B, N, d, h,
                                                 d_ff, causal, code, out.data_ptr(),
                                                 stats.data_ptr(), keep_o.data_ptr(),
                                                 workspace.data_ptr(), workspace.numel(), opts,
                                                 s.cuda_stream)
    elif opts is None:
        st = _lib.bpt_layer_forward_train(*[t.data_ptr() for t in tensors], B, N, d, h, d_ff,
                                          causal, code, out.data_ptr(), stats.data_ptr(),
                                          workspace.data_ptr(), workspace.numel(), s.cuda_stream)
    else:
        st = _lib.bpt_layer_forward_opt(*[t.data_ptr() for t in tensors], B, N, d, h, d_ff,
                                        causal, code, out.data_ptr(), stats.data_ptr(),
                                        workspace.data_ptr(), workspace.numel(), opts,
                                        s.cuda_stream)
    if st != _lib.BPT_OK:
        raise _lib.BptError(st, "bpt_layer_forward_train")
    return out, stats, workspace


def layer_forward_bsfa(x: torch.Tensor, p: Dict[str, torch.Tensor], h: int, causal: bool,
                       thresholds: torch.Tensor, block_max: bool = False, kept: bool = False,
                       out: Optional[torch.Tensor] = None,
                       workspace: Optional[torch.Tensor] = None,
                       stream: Optional[torch.cuda.Stream] = None, opts=None):
    """``layer_forward`` with block-gated attention via ``bpt_layer_forward_bsfa``.

    thresholds: fp32 CUDA tensor [h, nb], nb = ceil(N / 128).  Returns
    (out, block_max or None, kept or None, workspace); block_max [B, h, nb, nb]
    fp32 and kept [B, h, nb, nb] uint8 are allocated when requested and hold
    -inf / 0 where a causal mask visits no pair."""
    if x.dim() != 3:
        raise ValueError("x must be [B, N, d]")
    B, N, d = x.shape
    d_ff = p["W_1"].shape[1]
    nb = (N + 127) // 128
    code = _dtype_code(x)
    tensors = [x] + [p[k] for k in PARAM_NAMES]
    for t in tensors:
        if not t.is_cuda or not t.is_contiguous() or t.dtype != x.dtype:
            raise ValueError("inputs must be contiguous CUDA tensors of one dtype")
    if (not thresholds.is_cuda or thresholds.dtype != torch.float32
            or tuple(thresholds.shape) != (h, nb) or not thresholds.is_contiguous()):
        raise ValueError(f"thresholds must be a contiguous fp32 CUDA tensor [{h}, {nb}]")
    bm = (torch.full((B, h, nb, nb), float("-inf"), dtype=torch.float32, device=x.device)
          if block_max else None)
    kp = torch.zeros((B, h, nb, nb), dtype=torch.uint8, device=x.device) if kept else None
    if out is None:
        out = torch.empty((B, N, d), dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = workspace_for(B, N, d, h, d_ff, causal, x.dtype, x.device, opts)
    s = stream if stream is not None else torch.cuda.current_stream(x.device)
    st = _lib.bpt_layer_forward_bsfa_opt(*[t.data_ptr() for t in tensors], B, N, d, h, d_ff,
                                         causal, code, thresholds.data_ptr(),
                                         bm.data_ptr() if bm is not None else None,
                                         kp.data_ptr() if kp is not None else None,
                                         out.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                         opts, s.cuda_stream)
    if st != _lib.BPT_OK:
        raise _lib.BptError(st, "bpt_layer_forward_bsfa")
    return out, bm, kp, workspace


GRAD_SHAPES = ["x", "ln1", "W_Q", "W_K", "W_V", "W_O", "ln2", "W_1", "b_1", "W_2", "b_2"]


def layer_backward(x: torch.Tensor, p: Dict[str, torch.Tensor], h: int, causal: bool,
                   stats: torch.Tensor, dZ: torch.Tensor,
                   workspace: Optional[torch.Tensor] = None,
                   stream: Optional[torch.cuda.Stream] = None, opts=None,
                   o: Optional[torch.Tensor] = None):
    """Gradients via ``bpt_layer_backward``; returns (grads, workspace) with
    grads[name] fp32 for name in GRAD_SHAPES (ln1 / ln2 as [2, d]: d gamma;
    d beta).  x and p as for ``layer_forward`` (bf16 or fp32); stats from
    ``layer_forward_train``; dZ [B, N, d] fp32.  ``o``: the attention output
    ``layer_forward_train(keep_o=...)`` kept (``bpt_layer_backward_keep_o``:
    no attention recomputation, same gradients)."""
    if x.dim() != 3:
        raise ValueError("x must be [B, N, d]")
    B, N, d = x.shape
    d_ff = p["W_1"].shape[1]
    code = _dtype_code(x)
    tensors = [x] + [p[k] for k in PARAM_NAMES]
    for t in tensors:
        if not t.is_cuda or not t.is_contiguous() or t.dtype != x.dtype:
            raise ValueError("inputs must be contiguous CUDA tensors of one dtype")
    if stats.dtype != torch.float32 or dZ.dtype != torch.float32 or not dZ.is_contiguous():
        raise ValueError("stats and dZ must be contiguous fp32 CUDA tensors")
    if workspace is None:
        st, nbytes = _lib.bpt_layer_backward_workspace_size_opt(B, N, d, h, d_ff, causal, code,
                                                                opts)
        if st != _lib.BPT_OK:
            raise _lib.BptError(st, "bpt_layer_backward_workspace_size")
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=x.device)
    grads = {k: torch.empty(p[k].shape if k != "x" else x.shape, dtype=torch.float32,
                            device=x.device) for k in GRAD_SHAPES}
    s = stream if stream is not None else torch.cuda.current_stream(x.device)
    order = ["x", "ln1", "W_Q", "W_K", "W_V", "W_O", "ln2", "W_1", "b_1", "W_2", "b_2"]
    if o is not None:
        if o.dtype != torch.float16 or tuple(o.shape) != (B, N, d) or not o.is_contiguous():
            raise ValueError(f"o must be a contiguous fp16 [{B}, {N}, {d}] tensor")
        st = _lib.bpt_layer_backward_keep_o(*[t.data_ptr() for t in tensors], stats.data_ptr(),
                                            o.data_ptr(), dZ.data_ptr(), B, N, d, h, d_ff,
                                            causal, code, *[grads[k].data_ptr() for k in order],
                                            workspace.data_ptr(), workspace.numel(), opts,
                                            s.cuda_stream)
    else:
        st = _lib.bpt_layer_backward_opt(*[t.data_ptr() for t in tensors], stats.data_ptr(),
                                         dZ.data_ptr(), B, N, d, h, d_ff, causal, code,
                                         *[grads[k].data_ptr() for k in order],
                                         workspace.data_ptr(), workspace.numel(), opts,
                                         s.cuda_stream)
    if st != _lib.BPT_OK:
        raise _lib.BptError(st, "bpt_layer_backward")
    return grads, workspace
