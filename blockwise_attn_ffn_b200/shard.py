"""Sequence sharding of the layer over G GPUs (marshalling and the host-side
partition; the layer itself runs in libbpt's kernels).

"Blockwise Parallel Transformer — BPT", section "BPT and Ring Attention":
the blockwise layer is the per-device kernel and the sequence is split
across devices, whose queries then need every device's keys and values.
Zig-zag ownership balances the causal work: N tokens are cut into 2G chunks
and rank r owns chunks r and 2G-1-r (its local rows, in that order).  One
forward is: ``project`` (LN1 + Q/K/V of the rank's rows; K | V to
``kv_loc``), one all-gather of ``kv_loc`` into ``kv_all`` [G, B, n_loc, 2d]
(torch.distributed; NCCL on GPUs), ``forward`` (attention against kv_all
and the fused layer body for the rank's rows).
"""
from __future__ import annotations

from typing import Dict, Optional, Tuple

import numpy as np
import torch

from . import _lib
from .layer import PARAM_NAMES


def check_shardable(N: int, G: int) -> None:
    if G < 1 or N % (256 * G) != 0:
        raise ValueError(f"N = {N} must be a multiple of 256 * G = {256 * G}")


def token_rows(N: int, G: int, rank: int) -> np.ndarray:
    """Global token indices of rank `rank`'s local rows (chunk r, then chunk
    2G-1-r)."""
    check_shardable(N, G)
    c = N // (2 * G)
    a, b = rank, 2 * G - 1 - rank
    return np.concatenate([np.arange(a * c, (a + 1) * c), np.arange(b * c, (b + 1) * c)])


def kv_source(N: int, G: int, token: int) -> Tuple[int, int]:
    """(owner rank, local row) of a token's K | V in the all-gathered buffer:
    the lookup the attention kernel performs per key block."""
    check_shardable(N, G)
    c = N // (2 * G)
    chunk = token // c
    owner = chunk if chunk < G else 2 * G - 1 - chunk
    local = (0 if chunk < G else c) + token - chunk * c
    return owner, local


def _ptrs(x: torch.Tensor, p: Dict[str, torch.Tensor]):
    tensors = [x] + [p[k] for k in PARAM_NAMES]
    for t in tensors:
        if not t.is_cuda or not t.is_contiguous() or t.dtype != torch.bfloat16:
            raise ValueError("shard inputs must be contiguous bf16 CUDA tensors")
    return [t.data_ptr() for t in tensors]


def workspace_for(B: int, N: int, G: int, d: int, h: int, d_ff: int, causal: bool,
                  device) -> torch.Tensor:
    st, nbytes = _lib.bpt_layer_shard_workspace_size(B, N, G, d, h, d_ff, causal, _lib.BPT_BF16)
    if st != _lib.BPT_OK:
        raise _lib.BptError(st, "bpt_layer_shard_workspace_size")
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def project(x_loc: torch.Tensor, p: Dict[str, torch.Tensor], h: int, causal: bool, N: int,
            G: int, rank: int, kv_loc: Optional[torch.Tensor] = None,
            out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
            stream: Optional[torch.cuda.Stream] = None):
    """Step 1 via ``bpt_layer_shard_project``: returns (kv_loc, out, workspace);
    x_loc [B, N / G, d] bf16 (the rank's rows, ``token_rows`` order)."""
    B, n_loc, d = x_loc.shape
    if n_loc * G != N:
        raise ValueError("x_loc must hold N / G rows")
    d_ff = p["W_1"].shape[1]
    if kv_loc is None:
        kv_loc = torch.empty((B, n_loc, 2 * d), dtype=torch.float16, device=x_loc.device)
    if out is None:
        out = torch.empty((B, n_loc, d), dtype=torch.float32, device=x_loc.device)
    if workspace is None:
        workspace = workspace_for(B, N, G, d, h, d_ff, causal, x_loc.device)
    s = stream if stream is not None else torch.cuda.current_stream(x_loc.device)
    st = _lib.bpt_layer_shard_project(*_ptrs(x_loc, p), B, N, G, rank, d, h, d_ff, causal,
                                      _lib.BPT_BF16, kv_loc.data_ptr(), out.data_ptr(),
                                      workspace.data_ptr(), workspace.numel(), s.cuda_stream)
    if st != _lib.BPT_OK:
        raise _lib.BptError(st, "bpt_layer_shard_project")
    return kv_loc, out, workspace


def forward(x_loc: torch.Tensor, p: Dict[str, torch.Tensor], h: int, causal: bool, N: int,
            G: int, rank: int, kv_all: torch.Tensor, out: torch.Tensor,
            workspace: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Step 3 via ``bpt_layer_shard_forward`` (the workspace of step 1)."""
    B, n_loc, d = x_loc.shape
    d_ff = p["W_1"].shape[1]
    if tuple(kv_all.shape) != (G, B, n_loc, 2 * d) or kv_all.dtype != torch.float16:
        raise ValueError(f"kv_all must be fp16 [{G}, {B}, {n_loc}, {2 * d}]")
    s = stream if stream is not None else torch.cuda.current_stream(x_loc.device)
    st = _lib.bpt_layer_shard_forward(*_ptrs(x_loc, p), B, N, G, rank, d, h, d_ff, causal,
                                      _lib.BPT_BF16, kv_all.data_ptr(), out.data_ptr(),
                                      workspace.data_ptr(), workspace.numel(), s.cuda_stream)
    if st != _lib.BPT_OK:
        raise _lib.BptError(st, "bpt_layer_shard_forward")
    return out


def gather_kv(kv_loc: torch.Tensor, kv_all: torch.Tensor, dist, group=None) -> torch.Tensor:
    """Step 2: every rank's kv_loc into kv_all [G, ...] (rank-major), one
    all-gather into this process's own buffer."""
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(kv_all.view(-1), kv_loc.reshape(-1), group=group)
    else:  # gloo (CPU tests)
        parts = [torch.empty_like(kv_loc) for _ in range(kv_all.shape[0])]
        dist.all_gather(parts, kv_loc, group=group)
        kv_all.copy_(torch.stack(parts))
    return kv_all


def sequence_parallel_forward(x_loc, p, h, causal, N, dist, group=None, bufs=None,
                              stream=None):
    """One sharded forward of this rank (steps 1-3).  ``bufs`` (from a
    previous call) reuses kv_loc, kv_all, out and the workspace.  Returns
    (out, bufs)."""
    G, rank = dist.get_world_size(group), dist.get_rank(group)
    B, n_loc, d = x_loc.shape
    if bufs is None:
        kv_loc, out, ws = project(x_loc, p, h, causal, N, G, rank, stream=stream)
        kv_all = torch.empty((G, B, n_loc, 2 * d), dtype=torch.float16, device=x_loc.device)
        bufs = {"kv_loc": kv_loc, "kv_all": kv_all, "out": out, "ws": ws}
    else:
        project(x_loc, p, h, causal, N, G, rank, kv_loc=bufs["kv_loc"], out=bufs["out"],
                workspace=bufs["ws"], stream=stream)
    gather_kv(bufs["kv_loc"], bufs["kv_all"], dist, group)
    forward(x_loc, p, h, causal, N, G, rank, bufs["kv_all"], bufs["out"], bufs["ws"], stream)
    return bufs["out"], bufs
