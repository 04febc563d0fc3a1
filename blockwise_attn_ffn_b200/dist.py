"""Host-side helpers for running the layer on several GPUs, one process each.

The BPT outer loop is data parallel across sequences ("Blockwise Parallel
Transformer — BPT", section "Why parallel is in the name": query blocks, and
a fortiori whole sequences, never read each other's state).  Each rank
therefore runs its own batch of the workload with no collective on the data
path; the only communication is the timing reduction (max over ranks) done
by the caller.  Works with the nccl backend on GPUs and gloo on CPU.
"""
from __future__ import annotations

import datetime
import os
from typing import Dict, Tuple

import numpy as np

from .inputs import LayerShape, bf16_bits_to_f32, f32_to_bf16_bits, make_inputs


def env_rank() -> Tuple[int, int, int]:
    """(rank, local_rank, world_size) from the torchrun environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def init_process_group(backend: str, device=None, timeout_s: int = 120):
    """Initialise torch.distributed from the environment with a short timeout."""
    import torch.distributed as dist
    kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if device is not None:
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)
    return dist


def rank_inputs(cfg: LayerShape, rank: int) -> Dict[str, np.ndarray]:
    """Inputs of rank `rank`: the workload's weights (identical on every
    rank) and the rank's own batch of x.  Rank 0's x is the workload's x; rank
    r > 0 draws its x from default_rng([seed, r]) with the same distribution
    and rounding."""
    inp = make_inputs(cfg)
    if rank > 0:
        rng = np.random.default_rng([cfg.seed, rank])
        x32 = rng.standard_normal(size=inp["x"].shape, dtype=np.float32)
        if cfg.dtype == "bf16":
            inp["x_bits"] = f32_to_bf16_bits(x32)
            inp["x"] = bf16_bits_to_f32(inp["x_bits"])
        else:
            inp["x"] = x32
    return inp


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """Max of a per-rank scalar (e.g. device milliseconds) over all ranks."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_tokens_per_s(cfg: LayerShape, world: int, ms_per_step_max: float) -> float:
    """Whole-job throughput: every rank's tokens over the slowest rank's time."""
    return cfg.B * cfg.N * world / (ms_per_step_max / 1e3)
