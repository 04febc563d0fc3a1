"""Seeded synthetic inputs for one pre-LN BPT layer.

This module is shared by the CUDA path's harness (tests, bench) and by the
fp64 oracle.  It holds none of the layer's arithmetic: it only draws random
numbers in a fixed order and rounds them to bfloat16 where the workload asks
for bfloat16 inputs.

Recipe (the same for every workload):

* ``numpy.random.default_rng(seed)`` (PCG64), float32 standard normals drawn in
  this order: x, W_Q, W_K, W_V, W_O, W_1, b_1, W_2, b_2, gamma1, beta1,
  gamma2, beta2.
* Every weight is scaled by 1/sqrt(fan_in): fan_in = d for W_Q, W_K, W_V, W_O
  and W_1, fan_in = d_ff for W_2.  Weights are row-major [d_in, d_out], so the
  layer computes ``x @ W`` as the pages write it.
* Biases are ``bias_scale * N(0, 1)``; every named workload uses
  ``bias_scale = 0`` (biases zero).
* LayerNorm parameters: ``gamma = 1 + ln_scale * N(0,1)``,
  ``beta = ln_scale * N(0,1)``; the tiny fp32 workload uses ``ln_scale = 0``
  (gamma = 1, beta = 0), the bf16 workloads ``ln_scale = 0.1``.
* For bf16 workloads every tensor is rounded to bfloat16 by round to nearest,
  ties to even, from the float32 draw.  Both sides receive exactly these
  rounded values (the oracle promotes them to float64).
"""
from __future__ import annotations

import dataclasses
from typing import Dict

import numpy as np


@dataclasses.dataclass(frozen=True)
class LayerShape:
    """Shape and numerics of one BPT layer workload."""

    name: str
    B: int
    N: int
    d: int
    h: int
    d_ff: int
    causal: bool
    dtype: str          # "f32" or "bf16": the type of x, weights and params
    block: int          # query / key-value block size b
    seed: int
    ln_scale: float     # spread of LayerNorm gamma/beta around (1, 0)
    bias_scale: float = 0.0

    @property
    def d_k(self) -> int:
        return self.d // self.h

    def with_(self, **kw) -> "LayerShape":
        return dataclasses.replace(self, **kw)


# The five workloads the layer is measured on.  The tiny fp32 one is the case
# the CPU oracle finishes in well under a second; the long-context one
# (N = 65536) is the throughput workload.
WORKLOADS: Dict[str, LayerShape] = {
    "tiny_f32": LayerShape("tiny_f32", B=1, N=256, d=64, h=1, d_ff=256,
                           causal=False, dtype="f32", block=64, seed=0,
                           ln_scale=0.0),
    "gpt2s_n2k": LayerShape("gpt2s_n2k", B=8, N=2048, d=768, h=12, d_ff=3072,
                            causal=True, dtype="bf16", block=128, seed=1,
                            ln_scale=0.1),
    "mid_n16k": LayerShape("mid_n16k", B=1, N=16384, d=1024, h=16, d_ff=4096,
                           causal=True, dtype="bf16", block=128, seed=2,
                           ln_scale=0.1),
    "long_n64k": LayerShape("long_n64k", B=1, N=65536, d=2048, h=16, d_ff=8192,
                            causal=True, dtype="bf16", block=128, seed=3,
                            ln_scale=0.1),
    "wide_n128k": LayerShape("wide_n128k", B=1, N=131072, d=4096, h=32,
                             d_ff=16384, causal=True, dtype="bf16", block=128,
                             seed=4, ln_scale=0.1),
}

# Order of the workloads as the throughput table lists them.
WORKLOAD_ORDER = ["tiny_f32", "gpt2s_n2k", "mid_n16k", "long_n64k", "wide_n128k"]


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); uint16 bits.

    Inputs are finite normals, so no NaN handling is needed.
    """
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns (uint16) to float32 exactly."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


PARAM_ORDER = ["x", "W_Q", "W_K", "W_V", "W_O", "W_1", "b_1", "W_2", "b_2",
               "gamma1", "beta1", "gamma2", "beta2"]


def make_inputs(cfg: LayerShape, B: int | None = None) -> Dict[str, np.ndarray]:
    """Draw the layer's inputs for ``cfg``.

    Returns float32 arrays holding exactly the values both sides use (already
    rounded to bfloat16 for bf16 workloads) plus, for bf16 workloads, the
    matching uint16 bit patterns under ``<name>_bits``.  ``B`` overrides the
    batch count of x (the draw order is unchanged, so batch element 0 is the
    same for every B).

    Shapes: x [B, N, d]; W_Q, W_K, W_V, W_O [d, d]; W_1 [d, d_ff];
    b_1 [d_ff]; W_2 [d_ff, d]; b_2 [d]; gamma*/beta* [d].
    """
    Bx = cfg.B if B is None else B
    d, d_ff, N = cfg.d, cfg.d_ff, cfg.N
    rng = np.random.default_rng(cfg.seed)

    def normal(*shape):
        return rng.standard_normal(size=shape, dtype=np.float32)

    out: Dict[str, np.ndarray] = {}
    out["x"] = normal(Bx, N, d)
    s_d = np.float32(1.0 / np.sqrt(d))
    s_ff = np.float32(1.0 / np.sqrt(d_ff))
    out["W_Q"] = normal(d, d) * s_d
    out["W_K"] = normal(d, d) * s_d
    out["W_V"] = normal(d, d) * s_d
    out["W_O"] = normal(d, d) * s_d
    out["W_1"] = normal(d, d_ff) * s_d
    out["b_1"] = normal(d_ff) * np.float32(cfg.bias_scale)
    out["W_2"] = normal(d_ff, d) * s_ff
    out["b_2"] = normal(d) * np.float32(cfg.bias_scale)
    ln = np.float32(cfg.ln_scale)
    out["gamma1"] = np.float32(1.0) + normal(d) * ln
    out["beta1"] = normal(d) * ln
    out["gamma2"] = np.float32(1.0) + normal(d) * ln
    out["beta2"] = normal(d) * ln

    if cfg.dtype == "bf16":
        for k in PARAM_ORDER:
            bits = f32_to_bf16_bits(out[k])
            out[k + "_bits"] = bits
            out[k] = bf16_bits_to_f32(bits)
    elif cfg.dtype != "f32":
        raise ValueError(f"unknown dtype {cfg.dtype!r}")
    return out


def sample_rows(cfg: LayerShape, count: int = 256, B: int | None = None) -> np.ndarray:
    """Seeded sample of (batch, row) pairs, as an int64 array [count, 2].

    Drawn with ``default_rng(seed + 1000)`` over all B*N rows; always holds the
    rows 0, b-1, b (when they exist) and N-1 of batch element 0, which sit at
    block edges and at the far end of the causal range.
    """
    Bx = cfg.B if B is None else B
    total = Bx * cfg.N
    must = [r for r in (0, cfg.block - 1, cfg.block, cfg.N - 1) if 0 <= r < cfg.N]
    must = sorted(set(must))
    rng = np.random.default_rng(cfg.seed + 1000)
    want = max(0, min(count, total) - len(must))
    pool = rng.choice(total, size=min(total, want + len(must) + 8), replace=False)
    flat = list(must)
    for p in pool:
        if len(flat) >= min(count, total):
            break
        if int(p) not in flat:
            flat.append(int(p))
    flat = np.array(sorted(flat), dtype=np.int64)
    return np.stack([flat // cfg.N, flat % cfg.N], axis=1)
