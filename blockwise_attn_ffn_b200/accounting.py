"""Algorithmic FLOP and activation-byte counts of one pre-LN BPT layer.

Host-side bookkeeping used by the bench; no layer arithmetic.

FLOP convention ("Blockwise Parallel Transformer — BPT", section "FLOPs are
unchanged — so where is the win?"): a GEMM of [M, K] x [K, N] costs 2*M*N*K;
attention costs 2*d per (query, key) pair for QK^T and 2*d for AV, counted
over the pairs the mask allows (j <= i under a causal mask, every pair
otherwise); softmax, LayerNorm and GELU are not counted.  With d_ff = 4d this
gives the page's 4N^2 d (non-causal), 8Nd^2 and 16Nd^2.

Byte convention (same page, "The bottleneck that survives FlashAttention" and
"Memory accounting"): the activations one layer keeps alive, in elements of
the activation type.
"""
from __future__ import annotations

from typing import Dict


def attention_pairs(N: int, causal: bool) -> int:
    """(query, key) pairs one head scores over one sequence."""
    return N * (N + 1) // 2 if causal else N * N


def layer_flops(B: int, N: int, d: int, h: int, d_ff: int, causal: bool) -> Dict[str, int]:
    """Algorithmic FLOPs of one layer forward, split by step."""
    del h  # the head split does not change the count
    f = {
        "qkv": 6 * B * N * d * d,
        "wo": 2 * B * N * d * d,
        "ffn": 4 * B * N * d * d_ff,
        "attention": 4 * B * d * attention_pairs(N, causal),
    }
    f["total"] = sum(f.values())
    return f


def attention_bytes(B: int, N: int, d: int, h: int, elem_bytes: int = 2) -> int:
    """Least HBM bytes of the attention step of one layer forward: Q, K and V
    read once and the per-head outputs o written once, 16-bit elements."""
    del h
    return 4 * B * N * d * elem_bytes


def unfused_activation_elems(N: int, d: int, h: int, d_ff: int,
                             with_logits: bool = True) -> Dict[str, int]:
    """Per-layer activation audit of the unfused layer (elements).

    residual [N, d]; Q, K, V 3x[N, d]; attention out + projection 2x[N, d];
    logits [h, N, N] (removed by a FlashAttention-style kernel); FFN hidden
    2x[N, d_ff] (before and after the nonlinearity).
    """
    a = {
        "residual": N * d,
        "qkv": 3 * N * d,
        "attn_out_proj": 2 * N * d,
        "ffn_hidden": 2 * N * d_ff,
    }
    if with_logits:
        a["logits"] = h * N * N
    a["total"] = sum(a.values())
    return a


def bpt_block_hidden_elems(b: int, d_ff: int) -> int:
    """FFN hidden of one query block, before and after the nonlinearity."""
    return 2 * b * d_ff


def hidden_reduction(N: int, b: int) -> float:
    """How much smaller the block hidden is than the sequence hidden: N / b."""
    return N / b
