"""Block-sparse attention gating (BSFA) in fp64: TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may use this module; the CUDA path never does.

Source: "Block Sparse Flash Attention" (m.montaan.com), sections
"Methodology and Mechanism" (exact scores first, then a per-block gate,
then value blocks only for the blocks that pass), "Gating Mechanism and
Threshold Calibration" (the block's maximum score against a threshold per
layer, head and query-block position; calibration keeps the top-k
off-diagonal blocks per query position, averaged over samples) and
"Complexity and Practical Considerations" (what a skipped block saves).

What is computed, per batch element and head t, with blocks of b rows
(query block i = rows i*b .. i*b+b-1, key block j likewise):

  s_max(i, j) = max of s_pq = q_p . k_q / sqrt(d_k) over the valid query
                rows p of block i (p < N), the valid keys q of block j
                (q < N) and, when causal, q <= p;
  keep(i, j)  = (j == i) or s_max(i, j) >= T[t, i];
  row p's attention = softmax over the allowed keys of the kept blocks only,
                times their values.

Readings where the page is silent: a pruned block is left out of the softmax
as well as the value product (the page skips the block after the gate, so it
enters neither the normaliser nor the output); the diagonal block is never
gated (the page gates off-diagonal blocks); without a causal mask every
block j != i is off-diagonal; a NaN threshold prunes (the comparison fails).
Calibration: for query block i the off-diagonal blocks are ranked by s_max
and the threshold is the k-th largest, so that exactly the top k pass (ties
aside); fewer than k candidates give -inf (keep all); thresholds from several
samples are averaged.
"""
import math
from typing import Dict, Iterable, List, Tuple

import numpy as np

from .bpt_oracle import _as64, ffn_residual, layer_norm


def _block_rows(N: int, b: int, i: int) -> slice:
    return slice(i * b, min(N, (i + 1) * b))


def head_scores(Q: np.ndarray, K: np.ndarray, h: int, t: int) -> np.ndarray:
    """Scaled scores s = q . k / sqrt(d_k) of head t, [N, N] (small N)."""
    d_k = Q.shape[1] // h
    c = slice(t * d_k, (t + 1) * d_k)
    return (Q[:, c] @ K[:, c].T) / math.sqrt(d_k)


def block_max(S: np.ndarray, causal: bool, b: int) -> np.ndarray:
    """s_max(i, j) of one head's [N, N] scores; -inf where no pair is allowed
    (j > i under a causal mask)."""
    N = S.shape[0]
    nb = (N + b - 1) // b
    out = np.full((nb, nb), -np.inf)
    if causal:
        S = np.where(np.arange(N)[None, :] > np.arange(N)[:, None], -np.inf, S)
    for i in range(nb):
        for j in range(nb):
            if causal and j > i:
                continue
            out[i, j] = S[_block_rows(N, b, i), _block_rows(N, b, j)].max()
    return out


def keep_mask(bmax: np.ndarray, thresholds: np.ndarray, causal: bool) -> np.ndarray:
    """keep(i, j) for one head: the diagonal always, other visited blocks by
    s_max >= T[i]; blocks a causal mask never visits are False."""
    nb = bmax.shape[0]
    keep = np.zeros((nb, nb), dtype=bool)
    for i in range(nb):
        for j in range(nb):
            if causal and j > i:
                continue
            keep[i, j] = (j == i) or bool(bmax[i, j] >= thresholds[i])
    return keep


def attention_gated(Q: np.ndarray, K: np.ndarray, V: np.ndarray, h: int, causal: bool,
                    thresholds: np.ndarray, b: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Gated multi-head attention of one sequence.

    thresholds [h, nb].  Returns (O [N, d], keep [h, nb, nb], bmax [h, nb, nb]).
    """
    N, d = Q.shape
    d_k = d // h
    nb = (N + b - 1) // b
    O = np.empty((N, d))
    keeps = np.zeros((h, nb, nb), dtype=bool)
    bmaxs = np.full((h, nb, nb), -np.inf)
    key_block = np.arange(N) // b
    for t in range(h):
        S = head_scores(Q, K, h, t)
        bm = block_max(S, causal, b)
        keep = keep_mask(bm, thresholds[t], causal)
        # allowed[p, q]: causal order and the key's block kept for p's block
        allowed = keep[(np.arange(N) // b)[:, None], key_block[None, :]]
        if causal:
            allowed &= np.arange(N)[None, :] <= np.arange(N)[:, None]
        Sm = np.where(allowed, S, -np.inf)
        Sm = Sm - Sm.max(axis=1, keepdims=True)
        E = np.exp(Sm)
        c = slice(t * d_k, (t + 1) * d_k)
        O[:, c] = (E / E.sum(axis=1, keepdims=True)) @ V[:, c]
        keeps[t], bmaxs[t] = keep, bm
    return O, keeps, bmaxs


def layer_gated(inp: Dict[str, np.ndarray], h: int, causal: bool, thresholds: np.ndarray,
                b: int = 128) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """The layer (steps 1-7 of ``bpt_oracle``) with the attention of step 3
    gated.  thresholds [h, nb].  Returns (Z [B, N, d], keep [B, h, nb, nb],
    bmax [B, h, nb, nb])."""
    X = _as64(inp, "x")
    Bx, N, d = X.shape
    nb = (N + b - 1) // b
    Z = np.empty((Bx, N, d))
    keeps = np.zeros((Bx, h, nb, nb), dtype=bool)
    bmaxs = np.full((Bx, h, nb, nb), -np.inf)
    for bi in range(Bx):
        U = layer_norm(X[bi], _as64(inp, "gamma1"), _as64(inp, "beta1"))
        Q, K, V = U @ _as64(inp, "W_Q"), U @ _as64(inp, "W_K"), U @ _as64(inp, "W_V")
        O, keeps[bi], bmaxs[bi] = attention_gated(Q, K, V, h, causal, thresholds, b)
        Y = X[bi] + O @ _as64(inp, "W_O")
        Z[bi] = ffn_residual(Y, inp)
    return Z, keeps, bmaxs


def layer_block_max(inp: Dict[str, np.ndarray], h: int, causal: bool,
                    b: int = 128) -> np.ndarray:
    """s_max of every visited block pair of the layer's attention,
    [B, h, nb, nb] (-inf where a causal mask visits none)."""
    X = _as64(inp, "x")
    Bx, N, _ = X.shape
    nb = (N + b - 1) // b
    out = np.full((Bx, h, nb, nb), -np.inf)
    for bi in range(Bx):
        U = layer_norm(X[bi], _as64(inp, "gamma1"), _as64(inp, "beta1"))
        Q, K = U @ _as64(inp, "W_Q"), U @ _as64(inp, "W_K")
        for t in range(h):
            out[bi, t] = block_max(head_scores(Q, K, h, t), causal, b)
    return out


def calibrate_thresholds(bmax_samples: Iterable[np.ndarray], k: int,
                         causal: bool) -> np.ndarray:
    """Thresholds T [h, nb] that keep the top-k off-diagonal blocks of each
    query block, averaged over samples (each sample: s_max [h, nb, nb] of one
    sequence)."""
    if k < 0:
        raise ValueError("k must be >= 0")
    samples: List[np.ndarray] = [np.asarray(s, np.float64) for s in bmax_samples]
    h, nb, _ = samples[0].shape
    per = np.empty((len(samples), h, nb))
    for si, bm in enumerate(samples):
        for t in range(h):
            for i in range(nb):
                cand = [bm[t, i, j] for j in range(nb) if j != i and (j < i or not causal)]
                if k == 0:
                    per[si, t, i] = np.inf           # no off-diagonal block passes
                elif len(cand) <= k:
                    per[si, t, i] = -np.inf          # every candidate passes
                else:
                    per[si, t, i] = sorted(cand, reverse=True)[k - 1]
    with np.errstate(invalid="ignore"):
        return per.mean(axis=0)
