"""Threshold calibration for block-sparse attention gating (host side).

"Block Sparse Flash Attention", section "Gating Mechanism and Threshold
Calibration": for every query-block position the off-diagonal key blocks
are ranked by their maximum score, the threshold is the value that keeps
exactly the top k of them, and the thresholds of the calibration samples are
averaged.  This is the one-time preprocessing step of the method; the gated
forward itself runs in ``bpt_layer_forward_bsfa``.  The block maxima come
from that call (``layer_forward_bsfa(..., block_max=True)`` with thresholds
-inf) on calibration sequences.
"""
import numpy as np


def calibrate(block_max: np.ndarray, k: int, causal: bool) -> np.ndarray:
    """Thresholds [h, nb] (float32) from block maxima [S, h, nb, nb] of S
    calibration sequences: per (head, query block i) the k-th largest
    off-diagonal maximum, averaged over the sequences; -inf where i has at
    most k off-diagonal blocks (keep them all); +inf for k = 0."""
    if k < 0:
        raise ValueError("k must be >= 0")
    bm = np.asarray(block_max, dtype=np.float64)
    S, h, nb, _ = bm.shape
    if k == 0:
        return np.full((h, nb), np.inf, dtype=np.float32)
    if k >= nb:
        return np.full((h, nb), -np.inf, dtype=np.float32)
    off = ~np.eye(nb, dtype=bool)
    if causal:
        off &= np.tril(np.ones((nb, nb), dtype=bool))
    cand = np.where(off[None, None], bm, -np.inf)          # excluded -> -inf
    desc = -np.sort(-cand, axis=-1)                         # descending per row
    kth = desc[..., k - 1]                                  # [S, h, nb]
    n_cand = off.sum(axis=1)                                # [nb]
    kth = np.where((n_cand <= k)[None, None, :], -np.inf, kth)
    return kth.mean(axis=0).astype(np.float32)
