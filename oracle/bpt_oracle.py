"""fp64 CPU oracle for one pre-LN Blockwise Parallel Transformer layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` use it.  It shares no code with the CUDA path;
the two meet only in ``blockwise_attn_ffn_b200.inputs`` (seeded draws, no
layer arithmetic).

Sources (web pages, cited by title and section):

* "Blockwise Parallel Transformer — BPT" (aicassindra.com), sections
  "The bottleneck that survives FlashAttention" (the layer's tensors),
  "The structural fact that makes fusion legal" (LN, FFN and residuals act
  per token), "The fused blockwise algorithm" (the two-level loop, the online
  softmax state and the block FFN) and "Pitfalls and misconceptions" (causal
  blocks j > i are skipped).
* "transformer-cost" (raminaeye.github.io), FlashAttention section: the
  max-subtracted softmax and the running-max / running-sum rescaling.
* "Blockwise Parallel Transformer — BPT", section "The backward pass": the
  forward keeps, per row, the softmax statistics (m, l) that the backward's
  block recomputation reads.

What the layer computes, for every batch element independently (the unfused
reading, which is the plain definition; the fused schedule reaches the same
value up to rounding order):

1. U = LN1(X)                         (per row, gamma1, beta1)
2. Q = U W_Q, K = U W_K, V = U W_V    (no projection biases)
3. per head t (columns t*d_k .. (t+1)*d_k):
   S = Q_t K_t^T / sqrt(d_k); causal: S_ij = -inf for j > i;
   A = softmax over each row; O_t = A V_t
4. Y = X + O W_O
5. Vn = LN2(Y)
6. H = GELU(Vn W_1 + b_1), GELU(z) = z/2 (1 + erf(z / sqrt 2))
7. Z = Y + H W_2 + b_2

Readings taken where the pages are silent:
LayerNorm epsilon 1e-5 inside the square root, biased variance; exact erf
GELU; heads are contiguous column slices concatenated in head order; the
causal mask keeps the diagonal (j <= i); Q/K/V/O carry no bias.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
(library routines, closed forms, invariants, pure-Python brute force).
"""
from __future__ import annotations

import math
from typing import Dict, Iterable, Optional, Tuple

import numpy as np
from scipy.special import erf as _erf

LN_EPS = 1e-5

# Rows per chunk when a sequence-long step is formed piecewise; chunking the
# query rows does not change any row's arithmetic (every row is computed from
# the same full operands), it only bounds host memory.
ROW_CHUNK = 2048


# --------------------------------------------------------------------------
# Elementwise and per-row pieces
# --------------------------------------------------------------------------
def layer_norm(X: np.ndarray, gamma: np.ndarray, beta: np.ndarray,
               eps: float = LN_EPS) -> np.ndarray:
    """LayerNorm over the last axis (the feature axis of a token).

    The BPT page's "structural fact" section: LN normalises within a token,
    across the feature axis.  Mean, then the biased variance of the deviations
    (two passes), eps inside the square root.
    """
    X = np.asarray(X, dtype=np.float64)
    mu = X.mean(axis=-1, keepdims=True)
    dev = X - mu
    var = (dev * dev).mean(axis=-1, keepdims=True)
    return dev / np.sqrt(var + eps) * np.asarray(gamma, np.float64) \
        + np.asarray(beta, np.float64)


def gelu(z: np.ndarray) -> np.ndarray:
    """Exact GELU, z * Phi(z) = z/2 * (1 + erf(z / sqrt 2)).

    The BPT pseudocode writes ``act``; the workloads name GELU.  The erf form
    (not the tanh approximation) is the reading taken.
    """
    z = np.asarray(z, dtype=np.float64)
    return 0.5 * z * (1.0 + _erf(z / math.sqrt(2.0)))


def softmax_rows(S: np.ndarray) -> np.ndarray:
    """Row softmax with the row maximum subtracted before exp.

    transformer-cost, FlashAttention section: subtract each row's maximum so
    exp never overflows.  -inf entries give exactly zero weight.
    """
    m = S.max(axis=-1, keepdims=True)
    e = np.exp(S - m)
    return e / e.sum(axis=-1, keepdims=True)


# --------------------------------------------------------------------------
# The online softmax state (used by the blockwise schedule below)
# --------------------------------------------------------------------------
def online_softmax_init(rows: int, width: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """State (m, l, o) = (-inf, 0, 0) of the BPT inner loop."""
    return (np.full(rows, -np.inf), np.zeros(rows), np.zeros((rows, width)))


def online_softmax_update(m: np.ndarray, l: np.ndarray, o: np.ndarray,
                          s: np.ndarray, v: np.ndarray):
    """One inner-loop step of the BPT pseudocode for a key/value block.

    m' = max(m, rowmax s); alpha = exp(m - m'); l = alpha l + sum exp(s - m');
    o = alpha o + exp(s - m') v.   (BPT page, "The fused blockwise
    algorithm"; transformer-cost, running max and sum.)  A row whose entries
    so far are all -inf keeps m = -inf and contributes nothing.
    """
    m_new = np.maximum(m, s.max(axis=-1))
    # exp(-inf - (-inf)) would be NaN; a row still at -inf has l = o = 0, so
    # its factor is irrelevant and is set to 0.
    finite = np.isfinite(m_new)
    safe = np.where(finite, m_new, 0.0)
    alpha = np.where(np.isfinite(m), np.exp(m - safe), 0.0)
    p = np.where(finite[:, None], np.exp(s - safe[:, None]), 0.0)
    l_new = alpha * l + p.sum(axis=-1)
    o_new = alpha[:, None] * o + p @ v
    return m_new, l_new, o_new


# --------------------------------------------------------------------------
# The unfused layer (the definition)
# --------------------------------------------------------------------------
def _as64(inp: Dict[str, np.ndarray], k: str) -> np.ndarray:
    return np.asarray(inp[k], dtype=np.float64)


def attention_rows(Qr: np.ndarray, K: np.ndarray, V: np.ndarray, h: int,
                   causal: bool, qpos: np.ndarray) -> np.ndarray:
    """Multi-head attention output for query rows ``Qr`` at positions ``qpos``.

    Step 3 of the layer.  K, V hold every key the rows may see (positions
    0..len(K)-1).  Head t uses the columns t*d_k .. (t+1)*d_k; the heads'
    outputs are concatenated in head order.
    """
    d = Qr.shape[1]
    d_k = d // h
    scale = 1.0 / math.sqrt(d_k)
    n_keys = K.shape[0]
    O = np.empty_like(Qr)
    if causal:
        masked = np.arange(n_keys)[None, :] > qpos[:, None]
    for t in range(h):
        c = slice(t * d_k, (t + 1) * d_k)
        S = (Qr[:, c] @ K[:, c].T) * scale
        if causal:
            S = np.where(masked, -np.inf, S)
        O[:, c] = softmax_rows(S) @ V[:, c]
    return O


def ffn_residual(Y: np.ndarray, inp: Dict[str, np.ndarray]) -> np.ndarray:
    """Steps 5-7 for a set of rows: Y + GELU(LN2(Y) W_1 + b_1) W_2 + b_2.

    BPT page, "The fused blockwise algorithm" (h_i = act(LN(y_i) W_1),
    Z[i] = y_i + h_i W_2) with the workloads' biases b_1, b_2.  Row r of the
    result reads row r of Y alone ("The structural fact that makes fusion
    legal").
    """
    Hh = gelu(layer_norm(Y, _as64(inp, "gamma2"), _as64(inp, "beta2"))
              @ _as64(inp, "W_1") + _as64(inp, "b_1"))
    return Y + Hh @ _as64(inp, "W_2") + _as64(inp, "b_2")


def layer_unfused(inp: Dict[str, np.ndarray], h: int, causal: bool,
                  batches: Optional[Iterable[int]] = None) -> np.ndarray:
    """Z for the whole input, as the plain unfused layer (steps 1-7).

    Returns float64 [B, N, d].  ``batches`` restricts the batch elements
    computed (the others are left as NaN).
    """
    X = _as64(inp, "x")
    Bx, N, d = X.shape
    Z = np.full((Bx, N, d), np.nan)
    W_Q, W_K, W_V, W_O = (_as64(inp, k) for k in ("W_Q", "W_K", "W_V", "W_O"))
    g1, be1 = _as64(inp, "gamma1"), _as64(inp, "beta1")
    for b in (range(Bx) if batches is None else batches):
        U = layer_norm(X[b], g1, be1)
        Q, K, V = U @ W_Q, U @ W_K, U @ W_V
        O = np.empty((N, d))
        for r0 in range(0, N, ROW_CHUNK):
            r1 = min(N, r0 + ROW_CHUNK)
            # Under a causal mask rows < r1 give keys >= r1 weight exactly 0,
            # so those keys are left out of the chunk's score rows.
            nk = r1 if causal else N
            O[r0:r1] = attention_rows(Q[r0:r1], K[:nk], V[:nk], h, causal,
                                      np.arange(r0, r1))
        Y = X[b] + O @ W_O
        for r0 in range(0, N, ROW_CHUNK):
            r1 = min(N, r0 + ROW_CHUNK)
            Z[b, r0:r1] = ffn_residual(Y[r0:r1], inp)
    return Z


def layer_intermediates(inp: Dict[str, np.ndarray], h: int, causal: bool,
                        b: int = 0) -> Dict[str, np.ndarray]:
    """Every intermediate of steps 1-7 for batch element ``b`` (small N only).

    Keys: U, Q, K, V, O, Y, Vn, Hpre (Vn W_1 + b_1), H, Z; all float64.
    """
    X = _as64(inp, "x")[b]
    N, d = X.shape
    U = layer_norm(X, _as64(inp, "gamma1"), _as64(inp, "beta1"))
    Q, K, V = U @ _as64(inp, "W_Q"), U @ _as64(inp, "W_K"), U @ _as64(inp, "W_V")
    O = attention_rows(Q, K, V, h, causal, np.arange(N))
    Y = X + O @ _as64(inp, "W_O")
    Vn = layer_norm(Y, _as64(inp, "gamma2"), _as64(inp, "beta2"))
    Hpre = Vn @ _as64(inp, "W_1") + _as64(inp, "b_1")
    H = gelu(Hpre)
    Z = Y + H @ _as64(inp, "W_2") + _as64(inp, "b_2")
    return dict(U=U, Q=Q, K=K, V=V, O=O, Y=Y, Vn=Vn, Hpre=Hpre, H=H, Z=Z)


def layer_rows(inp: Dict[str, np.ndarray], h: int, causal: bool,
               rows: np.ndarray) -> np.ndarray:
    """Z at sampled (batch, row) pairs only; float64 [len(rows), d].

    Exact for those rows by the token-wise property (BPT page, "The structural
    fact that makes fusion legal"): after attention, every remaining step of a
    row reads that row alone.  K and V are formed for every key the sampled
    rows can see (all keys up to the largest sampled row under a causal mask,
    all keys otherwise), in row chunks to bound host memory.
    """
    X = _as64(inp, "x")
    Bx, N, d = X.shape
    rows = np.asarray(rows, dtype=np.int64).reshape(-1, 2)
    out = np.empty((rows.shape[0], d))
    W_Q, W_K, W_V, W_O = (_as64(inp, k) for k in ("W_Q", "W_K", "W_V", "W_O"))
    g1, be1 = _as64(inp, "gamma1"), _as64(inp, "beta1")
    for b in np.unique(rows[:, 0]):
        sel = np.nonzero(rows[:, 0] == b)[0]
        pos = rows[sel, 1]
        n_keys = int(pos.max()) + 1 if causal else N
        K = np.empty((n_keys, d))
        V = np.empty((n_keys, d))
        for r0 in range(0, n_keys, ROW_CHUNK):
            r1 = min(n_keys, r0 + ROW_CHUNK)
            U = layer_norm(X[b, r0:r1], g1, be1)
            K[r0:r1] = U @ W_K
            V[r0:r1] = U @ W_V
        Ur = layer_norm(X[b, pos], g1, be1)
        O = attention_rows(Ur @ W_Q, K, V, h, causal, pos)
        Y = X[b, pos] + O @ W_O
        out[sel] = ffn_residual(Y, inp)
    return out


def attention_stats_rows(inp: Dict[str, np.ndarray], h: int, causal: bool,
                         rows: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Per-row softmax statistics (m, l) at sampled (batch, row) pairs.

    BPT page, "The backward pass": the forward keeps, for every row, the
    softmax statistics it needs to recompute the row's attention exactly.
    For head t of row i, with s_j = q_i . k_j / sqrt(d_k) over the keys the
    row may attend to (j <= i under the causal mask):
        m = max_j s_j,   l = sum_j exp(s_j - m).
    Returns float64 arrays m, l of shape [len(rows), h].  Q and K are those
    of steps 1-2 (LN1, then the projections); K is formed in row chunks as in
    ``layer_rows``.
    """
    X = _as64(inp, "x")
    Bx, N, d = X.shape
    d_k = d // h
    scale = 1.0 / math.sqrt(d_k)
    rows = np.asarray(rows, dtype=np.int64).reshape(-1, 2)
    m_out = np.empty((rows.shape[0], h))
    l_out = np.empty((rows.shape[0], h))
    W_Q, W_K = _as64(inp, "W_Q"), _as64(inp, "W_K")
    g1, be1 = _as64(inp, "gamma1"), _as64(inp, "beta1")
    for b in np.unique(rows[:, 0]):
        sel = np.nonzero(rows[:, 0] == b)[0]
        pos = rows[sel, 1]
        n_keys = int(pos.max()) + 1 if causal else N
        K = np.empty((n_keys, d))
        for r0 in range(0, n_keys, ROW_CHUNK):
            r1 = min(n_keys, r0 + ROW_CHUNK)
            K[r0:r1] = layer_norm(X[b, r0:r1], g1, be1) @ W_K
        Qr = layer_norm(X[b, pos], g1, be1) @ W_Q
        for t in range(h):
            c = slice(t * d_k, (t + 1) * d_k)
            S = (Qr[:, c] @ K[:, c].T) * scale
            if causal:
                S = np.where(np.arange(n_keys)[None, :] > pos[:, None], -np.inf, S)
            m = S.max(axis=1)
            m_out[sel, t] = m
            l_out[sel, t] = np.exp(S - m[:, None]).sum(axis=1)
    return m_out, l_out


# --------------------------------------------------------------------------
# The fused blockwise schedule (the pages' two-level loop), fp64
# --------------------------------------------------------------------------
def layer_blockwise(inp: Dict[str, np.ndarray], h: int, causal: bool,
                    block: int) -> np.ndarray:
    """Z by the BPT two-level loop, literally: float64 [B, N, d].

    BPT page, "The fused blockwise algorithm": for each query block i, q_i =
    LN(x_i) W_Q and (m, l, o) start at (-inf, 0, 0); for each key/value block
    j, k_j and v_j are formed from LN(X[j]) and the online-softmax state is
    updated; then y_i = x_i + (o / l) W_O, h_i = act(LN(y_i) W_1) and
    Z[i] = y_i + h_i W_2.  Per head, as the multi-head reading requires.
    Causal: blocks j > i are skipped outright ("Pitfalls and misconceptions")
    and the diagonal block masks keys after the query.  b_1 and b_2 enter as
    in the unfused definition.  The last block of a sequence may be short.
    """
    X = _as64(inp, "x")
    Bx, N, d = X.shape
    d_k = d // h
    scale = 1.0 / math.sqrt(d_k)
    W_Q, W_K, W_V, W_O = (_as64(inp, k) for k in ("W_Q", "W_K", "W_V", "W_O"))
    W_1, b_1, W_2, b_2 = (_as64(inp, k) for k in ("W_1", "b_1", "W_2", "b_2"))
    g1, be1, g2, be2 = (_as64(inp, k) for k in ("gamma1", "beta1", "gamma2", "beta2"))
    Z = np.empty((Bx, N, d))
    starts = list(range(0, N, block))
    for b in range(Bx):
        for i0 in starts:                       # outer loop: query blocks
            i1 = min(N, i0 + block)
            x_i = X[b, i0:i1]
            q_i = layer_norm(x_i, g1, be1) @ W_Q
            attn = np.empty_like(x_i)
            for t in range(h):
                c = slice(t * d_k, (t + 1) * d_k)
                m, l, o = online_softmax_init(i1 - i0, d_k)
                for j0 in starts:               # inner loop: key/value blocks
                    if causal and j0 > i0:
                        continue                # skipped, not computed
                    j1 = min(N, j0 + block)
                    u_j = layer_norm(X[b, j0:j1], g1, be1)
                    k_j, v_j = u_j @ W_K[:, c], u_j @ W_V[:, c]
                    s = (q_i[:, c] @ k_j.T) * scale
                    if causal and j0 == i0:
                        qp = np.arange(i0, i1)[:, None]
                        kp = np.arange(j0, j1)[None, :]
                        s = np.where(kp > qp, -np.inf, s)
                    m, l, o = online_softmax_update(m, l, o, s, v_j)
                attn[:, c] = o / l[:, None]
            y_i = x_i + attn @ W_O
            h_i = gelu(layer_norm(y_i, g2, be2) @ W_1 + b_1)
            Z[b, i0:i1] = y_i + h_i @ W_2 + b_2
    return Z
