"""fp64 CPU oracle for the backward pass of one pre-LN BPT layer.

TEST INFRASTRUCTURE ONLY, like ``bpt_oracle``: nothing on the product path
imports, calls or executes it.

Source: "Blockwise Parallel Transformer — BPT", section "The backward pass":
the forward keeps the layer input, the layer output and the per-row softmax
statistics (m, l); backward, each block recomputes its own scores, attention
output and FFN hidden from those statistics and consumes them at once to
accumulate the gradients of W_1, W_2, W_O and the QKV projections, in one
pass (no re-derivation of the softmax normalisation).

Two functions compute the same gradients:

* ``layer_backward`` -- the chain rule through the unfused layer (steps 1-7
  of ``bpt_oracle``), the plain definition.
* ``layer_backward_blockwise`` -- the pages' schedule: query blocks in
  order; each recomputes its attention output in one pass from (m, l), its
  y, LN2 and FFN hidden, back-propagates the FFN and W_O for its rows and
  the attention for its (query, key) block pairs, accumulating into the
  weight gradients and dQ, dK, dV; the QKV projection and LN1 gradients
  follow once dQ, dK, dV are complete.

Gradient formulas (standard calculus, written out here):
  LayerNorm y = g * xh + b, xh = (x - mu) / sigma, sigma = sqrt(var + eps):
    dg = sum_rows dy * xh,  db = sum_rows dy,
    dx = (dxh - mean(dxh) - xh * mean(dxh * xh)) / sigma,  dxh = dy * g
  GELU(z) = z Phi(z):  GELU'(z) = Phi(z) + z phi(z)
  attention per head, P = softmax(S), S = Q K^T / sqrt(d_k) (masked -inf):
    dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D),  D = rowsum(dO * O),
    dQ = dS K / sqrt(d_k),  dK = dS^T Q / sqrt(d_k)
Readings: as in ``bpt_oracle`` (eps 1e-5, biased variance, exact erf GELU,
no projection biases).  The upstream gradient dZ is an input.
"""
from __future__ import annotations

import math
from typing import Dict

import numpy as np

from .bpt_oracle import LN_EPS, _as64, attention_stats_rows, gelu, layer_intermediates, layer_norm

GRAD_NAMES = ["x", "W_Q", "W_K", "W_V", "W_O", "W_1", "b_1", "W_2", "b_2",
              "gamma1", "beta1", "gamma2", "beta2"]


def layer_norm_backward(X: np.ndarray, gamma: np.ndarray, dY: np.ndarray):
    """(dX, dgamma, dbeta) of y = LN(x) * gamma + beta over the last axis."""
    mu = X.mean(axis=-1, keepdims=True)
    var = ((X - mu) ** 2).mean(axis=-1, keepdims=True)
    sig = np.sqrt(var + LN_EPS)
    xh = (X - mu) / sig
    dxh = dY * gamma
    dX = (dxh - dxh.mean(axis=-1, keepdims=True)
          - xh * (dxh * xh).mean(axis=-1, keepdims=True)) / sig
    return dX, (dY * xh).reshape(-1, X.shape[-1]).sum(0), dY.reshape(-1, X.shape[-1]).sum(0)


def gelu_grad(z: np.ndarray) -> np.ndarray:
    """d/dz of z Phi(z) = Phi(z) + z phi(z)."""
    from scipy.special import erf
    return 0.5 * (1.0 + erf(z / math.sqrt(2.0))) + z * np.exp(-0.5 * z * z) / math.sqrt(2.0 * math.pi)


def attention_backward(Q, K, V, O, dO, h: int, causal: bool):
    """(dQ, dK, dV) of the multi-head attention of one sequence."""
    N, d = Q.shape
    d_k = d // h
    scale = 1.0 / math.sqrt(d_k)
    dQ, dK, dV = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V)
    mask = np.triu(np.ones((N, N), dtype=bool), 1) if causal else None
    for t in range(h):
        c = slice(t * d_k, (t + 1) * d_k)
        S = (Q[:, c] @ K[:, c].T) * scale
        if causal:
            S = np.where(mask, -np.inf, S)
        P = np.exp(S - S.max(axis=1, keepdims=True))
        P /= P.sum(axis=1, keepdims=True)
        dV[:, c] = P.T @ dO[:, c]
        D = (dO[:, c] * O[:, c]).sum(axis=1, keepdims=True)
        dS = P * (dO[:, c] @ V[:, c].T - D)
        dQ[:, c] = dS @ K[:, c] * scale
        dK[:, c] = dS.T @ Q[:, c] * scale
    return dQ, dK, dV


def layer_backward(inp: Dict[str, np.ndarray], h: int, causal: bool,
                   dZ: np.ndarray) -> Dict[str, np.ndarray]:
    """Gradients of sum(Z * dZ) with respect to x and every parameter.

    dZ: [B, N, d].  Returns float64 arrays keyed by GRAD_NAMES (``x`` is
    [B, N, d]; the parameters have their own shapes).
    """
    dZ = np.asarray(dZ, dtype=np.float64)
    W_Q, W_K, W_V, W_O, W_1, W_2 = (_as64(inp, k) for k in ("W_Q", "W_K", "W_V", "W_O", "W_1", "W_2"))
    g1, g2 = _as64(inp, "gamma1"), _as64(inp, "gamma2")
    X = _as64(inp, "x")
    g = {k: np.zeros_like(_as64(inp, k)) for k in GRAD_NAMES}
    for b in range(X.shape[0]):
        it = layer_intermediates(inp, h, causal, b=b)
        dz = dZ[b]
        # step 7: Z = Y + H W_2 + b_2
        g["W_2"] += it["H"].T @ dz
        g["b_2"] += dz.sum(0)
        dH = dz @ W_2.T
        # step 6: H = GELU(Vn W_1 + b_1)
        dHpre = dH * gelu_grad(it["Hpre"])
        g["W_1"] += it["Vn"].T @ dHpre
        g["b_1"] += dHpre.sum(0)
        dVn = dHpre @ W_1.T
        # step 5: Vn = LN2(Y)
        dY_ln, dg2, db2 = layer_norm_backward(it["Y"], g2, dVn)
        g["gamma2"] += dg2
        g["beta2"] += db2
        dY = dz + dY_ln
        # step 4: Y = X + O W_O
        g["W_O"] += it["O"].T @ dY
        dO = dY @ W_O.T
        # step 3: attention
        dQ, dK, dV = attention_backward(it["Q"], it["K"], it["V"], it["O"], dO, h, causal)
        # step 2: Q, K, V = U W
        g["W_Q"] += it["U"].T @ dQ
        g["W_K"] += it["U"].T @ dK
        g["W_V"] += it["U"].T @ dV
        dU = dQ @ W_Q.T + dK @ W_K.T + dV @ W_V.T
        # step 1: U = LN1(X)
        dX_ln, dg1, db1 = layer_norm_backward(X[b], g1, dU)
        g["gamma1"] += dg1
        g["beta1"] += db1
        g["x"][b] = dY + dX_ln
    return g


def layer_backward_blockwise(inp: Dict[str, np.ndarray], h: int, causal: bool,
                             dZ: np.ndarray, block: int) -> Dict[str, np.ndarray]:
    """The same gradients by the pages' block-recompute schedule.

    Saved from the forward: X and the per-row statistics (m, l)
    (``attention_stats_rows``).  Query block i recomputes o_i in one pass
    over its key blocks as sum_j exp(s_ij - m_i) v_j / l_i, then y_i, LN2,
    the FFN hidden, and consumes them: FFN and W_O gradients for its rows,
    dO_i, then per key block j the attention gradients with P_ij =
    exp(s_ij - m_i) / l_i.  dQ, dK, dV accumulate across blocks; the QKV
    projection and LN1 gradients follow.
    """
    dZ = np.asarray(dZ, dtype=np.float64)
    X = _as64(inp, "x")
    Bx, N, d = X.shape
    d_k = d // h
    scale = 1.0 / math.sqrt(d_k)
    W_Q, W_K, W_V, W_O, W_1, W_2 = (_as64(inp, k) for k in ("W_Q", "W_K", "W_V", "W_O", "W_1", "W_2"))
    b_1 = _as64(inp, "b_1")
    g1, be1, g2, be2 = (_as64(inp, k) for k in ("gamma1", "beta1", "gamma2", "beta2"))
    g = {k: np.zeros_like(_as64(inp, k)) for k in GRAD_NAMES}
    rows = np.array([(b, i) for b in range(Bx) for i in range(N)], dtype=np.int64)
    m_all, l_all = attention_stats_rows(inp, h, causal, rows)
    m_all, l_all = m_all.reshape(Bx, N, h), l_all.reshape(Bx, N, h)
    starts = list(range(0, N, block))
    for b in range(Bx):
        U = layer_norm(X[b], g1, be1)
        Q, K, V = U @ W_Q, U @ W_K, U @ W_V
        dQ, dK, dV = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V)
        dY_all = np.zeros_like(X[b])
        for i0 in starts:
            i1 = min(N, i0 + block)
            qi = np.arange(i0, i1)

            def probs(t, j0, j1):
                c = slice(t * d_k, (t + 1) * d_k)
                s = (Q[i0:i1, c] @ K[j0:j1, c].T) * scale
                if causal:
                    s = np.where(np.arange(j0, j1)[None, :] > qi[:, None], -np.inf, s)
                return np.exp(s - m_all[b, i0:i1, t][:, None]) / l_all[b, i0:i1, t][:, None]

            keys = [j0 for j0 in starts if not (causal and j0 > i0)]
            # recompute o_i in one pass from (m, l)
            o = np.zeros((i1 - i0, d))
            for t in range(h):
                c = slice(t * d_k, (t + 1) * d_k)
                for j0 in keys:
                    j1 = min(N, j0 + block)
                    o[:, c] += probs(t, j0, j1) @ V[j0:j1, c]
            y = X[b, i0:i1] + o @ W_O
            vn = layer_norm(y, g2, be2)
            hpre = vn @ W_1 + b_1
            hh = gelu(hpre)
            dz = dZ[b, i0:i1]
            g["W_2"] += hh.T @ dz
            g["b_2"] += dz.sum(0)
            dhpre = (dz @ W_2.T) * gelu_grad(hpre)
            g["W_1"] += vn.T @ dhpre
            g["b_1"] += dhpre.sum(0)
            dy_ln, dg2, db2 = layer_norm_backward(y, g2, dhpre @ W_1.T)
            g["gamma2"] += dg2
            g["beta2"] += db2
            dy = dz + dy_ln
            dY_all[i0:i1] = dy
            g["W_O"] += o.T @ dy
            do = dy @ W_O.T
            for t in range(h):
                c = slice(t * d_k, (t + 1) * d_k)
                D = (do[:, c] * o[:, c]).sum(axis=1, keepdims=True)
                for j0 in keys:
                    j1 = min(N, j0 + block)
                    p = probs(t, j0, j1)
                    dV[j0:j1, c] += p.T @ do[:, c]
                    ds = p * (do[:, c] @ V[j0:j1, c].T - D)
                    dQ[i0:i1, c] += ds @ K[j0:j1, c] * scale
                    dK[j0:j1, c] += ds.T @ Q[i0:i1, c] * scale
        g["W_Q"] += U.T @ dQ
        g["W_K"] += U.T @ dK
        g["W_V"] += U.T @ dV
        dU = dQ @ W_Q.T + dK @ W_K.T + dV @ W_V.T
        dX_ln, dg1, db1 = layer_norm_backward(X[b], g1, dU)
        g["gamma1"] += dg1
        g["beta1"] += db1
        g["x"][b] = dY_all + dX_ln
    return g
