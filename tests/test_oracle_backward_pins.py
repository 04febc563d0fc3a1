"""Pins of the backward oracle (``oracle.layer_backward`` and the pages'
block-recompute schedule ``oracle.layer_backward_blockwise``).

BPT page, section "The backward pass".  Pinned against torch autograd over a
layer composed of torch float64 library routines (independent of the
oracle's hand-written chain rule), central finite differences of the
oracle's own forward, closed forms, and the unfused == blockwise identity.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from blockwise_attn_ffn_b200.inputs import LayerShape, make_inputs

PARAMS = ["W_Q", "W_K", "W_V", "W_O", "W_1", "b_1", "W_2", "b_2",
          "gamma1", "beta1", "gamma2", "beta2"]


def tiny(N=24, d=16, h=2, d_ff=40, causal=True, seed=7, B=2):
    cfg = LayerShape("t", B=B, N=N, d=d, h=h, d_ff=d_ff, causal=causal, dtype="f32", block=8,
                     seed=seed, ln_scale=0.2, bias_scale=0.3)
    return cfg, make_inputs(cfg)


def upstream(cfg, seed=99):
    return np.random.default_rng(seed).standard_normal((cfg.B, cfg.N, cfg.d))


def torch_grads(inp, h, causal, dZ):
    """Gradients of sum(Z * dZ) by torch autograd over library routines."""
    T = {k: torch.tensor(np.asarray(inp[k], np.float64), requires_grad=True)
         for k in ["x"] + PARAMS}
    X = T["x"]
    Bx, N, d = X.shape
    d_k = d // h
    U = F.layer_norm(X, (d,), T["gamma1"], T["beta1"], eps=1e-5)
    heads = lambda A: A.reshape(Bx, N, h, d_k).transpose(1, 2)
    O = F.scaled_dot_product_attention(heads(U @ T["W_Q"]), heads(U @ T["W_K"]),
                                       heads(U @ T["W_V"]), is_causal=causal)
    Y = X + O.transpose(1, 2).reshape(Bx, N, d) @ T["W_O"]
    Hh = F.gelu(F.layer_norm(Y, (d,), T["gamma2"], T["beta2"], eps=1e-5) @ T["W_1"] + T["b_1"])
    Z = Y + Hh @ T["W_2"] + T["b_2"]
    (Z * torch.from_numpy(dZ)).sum().backward()
    return {k: v.grad.numpy() for k, v in T.items()}


@pytest.mark.parametrize("causal", [False, True])
def test_backward_vs_torch_autograd(causal):
    cfg, inp = tiny(N=29, d=32, h=4, d_ff=72, causal=causal)
    dZ = upstream(cfg)
    got = oracle.layer_backward(inp, cfg.h, causal, dZ)
    want = torch_grads(inp, cfg.h, causal, dZ)
    for k in ["x"] + PARAMS:
        np.testing.assert_allclose(got[k], want[k], rtol=1e-10, atol=1e-10, err_msg=k)


def test_backward_vs_central_differences():
    """d/de sum(Z(theta + e u) * dZ) at e = 0 equals <grad, u>, for a random
    direction u in x and in each parameter (the oracle's own forward)."""
    cfg, inp = tiny(N=11, d=8, h=2, d_ff=20, causal=True, B=1)
    dZ = upstream(cfg)
    g = oracle.layer_backward(inp, cfg.h, True, dZ)
    rng = np.random.default_rng(5)
    eps = 1e-5
    for k in ["x"] + PARAMS:
        u = rng.standard_normal(np.shape(inp[k]))
        plus, minus = dict(inp), dict(inp)
        plus[k] = np.asarray(inp[k], np.float64) + eps * u
        minus[k] = np.asarray(inp[k], np.float64) - eps * u
        fd = ((oracle.layer_unfused(plus, cfg.h, True) - oracle.layer_unfused(minus, cfg.h, True))
              * dZ).sum() / (2 * eps)
        assert (g[k] * u).sum() == pytest.approx(fd, rel=1e-6, abs=1e-8), k


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("block", [1, 5, 8, 64])
def test_blockwise_backward_equals_unfused(causal, block):
    cfg, inp = tiny(N=23, d=16, h=2, d_ff=40, causal=causal)
    dZ = upstream(cfg)
    a = oracle.layer_backward(inp, cfg.h, causal, dZ)
    b = oracle.layer_backward_blockwise(inp, cfg.h, causal, dZ, block)
    for k in ["x"] + PARAMS:
        np.testing.assert_allclose(b[k], a[k], rtol=1e-10, atol=1e-11, err_msg=k)


def test_zero_upstream_gives_zero_gradients():
    cfg, inp = tiny()
    g = oracle.layer_backward(inp, cfg.h, True, np.zeros((cfg.B, cfg.N, cfg.d)))
    for k, v in g.items():
        assert np.all(v == 0.0), k


def test_b2_gradient_is_the_summed_upstream_and_x_gets_it_through_the_residual():
    """Z = Y + ... + b_2: d b_2 = sum over rows of dZ.  With W_O = 0 and W_2 = 0
    (so Z = X + b_2 + 0 * ...) every row's dx equals its dZ."""
    cfg, inp = tiny()
    dZ = upstream(cfg)
    g = oracle.layer_backward(inp, cfg.h, True, dZ)
    np.testing.assert_allclose(g["b_2"], dZ.reshape(-1, cfg.d).sum(0), rtol=1e-13, atol=1e-13)
    inp2 = dict(inp)
    inp2["W_O"] = np.zeros_like(inp["W_O"])
    inp2["W_2"] = np.zeros_like(inp["W_2"])
    g2 = oracle.layer_backward(inp2, cfg.h, True, dZ)
    np.testing.assert_allclose(g2["x"], dZ, rtol=1e-13, atol=1e-13)
    for k in ["W_Q", "W_K", "W_V", "W_1", "b_1", "gamma1", "beta1", "gamma2", "beta2"]:
        assert np.all(g2[k] == 0.0), k


def test_layer_norm_backward_vs_torch():
    rng = np.random.default_rng(3)
    X = rng.standard_normal((7, 33)) * 3 + 1
    gam, dY = rng.standard_normal(33), rng.standard_normal((7, 33))
    dX, dg, db = oracle.layer_norm_backward(X, gam, dY)
    Xt = torch.tensor(X, requires_grad=True)
    gt = torch.tensor(gam, requires_grad=True)
    bt = torch.zeros(33, dtype=torch.float64, requires_grad=True)
    (F.layer_norm(Xt, (33,), gt, bt, eps=1e-5) * torch.from_numpy(dY)).sum().backward()
    np.testing.assert_allclose(dX, Xt.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dg, gt.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(db, bt.grad.numpy(), rtol=1e-12, atol=1e-12)


def test_gelu_grad_vs_torch():
    z = np.linspace(-6, 6, 241)
    zt = torch.tensor(z, requires_grad=True)
    F.gelu(zt).sum().backward()
    np.testing.assert_allclose(oracle.gelu_grad(z), zt.grad.numpy(), rtol=1e-13, atol=1e-14)
