"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test ties one part of ``oracle/`` to what the pages or the mathematics
fix: the two-tile running-sum identity printed on the transformer-cost page,
library routines (torch's layer_norm, gelu and scaled_dot_product_attention in
float64), closed forms, invariants the BPT page states (token-wise LN/FFN,
causal masking), pure-Python brute force on tiny inputs, and the pages' fused
schedule against the unfused definition.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from blockwise_attn_ffn_b200.inputs import LayerShape, WORKLOADS, make_inputs, sample_rows

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def tiny(N=24, d=16, h=2, d_ff=40, causal=True, seed=7, bias=0.3, ln=0.2, dtype="f32"):
    cfg = LayerShape("t", B=2, N=N, d=d, h=h, d_ff=d_ff, causal=causal,
                     dtype=dtype, block=8, seed=seed, ln_scale=ln, bias_scale=bias)
    return cfg, make_inputs(cfg)


# ---------------------------------------------------------------- softmax --
def test_two_tile_demo_from_page():
    """transformer-cost: one row of 8 scores in two tiles of 4; the rescaled
    tile sums equal the full sum (the page prints True for allclose)."""
    with open(os.path.join(GOLDEN, "two_tile_running_sum.json")) as f:
        g = json.load(f)
    rng = np.random.default_rng(g["seed"])
    for _ in range(g["trials"]):
        s = rng.standard_normal(2 * g["tile"])
        v = np.ones((s.size, 1))
        m, l, o = oracle.online_softmax_init(1, 1)
        for t in range(2):
            tile = s[t * g["tile"]:(t + 1) * g["tile"]]
            m, l, o = oracle.online_softmax_update(m, l, o, tile[None, :],
                                                   v[t * g["tile"]:(t + 1) * g["tile"]])
        # full sum of exp(s - max) by a plain accurate sum
        full = math.fsum(math.exp(x - max(s)) for x in s)
        assert bool(np.allclose(l[0], full)) is g["expected_allclose"]
        assert abs(l[0] - full) <= 1e-14 * full
        assert m[0] == max(s)


@pytest.mark.parametrize("seed", range(6))
def test_online_softmax_many_tiles(seed):
    """Random rows split into 2..8 tiles of 1..64 keys, some -inf entries:
    the online state equals softmax(s) @ v from torch (float64)."""
    rng = np.random.default_rng(100 + seed)
    rows, width = 5, 3
    n_tiles = rng.integers(2, 9)
    sizes = rng.integers(1, 65, size=n_tiles)
    n = int(sizes.sum())
    s = rng.standard_normal((rows, n)) * 4.0
    s[rng.random((rows, n)) < 0.2] = -np.inf
    s[:, 0] = rng.standard_normal(rows)           # every row keeps one finite key
    v = rng.standard_normal((n, width))
    m, l, o = oracle.online_softmax_init(rows, width)
    k0 = 0
    for sz in sizes:
        m, l, o = oracle.online_softmax_update(m, l, o, s[:, k0:k0 + sz], v[k0:k0 + sz])
        k0 += sz
    ref = torch.softmax(torch.from_numpy(s), dim=-1) @ torch.from_numpy(v)
    np.testing.assert_allclose(o / l[:, None], ref.numpy(), rtol=1e-13, atol=1e-14)
    ref_l = np.array([math.fsum(math.exp(x - np.max(r)) for x in r if np.isfinite(x)) for r in s])
    np.testing.assert_allclose(l * np.exp(m - s.max(axis=1)), ref_l, rtol=1e-13)


def test_online_softmax_leading_masked_tile():
    """A first tile that is fully -inf leaves the state untouched."""
    m, l, o = oracle.online_softmax_init(2, 2)
    m, l, o = oracle.online_softmax_update(m, l, o, np.full((2, 3), -np.inf), np.ones((3, 2)))
    assert np.all(np.isneginf(m)) and np.all(l == 0) and np.all(o == 0)
    m, l, o = oracle.online_softmax_update(m, l, o, np.array([[0.0], [1.0]]),
                                           np.array([[2.0, 3.0]]))
    np.testing.assert_array_equal(o / l[:, None], [[2.0, 3.0], [2.0, 3.0]])


def test_softmax_rows_vs_torch():
    rng = np.random.default_rng(3)
    S = rng.standard_normal((7, 33)) * 10
    S[2, 5:] = -np.inf
    np.testing.assert_allclose(oracle.softmax_rows(S),
                               torch.softmax(torch.from_numpy(S), -1).numpy(),
                               rtol=1e-14, atol=1e-300)


# ----------------------------------------------------------- LN and GELU --
def test_layer_norm_vs_torch():
    rng = np.random.default_rng(5)
    X = rng.standard_normal((9, 48)) * 3 + 1.5
    g = rng.standard_normal(48)
    b = rng.standard_normal(48)
    ref = F.layer_norm(torch.from_numpy(X), (48,), torch.from_numpy(g),
                       torch.from_numpy(b), eps=1e-5)
    np.testing.assert_allclose(oracle.layer_norm(X, g, b), ref.numpy(), rtol=1e-12, atol=1e-12)


def test_layer_norm_constant_row_gives_beta():
    g = np.linspace(0.5, 2, 16)
    b = np.linspace(-1, 1, 16)
    out = oracle.layer_norm(np.full((3, 16), 4.25), g, b)
    np.testing.assert_array_equal(out, np.broadcast_to(b, (3, 16)))


def test_gelu_vs_torch_and_erf():
    z = np.linspace(-8, 8, 1001)
    ref = F.gelu(torch.from_numpy(z), approximate="none").numpy()
    np.testing.assert_allclose(oracle.gelu(z), ref, rtol=1e-14, atol=1e-15)
    for v in (-3.0, -0.5, 0.25, 1.0, 2.5):
        assert abs(oracle.gelu(np.array(v)) - 0.5 * v * (1 + math.erf(v / math.sqrt(2)))) < 1e-15
    assert oracle.gelu(np.array(0.0)) == 0.0
    # the tanh form differs by far more than the oracle's error
    tanh_form = 0.5 * z * (1 + np.tanh(math.sqrt(2 / math.pi) * (z + 0.044715 * z ** 3)))
    assert np.max(np.abs(tanh_form - oracle.gelu(z))) > 1e-4


# ------------------------------------------------------------- attention --
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("h", [1, 2, 4])
def test_attention_vs_sdpa(causal, h):
    rng = np.random.default_rng(11 + h)
    N, d = 37, 8 * h
    Q, K, V = (rng.standard_normal((N, d)) for _ in range(3))
    got = oracle.attention_rows(Q, K, V, h, causal, np.arange(N))
    t = lambda a: torch.from_numpy(a).reshape(N, h, d // h).transpose(0, 1)
    ref = F.scaled_dot_product_attention(t(Q), t(K), t(V), is_causal=causal)
    ref = ref.transpose(0, 1).reshape(N, d).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


# ------------------------------------------------------------ whole layer --
def torch_layer(inp, h, causal):
    """The layer composed of torch float64 library routines."""
    T = lambda k: torch.from_numpy(np.asarray(inp[k], np.float64))
    X = T("x")
    Bx, N, d = X.shape
    d_k = d // h
    U = F.layer_norm(X, (d,), T("gamma1"), T("beta1"), eps=1e-5)
    heads = lambda A: A.reshape(Bx, N, h, d_k).transpose(1, 2)
    O = F.scaled_dot_product_attention(heads(U @ T("W_Q")), heads(U @ T("W_K")),
                                       heads(U @ T("W_V")), is_causal=causal)
    Y = X + O.transpose(1, 2).reshape(Bx, N, d) @ T("W_O")
    Hh = F.gelu(F.layer_norm(Y, (d,), T("gamma2"), T("beta2"), eps=1e-5) @ T("W_1") + T("b_1"))
    return (Y + Hh @ T("W_2") + T("b_2")).numpy()


@pytest.mark.parametrize("causal", [False, True])
def test_layer_vs_torch_library_composition(causal):
    cfg, inp = tiny(N=45, d=32, h=4, d_ff=96, causal=causal)
    np.testing.assert_allclose(oracle.layer_unfused(inp, cfg.h, causal),
                               torch_layer(inp, cfg.h, causal), rtol=1e-11, atol=1e-11)


def scalar_layer(inp, h, causal):
    """Pure-Python loops, no numpy arithmetic: the layer on tiny inputs."""
    L = lambda k: np.asarray(inp[k], np.float64).tolist()
    X = L("x")
    WQ, WK, WV, WO, W1, b1, W2, b2 = (L(k) for k in ("W_Q", "W_K", "W_V", "W_O", "W_1", "b_1", "W_2", "b_2"))
    g1, be1, g2, be2 = (L(k) for k in ("gamma1", "beta1", "gamma2", "beta2"))
    d, d_ff = len(WQ), len(b1)
    d_k = d // h

    def ln(row, g, be):
        mu = sum(row) / len(row)
        var = sum((a - mu) ** 2 for a in row) / len(row)
        return [(a - mu) / math.sqrt(var + 1e-5) * g[k] + be[k] for k, a in enumerate(row)]

    def vecmat(v, W):
        return [sum(v[i] * W[i][j] for i in range(len(v))) for j in range(len(W[0]))]

    out = []
    for Xb in X:
        N = len(Xb)
        U = [ln(r, g1, be1) for r in Xb]
        Q = [vecmat(u, WQ) for u in U]
        K = [vecmat(u, WK) for u in U]
        V = [vecmat(u, WV) for u in U]
        Zb = []
        for i in range(N):
            o = [0.0] * d
            for t in range(h):
                cols = range(t * d_k, (t + 1) * d_k)
                keys = range(i + 1) if causal else range(N)
                sc = {j: sum(Q[i][c] * K[j][c] for c in cols) / math.sqrt(d_k) for j in keys}
                mx = max(sc.values())
                w = {j: math.exp(s - mx) for j, s in sc.items()}
                tot = sum(w.values())
                for c in cols:
                    o[c] = sum(w[j] * V[j][c] for j in keys) / tot
            y = [Xb[i][c] + a for c, a in enumerate(vecmat(o, WO))]
            hid = vecmat(ln(y, g2, be2), W1)
            hid = [0.5 * (z + b1[k]) * (1 + math.erf((z + b1[k]) / math.sqrt(2))) for k, z in enumerate(hid)]
            f = vecmat(hid, W2)
            Zb.append([y[c] + f[c] + b2[c] for c in range(d)])
        out.append(Zb)
    return np.array(out)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 4, 1, 8), (5, 6, 2, 12), (8, 8, 2, 16)])
def test_layer_vs_scalar_brute_force(causal, shape):
    N, d, h, d_ff = shape
    cfg, inp = tiny(N=N, d=d, h=h, d_ff=d_ff, causal=causal, seed=N + d)
    np.testing.assert_allclose(oracle.layer_unfused(inp, h, causal),
                               scalar_layer(inp, h, causal), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("block", [1, 3, 64, 8])
def test_blockwise_schedule_equals_unfused(causal, block):
    """The pages' fused two-level loop reaches the unfused result (fp64)."""
    cfg, inp = tiny(N=29, d=24, h=3, d_ff=48, causal=causal)
    a = oracle.layer_blockwise(inp, cfg.h, causal, block)
    b = oracle.layer_unfused(inp, cfg.h, causal)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------- invariants --
def test_permutation_equivariance_noncausal():
    cfg, inp = tiny(N=20, causal=False)
    perm = np.random.default_rng(1).permutation(cfg.N)
    pin = dict(inp)
    pin["x"] = inp["x"][:, perm]
    np.testing.assert_allclose(oracle.layer_unfused(pin, cfg.h, False),
                               oracle.layer_unfused(inp, cfg.h, False)[:, perm],
                               rtol=1e-12, atol=1e-12)


def test_causal_rows_before_a_change_are_untouched():
    cfg, inp = tiny(N=20, causal=True)
    base = oracle.layer_unfused(inp, cfg.h, True)
    for r in (0, 7, 19):
        pin = dict(inp)
        pin["x"] = inp["x"].copy()
        pin["x"][0, r] += 1.0
        z = oracle.layer_unfused(pin, cfg.h, True)
        np.testing.assert_array_equal(z[0, :r], base[0, :r])
        assert np.all(np.abs(z[0, r:] - base[0, r:]).max(axis=-1) > 0)
        np.testing.assert_array_equal(z[1], base[1])   # other batch element


def test_ffn_half_is_token_wise():
    cfg, inp = tiny(N=12)
    Y = np.random.default_rng(9).standard_normal((12, cfg.d))
    base = oracle.ffn_residual(Y, inp)
    Y2 = Y.copy()
    Y2[5] += 0.5
    z = oracle.ffn_residual(Y2, inp)
    np.testing.assert_array_equal(np.delete(z, 5, 0), np.delete(base, 5, 0))
    assert np.abs(z[5] - base[5]).max() > 0


# ----------------------------------------------------------- closed forms --
@pytest.mark.parametrize("causal", [False, True])
def test_zero_WQ_gives_uniform_attention(causal):
    cfg, inp = tiny(N=15, causal=causal)
    inp = dict(inp, W_Q=np.zeros_like(inp["W_Q"]))
    it = oracle.layer_intermediates(inp, cfg.h, causal)
    V = it["V"]
    if causal:
        expect = np.cumsum(V, axis=0) / np.arange(1, cfg.N + 1)[:, None]
    else:
        expect = np.broadcast_to(V.mean(axis=0), V.shape)
    np.testing.assert_allclose(it["O"], expect, rtol=1e-12, atol=1e-13)


def test_zero_WV_gives_Y_equal_X():
    cfg, inp = tiny()
    inp = dict(inp, W_V=np.zeros_like(inp["W_V"]))
    it = oracle.layer_intermediates(inp, cfg.h, True)
    np.testing.assert_array_equal(it["Y"], inp["x"][0].astype(np.float64))


def test_zero_W1_gives_Z_equal_Y_plus_b2():
    cfg, inp = tiny()
    inp = dict(inp, W_1=np.zeros_like(inp["W_1"]), b_1=np.zeros_like(inp["b_1"]))
    it = oracle.layer_intermediates(inp, cfg.h, True)
    np.testing.assert_array_equal(it["Z"], it["Y"] + inp["b_2"].astype(np.float64))


def test_single_token_attention_is_V():
    cfg, inp = tiny(N=1)
    it = oracle.layer_intermediates(inp, cfg.h, False)
    np.testing.assert_allclose(it["O"], it["V"], rtol=1e-15, atol=0)


# ------------------------------------------------- every intermediate ----
def torch_intermediates(inp, h, causal, b):
    """Steps 1-7 of batch element b, each formed from torch float64 library
    routines (layer_norm, matmul, scaled_dot_product_attention, gelu)."""
    T = lambda k: torch.from_numpy(np.asarray(inp[k], np.float64))
    X = T("x")[b]
    N, d = X.shape
    d_k = d // h
    U = F.layer_norm(X, (d,), T("gamma1"), T("beta1"), eps=1e-5)
    Q, K, V = U @ T("W_Q"), U @ T("W_K"), U @ T("W_V")
    heads = lambda A: A.reshape(N, h, d_k).transpose(0, 1)
    O = F.scaled_dot_product_attention(heads(Q), heads(K), heads(V), is_causal=causal)
    O = O.transpose(0, 1).reshape(N, d)
    Y = X + O @ T("W_O")
    Vn = F.layer_norm(Y, (d,), T("gamma2"), T("beta2"), eps=1e-5)
    Hpre = Vn @ T("W_1") + T("b_1")
    H = F.gelu(Hpre)
    Z = Y + H @ T("W_2") + T("b_2")
    return {k: v.numpy() for k, v in dict(U=U, Q=Q, K=K, V=V, O=O, Y=Y, Vn=Vn, Hpre=Hpre,
                                          H=H, Z=Z).items()}


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("b", [0, 1])
def test_layer_intermediates_vs_torch_library(causal, b):
    """Every intermediate (the oracle the GPU's Q/K/V are compared with) equals
    the torch float64 library composition, with non-zero biases and LN
    parameters away from (1, 0), so a swapped weight, a swapped LN parameter
    or a dropped bias changes some key by far more than the tolerance."""
    cfg, inp = tiny(N=37, d=32, h=4, d_ff=96, causal=causal, bias=0.5, ln=0.4)
    got = oracle.layer_intermediates(inp, cfg.h, causal, b=b)
    want = torch_intermediates(inp, cfg.h, causal, b)
    assert sorted(got) == sorted(want)
    for k in want:
        np.testing.assert_allclose(got[k], want[k], rtol=1e-11, atol=1e-11, err_msg=k)
    # and the last step is the oracle's plain definition of the layer
    np.testing.assert_allclose(got["Z"], oracle.layer_unfused(inp, cfg.h, causal)[b],
                               rtol=1e-12, atol=1e-12)


def test_layer_intermediates_distinguish_the_projections():
    """Guards the comparison above against a fixture in which the three
    projections (or the two LayerNorms) would coincide."""
    cfg, inp = tiny(N=9, d=16, h=2, d_ff=32, bias=0.5, ln=0.4)
    it = oracle.layer_intermediates(inp, cfg.h, True)
    for a, c in (("Q", "K"), ("K", "V"), ("Q", "V")):
        assert np.abs(it[a] - it[c]).max() > 0.1
    assert np.abs(inp["gamma1"] - inp["gamma2"]).max() > 0.1
    assert np.abs(inp["b_1"]).max() > 0.1


# -------------------------------------------------------- sampled rows ----
@pytest.mark.parametrize("causal", [False, True])
def test_layer_rows_equals_full_layer_small(causal):
    cfg, inp = tiny(N=70, d=32, h=2, d_ff=64, causal=causal)
    rows = np.array([[0, 0], [0, 7], [0, 69], [1, 33], [1, 0]])
    full = oracle.layer_unfused(inp, cfg.h, causal)
    np.testing.assert_allclose(oracle.layer_rows(inp, cfg.h, causal, rows),
                               full[rows[:, 0], rows[:, 1]], rtol=1e-12, atol=1e-12)


def test_layer_rows_equals_full_layer_gpt2_shape():
    """The GPT-2-small-shaped workload (first batch element): sampled rows
    reproduce the full computation's rows."""
    cfg = WORKLOADS["gpt2s_n2k"]
    inp = make_inputs(cfg, B=1)
    rows = sample_rows(cfg, 64, B=1)
    full = oracle.layer_unfused(inp, cfg.h, cfg.causal)
    np.testing.assert_allclose(oracle.layer_rows(inp, cfg.h, cfg.causal, rows),
                               full[rows[:, 0], rows[:, 1]], rtol=1e-12, atol=1e-12)


def test_sample_rows_recipe():
    cfg = WORKLOADS["long_n64k"]
    r = sample_rows(cfg, 256)
    assert r.shape == (256, 2)
    assert len({tuple(x) for x in r.tolist()}) == 256
    for must in (0, 127, 128, cfg.N - 1):
        assert [0, must] in r.tolist()
    np.testing.assert_array_equal(r, sample_rows(cfg, 256))
