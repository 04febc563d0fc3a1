"""The FLOP and byte accountant against the BPT page's printed numbers."""
import json
import os

from blockwise_attn_ffn_b200 import accounting as acc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "bpt_memory_example.json")


def load():
    with open(GOLDEN) as f:
        return json.load(f)


def test_worked_example_32k():
    g = load()["worked_example"]
    N, d, h, d_ff, eb, b = g["N"], g["d"], g["h"], g["d_ff"], g["elem_bytes"], g["block"]
    a = acc.unfused_activation_elems(N, d, h, d_ff)
    assert round(a["residual"] / 1e6, 1) == g["Nd_elems_millions"]
    assert round(a["residual"] * eb / 1e6) == g["Nd_MB"]
    assert round(a["ffn_hidden"] * eb / 1e6) == g["ffn_hidden_MB"]
    assert round(a["logits"] * eb / 1e9, 1) == g["logits_GB"]
    blk = acc.bpt_block_hidden_elems(b, d_ff)
    assert round(blk / 1e6, 1) == g["bpt_block_elems_millions"]
    assert round(blk * eb / 1e6, 1) == g["bpt_block_MB"]
    assert acc.hidden_reduction(N, b) == g["reduction"]
    assert round(g["layers"] * a["ffn_hidden"] * eb / 1e9, 1) == g["layers_ffn_GB_before"]
    assert round(g["layers"] * blk * eb / 1e9, 1) == g["layers_ffn_GB_after"]


def test_cpu_slm_tile():
    g = load()["cpu_slm"]
    hid = g["N"] * g["d_ff"] * g["elem_bytes"]
    assert round(hid / 1e6) == g["hidden_MB"]
    assert round(acc.bpt_block_hidden_elems(g["block"], g["d_ff"]) / 2 * g["elem_bytes"] / 1e6) == g["tile_MB"]


def test_flop_formulas_match_page():
    # d_ff = 4d, non-causal: attention 4N^2 d, QKVO 8Nd^2, FFN 16Nd^2
    N, d = 1000, 64
    f = acc.layer_flops(1, N, d, 4, 4 * d, causal=False)
    assert f["attention"] == 4 * N * N * d
    assert f["qkv"] + f["wo"] == 8 * N * d * d
    assert f["ffn"] == 16 * N * d * d
    # attention dominates when N > 6d
    d = load()["flops_crossover"]["d"]
    lo = acc.layer_flops(1, 6 * d - 8, d, 32, 4 * d, False)
    hi = acc.layer_flops(1, 6 * d + 8, d, 32, 4 * d, False)
    assert lo["attention"] < lo["qkv"] + lo["wo"] + lo["ffn"]
    assert hi["attention"] > hi["qkv"] + hi["wo"] + hi["ffn"]
    assert abs(6 * d - load()["flops_crossover"]["crossover_N_approx"]) < 1000


def test_causal_pairs_and_long_workload_total():
    assert acc.attention_pairs(4, True) == 10
    f = acc.layer_flops(1, 65536, 2048, 16, 8192, True)
    assert abs(f["total"] / 1e12 - 24.19) < 0.01


def test_attention_bytes_counts_q_k_v_and_o_once():
    # long-context layer: 65536 x 2048 16-bit values each for Q, K, V and o
    assert acc.attention_bytes(1, 65536, 2048, 16) == 4 * 65536 * 2048 * 2
    assert acc.attention_bytes(8, 2048, 768, 12) == 8 * acc.attention_bytes(1, 2048, 768, 12)
