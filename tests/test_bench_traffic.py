"""The bench line's `roofline.traffic` comes from a recorded ncu capture of
the attention kernel (DRAM read + write bytes of one launch), valid only
while the attention sources it was taken on are unchanged: the bench hashes
them and reports null on a mismatch.  This test keeps the committed record
and the committed sources in step, so a change to the attention kernel, its
device helpers or its launch fails here until the capture is taken again."""
import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def load_bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_recorded_attention_traffic_matches_the_sources():
    bench = load_bench()
    entry = bench.ATTN_TRAFFIC["long_n64k"]
    assert entry["digest"] == bench.sources_digest(), \
        "attention sources changed since the recorded ncu capture: take it again"
    got = bench.attn_traffic("long_n64k")
    # at least Q, K, V read and o written once (8 N d bytes at N = 65536, d = 2048)
    assert got == entry["bytes_per_launch"] and got >= 8 * 65536 * 2048


def test_digest_ignores_the_layer_body_launch():
    """The digest spans the attention launch only: text after the fused
    attention call (the layer body's launch) is outside it."""
    bench = load_bench()
    with open(os.path.join(ROOT, bench.TRAFFIC_API)) as f:
        api = f.read()
    a = api.index("// attention over every query block")
    end = api.index("int dummy = 0, pairs_max = 0;", a)
    assert "tail_pair_kernel" not in api[a:end]
    assert "launch_attn(" in api[a:end]
