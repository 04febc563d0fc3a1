"""The C-ABI boundary on the host (no GPU needed).

The library loads, exports every function include/bpt.h declares, and rejects
bad arguments with the documented status before it touches the GPU.  The
workspace query is pure arithmetic, so its block-shaped growth is checked
here too.
"""
import ctypes
import os
import re

import pytest

import blockwise_attn_ffn_b200 as bpt
from blockwise_attn_ffn_b200 import build as bbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def lib():
    bbuild.build()
    return bpt.load()


def header_functions():
    src = open(os.path.join(ROOT, "include", "bpt.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bpt_[a-z_0-9]+)\s*\(", src)))


def test_every_declared_function_is_exported(lib):
    names = header_functions()
    assert "bpt_layer_forward" in names and "bpt_layer_workspace_size" in names
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(bpt.EXPORTED) == names


def test_status_strings():
    for s in range(7):
        assert bpt.status_string(s).startswith("BPT_")
    assert "UNKNOWN" in bpt.status_string(99)


BF, F32 = bpt.BPT_BF16, bpt.BPT_F32


@pytest.mark.parametrize("args,expect", [
    ((1, 256, 64, 1, 256, 0, F32), bpt.BPT_OK),
    ((8, 2048, 768, 12, 3072, 1, BF), bpt.BPT_OK),
    ((1, 300, 256, 4, 512, 1, BF), bpt.BPT_OK),            # ragged N
    ((1, 256, 100, 3, 256, 1, BF), bpt.BPT_ERR_INVALID_ARG),  # d % h
    ((1, 256, 96, 3, 256, 1, BF), bpt.BPT_ERR_UNSUPPORTED),   # d_k = 32
    ((1, 256, 256, 1, 512, 1, BF), bpt.BPT_ERR_UNSUPPORTED),  # d_k = 256
    ((1, 256, 256, 2, 500, 1, BF), bpt.BPT_ERR_UNSUPPORTED),  # d_ff % 64
    ((1, 256, 64, 1, 256, 0, 7), bpt.BPT_ERR_INVALID_ARG),    # dtype
    ((-1, 256, 64, 1, 256, 0, F32), bpt.BPT_ERR_INVALID_ARG),
    ((1, 256, 0, 1, 256, 0, F32), bpt.BPT_ERR_INVALID_ARG),
    ((1, 256, 1024, 4, 256, 0, F32), bpt.BPT_ERR_UNSUPPORTED),  # fp32 d_k = 256
])
def test_workspace_size_validation(args, expect):
    st, nbytes = bpt.bpt_layer_workspace_size(*args)
    assert st == expect
    if st == bpt.BPT_OK:
        assert nbytes > 0


def test_workspace_null_out_pointer(lib):
    assert lib.bpt_layer_workspace_size(1, 256, 64, 1, 256, 0, F32, None) == bpt.BPT_ERR_INVALID_ARG


def test_workspace_is_block_shaped():
    """Fused schedule: beyond the fp16 weights and the QKV projection (3 B N d
    elements) the workspace is at most 148 query blocks x b x (2d + 2 d_ff)
    bytes (LN2(y) and the FFN hidden of the blocks in flight) for EVERY N,
    and constant once the layer has that many blocks."""
    d, h, d_ff = 2048, 16, 8192
    weights = (4 * d * d + 2 * d * d_ff) * 2
    bound = 2 * bpt.BPT_TAIL_MAX_PAIRS * 128 * (2 * d + 2 * d_ff)
    extra = {}
    for B, N in ((1, 128), (1, 1000), (1, 8192), (1, 16384), (1, 32768), (1, 65536),
                 (1, 131072), (4, 65536), (64, 2048)):
        st, nbytes = bpt.bpt_layer_workspace_size(B, N, d, h, d_ff, 1, BF)
        assert st == bpt.BPT_OK
        e = nbytes - 3 * B * N * d * 2 - weights
        assert 0 < e <= bound + 4096, (B, N, e)
        blocks = B * ((N + 127) // 128)
        # never more than the blocks the layer has (2 per CTA pair, rounded up)
        assert e <= ((blocks + 1) // 2) * 256 * (2 * d + 2 * d_ff) + 4096, (B, N, e)
        extra[(B, N)] = e
    full = [e for (B, N), e in extra.items() if B * N >= 128 * 148]
    assert max(full) - min(full) <= 4096           # alignment slack only


def test_waves_workspace_is_wave_shaped():
    """Waves schedule: the scratch stops growing with N once a wave is full."""
    d, h, d_ff = 2048, 16, 8192
    weights = (4 * d * d + 2 * d * d_ff) * 2
    extra = []
    for N in (8192, 16384, 32768, 65536, 131072):
        st, nbytes = bpt.bpt_layer_workspace_size_opt(1, N, d, h, d_ff, 1, BF,
                                                      {"schedule": "waves"})
        assert st == bpt.BPT_OK
        extra.append(nbytes - 3 * N * d * 2 - weights)
    full = extra[2:]
    assert max(full) - min(full) <= 2048           # alignment slack only
    assert all(e <= max(full) for e in extra)
    bound = bpt.BPT_WAVE_BLOCKS * 128 * (2 * d + d_ff) * 2
    assert max(full) <= bound + 8192


def test_options_validation():
    ok = bpt.bpt_layer_workspace_size_opt
    args = (1, 1024, 256, 2, 512, 1, BF)
    assert ok(*args, None)[0] == bpt.BPT_OK
    assert ok(*args, None) == bpt.bpt_layer_workspace_size(*args)
    assert ok(*args, {})[1] == ok(*args, None)[1]            # zeroed struct = defaults
    for bad in ({"schedule": 2}, {"schedule": -1}, {"attn_block": 3}, {"max_wave": -1},
                {"max_wave": bpt.BPT_WAVE_BLOCKS + 1}, {"fault": 4}, {"reserved": 1}):
        assert ok(*args, bad)[0] == bpt.BPT_ERR_INVALID_ARG, bad
    # the wave size only shapes the waves schedule's scratch
    assert ok(*args, {"max_wave": 2})[1] == ok(*args, None)[1]
    assert (ok(*args, {"schedule": "waves", "max_wave": 2})[1]
            < ok(*args, {"schedule": "waves"})[1])
    # fp32 layers ignore the schedule
    f = (1, 256, 64, 1, 256, 0, F32)
    assert ok(*f, {"schedule": "waves"}) == ok(*f, None)


def test_launch_count():
    # fused: weight copy, LN1, QKV, attention, layer body
    st, n = bpt.bpt_layer_launch_count(1, 65536, 2048, 16, 8192, 1, BF)
    assert st == bpt.BPT_OK and n == 5
    waves = {"schedule": "waves"}
    st, n = bpt.bpt_layer_launch_count_opt(1, 65536, 2048, 16, 8192, 1, BF, waves)
    assert st == bpt.BPT_OK and n == 3 + 5 * 2   # weight copy, LN1, QKV; two waves
    st, n = bpt.bpt_layer_launch_count_opt(8, 2048, 768, 12, 3072, 1, BF, waves)
    assert st == bpt.BPT_OK and n == 3 + 5      # one wave of 8 sequences
    st, n = bpt.bpt_layer_launch_count(1, 256, 64, 1, 256, 0, F32)
    assert st == bpt.BPT_OK and n == 2 + 5      # fp32: no weight copy
    st, n = bpt.bpt_layer_launch_count(0, 2048, 768, 12, 3072, 1, BF)
    assert st == bpt.BPT_OK and n == 0


def fwd(ptrs, B=1, N=256, d=256, h=2, d_ff=512, causal=1, dtype=BF, ws_bytes=1 << 30):
    return bpt.bpt_layer_forward(*ptrs[:11], B, N, d, h, d_ff, causal, dtype, ptrs[11],
                                 ptrs[12], ws_bytes, None)


# Fake, never-dereferenced addresses: validation must fail before any use.
GOOD = [0x10000000 + i * 0x1000000 for i in range(13)]


def test_forward_rejects_null_pointers():
    for i in range(13):
        p = list(GOOD)
        p[i] = None
        assert fwd(p) == bpt.BPT_ERR_INVALID_ARG, i


def test_forward_rejects_misaligned_pointers():
    for i in range(13):
        p = list(GOOD)
        p[i] += 8
        assert fwd(p) == bpt.BPT_ERR_INVALID_ARG, i


def test_forward_rejects_small_workspace():
    st, need = bpt.bpt_layer_workspace_size(1, 256, 256, 2, 512, 1, BF)
    assert fwd(GOOD, ws_bytes=need - 1) == bpt.BPT_ERR_WORKSPACE


def test_forward_rejects_aliasing_out_and_x():
    p = list(GOOD)
    p[11] = p[0]
    assert fwd(p) == bpt.BPT_ERR_INVALID_ARG


@pytest.mark.parametrize("i", range(1, 11))
def test_forward_rejects_out_or_workspace_over_any_parameter(i):
    """out and the workspace are written while every parameter is still read."""
    p = list(GOOD)
    p[11] = p[i] + 16          # out starting inside parameter i
    assert fwd(p) == bpt.BPT_ERR_INVALID_ARG
    p = list(GOOD)
    p[i] = p[12] + 4096        # parameter i inside the workspace
    assert fwd(p) == bpt.BPT_ERR_INVALID_ARG


def test_forward_rejects_workspace_over_x_or_out():
    p = list(GOOD)
    p[12] = p[0] + 1024        # workspace starting inside x
    assert fwd(p) == bpt.BPT_ERR_INVALID_ARG
    p = list(GOOD)
    p[12] = p[11] + 1024       # workspace starting inside out
    assert fwd(p) == bpt.BPT_ERR_INVALID_ARG


def test_forward_rejects_unsupported_shapes():
    assert fwd(GOOD, d=96, h=3) == bpt.BPT_ERR_UNSUPPORTED
    assert fwd(GOOD, d=100, h=3) == bpt.BPT_ERR_INVALID_ARG


def test_forward_empty_is_a_no_op():
    assert fwd([None] * 13, B=0) == bpt.BPT_OK
    assert fwd([None] * 13, N=0) == bpt.BPT_OK


def test_read_error_null_means_the_static_array():
    """NULL selects the allocation-free entry point's array; with no GPU its
    address cannot be looked up, which is reported, not dereferenced."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("covered by the GPU test of the allocation-free entry point")
    st, _ = bpt.bpt_read_device_error(None, None)
    assert st == bpt.BPT_ERR_CUDA


def test_library_has_no_host_fallback_symbols(lib):
    """The library exports only the C ABI: no second implementation."""
    out = os.popen(f"nm -D --defined-only {bpt.LIB_PATH}").read()
    exported = sorted(set(re.findall(r" T (bpt_\w+)", out)))
    assert exported == header_functions()


def fwd_bsfa(ptrs, thr=0x70000000, bmax=0x71000000, kept=0x72000000, B=1, N=256, d=256, h=2,
             d_ff=512, causal=1, dtype=BF, ws_bytes=1 << 30):
    return bpt.bpt_layer_forward_bsfa(*ptrs[:11], B, N, d, h, d_ff, causal, dtype, thr, bmax,
                                      kept, ptrs[11], ptrs[12], ws_bytes, None)


def test_bsfa_rejects_bad_gate_buffers():
    assert fwd_bsfa(GOOD, thr=None) == bpt.BPT_ERR_INVALID_ARG
    assert fwd_bsfa(GOOD, thr=0x70000002) == bpt.BPT_ERR_INVALID_ARG      # misaligned
    assert fwd_bsfa(GOOD, bmax=0x71000002) == bpt.BPT_ERR_INVALID_ARG     # misaligned
    assert fwd_bsfa(GOOD, thr=GOOD[11]) == bpt.BPT_ERR_INVALID_ARG        # overlaps out
    assert fwd_bsfa(GOOD, thr=GOOD[12] + 64) == bpt.BPT_ERR_INVALID_ARG   # in the workspace
    assert fwd_bsfa(GOOD, bmax=GOOD[0]) == bpt.BPT_ERR_INVALID_ARG        # overlaps x
    assert fwd_bsfa(GOOD, kept=0x71000001) == bpt.BPT_ERR_INVALID_ARG     # inside block_max
    assert fwd_bsfa(GOOD, dtype=F32) == bpt.BPT_ERR_UNSUPPORTED
    assert fwd_bsfa(GOOD, d=96, h=3) == bpt.BPT_ERR_UNSUPPORTED
    p = list(GOOD)
    p[3] = None
    assert fwd_bsfa(p) == bpt.BPT_ERR_INVALID_ARG                          # a null weight


def test_bsfa_empty_is_a_no_op():
    assert fwd_bsfa([None] * 13, B=0) == bpt.BPT_OK
    assert fwd_bsfa([None] * 13, N=0) == bpt.BPT_OK


# ------------------------------------------------------------- backward ABI
def bwd(ins, outs, ws_bytes=1 << 31, B=1, N=256, d=64, h=1, d_ff=256, causal=1, dtype=F32):
    """ins: 14 fake pointers (x, ln1, W_Q..b_2, stats, dZ, workspace); outs: 11."""
    return bpt.bpt_layer_backward(*ins[:13], B, N, d, h, d_ff, causal, dtype, *outs, ins[13],
                                  ws_bytes, None)


BWD_IN = [0x10000000 + i * 0x1000000 for i in range(13)] + [0x80000000]
BWD_OUT = [0x30000000 + i * 0x1000000 for i in range(11)]


@pytest.mark.parametrize("dtype", [BF, F32])
def test_backward_workspace_size_for_both_dtypes(dtype):
    st, small_ws = bpt.bpt_layer_backward_workspace_size(1, 256, 256, 2, 512, 1, dtype)
    assert st == bpt.BPT_OK and small_ws > 0
    st, big_ws = bpt.bpt_layer_backward_workspace_size(1, 4096, 256, 2, 512, 1, dtype)
    assert st == bpt.BPT_OK and big_ws > small_ws
    assert bpt.bpt_layer_backward_workspace_size(1, 256, 100, 3, 512, 1, dtype)[0] == \
        bpt.BPT_ERR_INVALID_ARG


def test_backward_rejects_bad_pointers_and_small_workspace():
    for i in range(14):
        ins = list(BWD_IN)
        ins[i] = None
        assert bwd(ins, BWD_OUT) == bpt.BPT_ERR_INVALID_ARG, i
    for i in range(11):
        outs = list(BWD_OUT)
        outs[i] = None
        assert bwd(BWD_IN, outs) == bpt.BPT_ERR_INVALID_ARG, i
        outs = list(BWD_OUT)
        outs[i] += 8
        assert bwd(BWD_IN, outs) == bpt.BPT_ERR_INVALID_ARG, i
    outs = list(BWD_OUT)
    outs[1] = outs[0]  # two outputs overlap
    assert bwd(BWD_IN, outs) == bpt.BPT_ERR_INVALID_ARG
    outs = list(BWD_OUT)
    outs[0] = BWD_IN[12]  # dx over dZ
    assert bwd(BWD_IN, outs) == bpt.BPT_ERR_INVALID_ARG
    for dtype in (BF, F32):
        st, need = bpt.bpt_layer_backward_workspace_size(1, 256, 64, 1, 256, 1, dtype)
        assert bwd(BWD_IN, BWD_OUT, ws_bytes=need - 1, dtype=dtype) == bpt.BPT_ERR_WORKSPACE


def test_backward_empty_is_a_no_op():
    assert bwd([None] * 14, [None] * 11, B=0) == bpt.BPT_OK


# ---------------------------------------------- kept attention output (keep_o)
def fwd_keep_o(p, o, stats, dtype=BF, ws_bytes=1 << 31, B=1, N=256, d=256, h=2, d_ff=512):
    return bpt.bpt_layer_forward_train_keep_o(*p[:11], B, N, d, h, d_ff, 1, dtype, p[11], stats,
                                              o, p[12], ws_bytes, None, None)


def test_forward_keep_o_argument_checks():
    """Checked on the host before anything is enqueued (no GPU needed)."""
    stats, o = 0xA0000000, 0xB0000000
    assert fwd_keep_o(GOOD, None, stats) == bpt.BPT_ERR_INVALID_ARG
    assert fwd_keep_o(GOOD, o, None) == bpt.BPT_ERR_INVALID_ARG
    assert fwd_keep_o(GOOD, o + 8, stats) == bpt.BPT_ERR_INVALID_ARG       # misaligned
    assert fwd_keep_o(GOOD, GOOD[0], stats) == bpt.BPT_ERR_INVALID_ARG     # o over x
    assert fwd_keep_o(GOOD, GOOD[11], stats) == bpt.BPT_ERR_INVALID_ARG    # o over out
    assert fwd_keep_o(GOOD, GOOD[12] + 4096, stats) == bpt.BPT_ERR_INVALID_ARG  # in workspace
    assert fwd_keep_o(GOOD, stats + 64, stats) == bpt.BPT_ERR_INVALID_ARG  # o over stats
    for i in range(1, 11):
        assert fwd_keep_o(GOOD, GOOD[i], stats) == bpt.BPT_ERR_INVALID_ARG, i
    assert fwd_keep_o(GOOD, o, stats, dtype=F32) == bpt.BPT_ERR_UNSUPPORTED


def bwd_keep_o(ins, o, outs, ws_bytes=1 << 31, dtype=BF, B=1, N=256, d=64, h=1, d_ff=256):
    return bpt.bpt_layer_backward_keep_o(*ins[:12], o, ins[12], B, N, d, h, d_ff, 1, dtype,
                                         *outs, ins[13], ws_bytes, None, None)


def test_backward_keep_o_argument_checks():
    o = 0xC0000000
    assert bwd_keep_o(BWD_IN, None, BWD_OUT) == bpt.BPT_ERR_INVALID_ARG
    assert bwd_keep_o(BWD_IN, o + 8, BWD_OUT) == bpt.BPT_ERR_INVALID_ARG   # misaligned
    outs = list(BWD_OUT)
    outs[0] = o                                                             # dx over o
    assert bwd_keep_o(BWD_IN, o, outs) == bpt.BPT_ERR_INVALID_ARG
    assert bwd_keep_o(BWD_IN, BWD_IN[13] + 4096, BWD_OUT) == bpt.BPT_ERR_INVALID_ARG  # in ws
    assert bwd_keep_o(BWD_IN, o, BWD_OUT, dtype=F32) == bpt.BPT_ERR_UNSUPPORTED
