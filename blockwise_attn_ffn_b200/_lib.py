"""ctypes binding of libbpt (argument marshalling only).

The functions named ``bpt_*`` mirror the C ABI of ``include/bpt.h`` one to
one: pointers are passed as Python ints (device addresses), sizes as ints.
Every step of the layer runs in the library's CUDA kernels; there is no other
implementation behind this module, and loading fails loudly when the shared
library is missing.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libbpt.so")

BPT_OK, BPT_ERR_INVALID_ARG, BPT_ERR_UNSUPPORTED, BPT_ERR_WORKSPACE, BPT_ERR_CUDA, \
    BPT_ERR_TIMEOUT, BPT_ERR_RANGE = range(7)
BPT_F32, BPT_BF16 = 0, 1
KINDS = ["ln1", "qkv", "attn", "wo", "ln2", "w1", "w2", "cvt", "tail"]
BPT_WAVE_BLOCKS = 256
BPT_TAIL_MAX_PAIRS = 74
BPT_SCHEDULE_FUSED, BPT_SCHEDULE_WAVES = 0, 1
BPT_STATIC_WORKSPACE_BYTES = 64 * 1024 * 1024

EXPORTED = [
    "bpt_layer_workspace_size", "bpt_layer_forward", "bpt_read_device_error",
    "bpt_status_string", "bpt_profile_enable", "bpt_profile_read",
    "bpt_layer_launch_count", "bpt_layer_forward_static",
    "bpt_layer_forward_train", "bpt_layer_forward_bsfa", "bpt_layer_backward_workspace_size",
    "bpt_layer_backward",
    "bpt_layer_workspace_size_opt", "bpt_layer_forward_opt", "bpt_layer_forward_bsfa_opt",
    "bpt_layer_backward_workspace_size_opt", "bpt_layer_backward_opt",
    "bpt_layer_launch_count_opt",
    "bpt_layer_shard_workspace_size", "bpt_layer_shard_project", "bpt_layer_shard_forward",
    "bpt_layer_forward_train_keep_o", "bpt_layer_backward_keep_o",
    "bpt_layer_tail_plan",
]


class Options(ctypes.Structure):
    """``bpt_options`` (include/bpt.h): per-call choices of the *_opt calls."""
    _fields_ = [("schedule", ctypes.c_int32), ("attn_block", ctypes.c_int32),
                ("max_wave", ctypes.c_int64), ("fault", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


def make_options(schedule=None, attn_block=0, max_wave=0, fault=0, reserved=0) -> Options:
    """An ``Options`` value; ``schedule`` may be "fused", "waves" or the code."""
    if schedule is None or schedule == "fused":
        schedule = BPT_SCHEDULE_FUSED
    elif schedule == "waves":
        schedule = BPT_SCHEDULE_WAVES
    return Options(int(schedule), int(attn_block), int(max_wave), int(fault), int(reserved))


def _opts_ref(opts):
    """None, an ``Options`` or a dict of its fields -> argument for a const
    bpt_options* parameter."""
    if opts is None:
        return None
    if isinstance(opts, dict):
        opts = make_options(**opts)
    return ctypes.byref(opts)

_lib: Optional[ctypes.CDLL] = None


class BptError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)}")
        self.status = status


def load() -> ctypes.CDLL:
    """Load libbpt.so (built in-tree); raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m blockwise_attn_ffn_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    i64, vp, i32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
    lib.bpt_layer_workspace_size.argtypes = [i64, i64, i64, i64, i64, i32, i32,
                                             ctypes.POINTER(ctypes.c_size_t)]
    lib.bpt_layer_workspace_size.restype = i32
    lib.bpt_layer_forward.argtypes = [vp] * 11 + [i64] * 5 + [i32, i32, vp, vp, ctypes.c_size_t, vp]
    lib.bpt_layer_forward.restype = i32
    lib.bpt_layer_forward_train.argtypes = ([vp] * 11 + [i64] * 5 +
                                            [i32, i32, vp, vp, vp, ctypes.c_size_t, vp])
    lib.bpt_layer_forward_train.restype = i32
    lib.bpt_layer_forward_bsfa.argtypes = ([vp] * 11 + [i64] * 5 +
                                           [i32, i32, vp, vp, vp, vp, vp, ctypes.c_size_t, vp])
    lib.bpt_layer_forward_bsfa.restype = i32
    lib.bpt_layer_backward_workspace_size.argtypes = [i64, i64, i64, i64, i64, i32, i32,
                                                      ctypes.POINTER(ctypes.c_size_t)]
    lib.bpt_layer_backward_workspace_size.restype = i32
    lib.bpt_layer_backward.argtypes = ([vp] * 13 + [i64] * 5 + [i32, i32] + [vp] * 12 +
                                       [ctypes.c_size_t, vp])
    lib.bpt_layer_backward.restype = i32
    op = ctypes.POINTER(Options)
    lib.bpt_layer_workspace_size_opt.argtypes = [i64, i64, i64, i64, i64, i32, i32, op,
                                                 ctypes.POINTER(ctypes.c_size_t)]
    lib.bpt_layer_workspace_size_opt.restype = i32
    lib.bpt_layer_forward_opt.argtypes = ([vp] * 11 + [i64] * 5 +
                                          [i32, i32, vp, vp, vp, ctypes.c_size_t, op, vp])
    lib.bpt_layer_forward_opt.restype = i32
    lib.bpt_layer_forward_bsfa_opt.argtypes = ([vp] * 11 + [i64] * 5 +
                                               [i32, i32, vp, vp, vp, vp, vp, ctypes.c_size_t,
                                                op, vp])
    lib.bpt_layer_forward_bsfa_opt.restype = i32
    lib.bpt_layer_backward_workspace_size_opt.argtypes = [i64, i64, i64, i64, i64, i32, i32, op,
                                                          ctypes.POINTER(ctypes.c_size_t)]
    lib.bpt_layer_backward_workspace_size_opt.restype = i32
    lib.bpt_layer_backward_opt.argtypes = ([vp] * 13 + [i64] * 5 + [i32, i32] + [vp] * 12 +
                                           [ctypes.c_size_t, op, vp])
    lib.bpt_layer_backward_opt.restype = i32
    lib.bpt_layer_forward_train_keep_o.argtypes = ([vp] * 11 + [i64] * 5 +
                                                   [i32, i32, vp, vp, vp, vp, ctypes.c_size_t,
                                                    op, vp])
    lib.bpt_layer_forward_train_keep_o.restype = i32
    lib.bpt_layer_backward_keep_o.argtypes = ([vp] * 14 + [i64] * 5 + [i32, i32] + [vp] * 12 +
                                              [ctypes.c_size_t, op, vp])
    lib.bpt_layer_backward_keep_o.restype = i32
    lib.bpt_layer_launch_count_opt.argtypes = [i64, i64, i64, i64, i64, i32, i32, op,
                                               ctypes.POINTER(ctypes.c_int64)]
    lib.bpt_layer_launch_count_opt.restype = i32
    lib.bpt_layer_shard_workspace_size.argtypes = [i64] * 6 + [i32, i32,
                                                               ctypes.POINTER(ctypes.c_size_t)]
    lib.bpt_layer_shard_workspace_size.restype = i32
    for fn in (lib.bpt_layer_shard_project, lib.bpt_layer_shard_forward):
        fn.argtypes = [vp] * 11 + [i64] * 7 + [i32, i32, vp, vp, vp, ctypes.c_size_t, vp]
        fn.restype = i32
    lib.bpt_read_device_error.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_uint32)]
    lib.bpt_read_device_error.restype = i32
    lib.bpt_status_string.argtypes = [i32]
    lib.bpt_status_string.restype = ctypes.c_char_p
    lib.bpt_profile_enable.argtypes = [i32]
    lib.bpt_profile_enable.restype = i32
    lib.bpt_profile_read.argtypes = [ctypes.POINTER(ctypes.c_double),
                                     ctypes.POINTER(ctypes.c_int64), i32]
    lib.bpt_profile_read.restype = i32
    lib.bpt_layer_launch_count.argtypes = [i64, i64, i64, i64, i64, i32, i32,
                                           ctypes.POINTER(ctypes.c_int64)]
    lib.bpt_layer_launch_count.restype = i32
    p32 = ctypes.POINTER(ctypes.c_int32)
    lib.bpt_layer_tail_plan.argtypes = [i64, i64, i64, i64, i64, i32, i32, p32, p32, p32, i32]
    lib.bpt_layer_tail_plan.restype = i32
    lib.bpt_layer_forward_static.argtypes = [vp] * 11 + [i64] * 5 + [i32, i32, vp, vp]
    lib.bpt_layer_forward_static.restype = i32
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().bpt_status_string(int(status)).decode()


# ------------------------------------------------------------ C ABI mirror --
def bpt_layer_workspace_size(B, N, d, h, d_ff, causal, dtype) -> Tuple[int, int]:
    """Returns (status, bytes)."""
    out = ctypes.c_size_t(0)
    st = load().bpt_layer_workspace_size(B, N, d, h, d_ff, int(bool(causal)), dtype,
                                         ctypes.byref(out))
    return st, out.value


def bpt_layer_workspace_size_opt(B, N, d, h, d_ff, causal, dtype, opts) -> Tuple[int, int]:
    """Returns (status, bytes) for the given options (None, Options or dict)."""
    out = ctypes.c_size_t(0)
    st = load().bpt_layer_workspace_size_opt(B, N, d, h, d_ff, int(bool(causal)), dtype,
                                             _opts_ref(opts), ctypes.byref(out))
    return st, out.value


def bpt_layer_forward_opt(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2,
                          B, N, d, h, d_ff, causal, dtype, out, stats, workspace,
                          workspace_bytes, opts, stream) -> int:
    """Pointer-level call with options (stats may be None); returns the status."""
    return load().bpt_layer_forward_opt(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2,
                                        B, N, d, h, d_ff, int(bool(causal)), dtype, out, stats,
                                        workspace, workspace_bytes, _opts_ref(opts), stream)


def bpt_layer_forward_bsfa_opt(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2,
                               B, N, d, h, d_ff, causal, dtype, thresholds, block_max, kept,
                               out, workspace, workspace_bytes, opts, stream) -> int:
    return load().bpt_layer_forward_bsfa_opt(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2,
                                             b_2, B, N, d, h, d_ff, int(bool(causal)), dtype,
                                             thresholds, block_max, kept, out, workspace,
                                             workspace_bytes, _opts_ref(opts), stream)


def bpt_layer_backward_workspace_size_opt(B, N, d, h, d_ff, causal, dtype,
                                          opts) -> Tuple[int, int]:
    out = ctypes.c_size_t(0)
    st = load().bpt_layer_backward_workspace_size_opt(B, N, d, h, d_ff, int(bool(causal)),
                                                      dtype, _opts_ref(opts), ctypes.byref(out))
    return st, out.value


def bpt_layer_backward_opt(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, stats, dZ,
                           B, N, d, h, d_ff, causal, dtype, dx, d_ln1, dW_Q, dW_K, dW_V, dW_O,
                           d_ln2, dW_1, db_1, dW_2, db_2, workspace, workspace_bytes, opts,
                           stream) -> int:
    return load().bpt_layer_backward_opt(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2,
                                         stats, dZ, B, N, d, h, d_ff, int(bool(causal)), dtype,
                                         dx, d_ln1, dW_Q, dW_K, dW_V, dW_O, d_ln2, dW_1, db_1,
                                         dW_2, db_2, workspace, workspace_bytes,
                                         _opts_ref(opts), stream)


def bpt_layer_forward_train_keep_o(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2,
                                   B, N, d, h, d_ff, causal, dtype, out, stats, o, workspace,
                                   workspace_bytes, opts, stream) -> int:
    return load().bpt_layer_forward_train_keep_o(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2,
                                                 b_2, B, N, d, h, d_ff, int(bool(causal)),
                                                 dtype, out, stats, o, workspace,
                                                 workspace_bytes, _opts_ref(opts), stream)


def bpt_layer_backward_keep_o(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, stats, o,
                              dZ, B, N, d, h, d_ff, causal, dtype, dx, d_ln1, dW_Q, dW_K, dW_V,
                              dW_O, d_ln2, dW_1, db_1, dW_2, db_2, workspace, workspace_bytes,
                              opts, stream) -> int:
    return load().bpt_layer_backward_keep_o(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2,
                                            stats, o, dZ, B, N, d, h, d_ff, int(bool(causal)),
                                            dtype, dx, d_ln1, dW_Q, dW_K, dW_V, dW_O, d_ln2,
                                            dW_1, db_1, dW_2, db_2, workspace, workspace_bytes,
                                            _opts_ref(opts), stream)


def bpt_layer_shard_workspace_size(B, N, G, d, h, d_ff, causal, dtype) -> Tuple[int, int]:
    out = ctypes.c_size_t(0)
    st = load().bpt_layer_shard_workspace_size(B, N, G, d, h, d_ff, int(bool(causal)), dtype,
                                               ctypes.byref(out))
    return st, out.value


def bpt_layer_shard_project(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, B, N, G, rank,
                            d, h, d_ff, causal, dtype, kv_loc, out, workspace, workspace_bytes,
                            stream) -> int:
    return load().bpt_layer_shard_project(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2,
                                          B, N, G, rank, d, h, d_ff, int(bool(causal)), dtype,
                                          kv_loc, out, workspace, workspace_bytes, stream)


def bpt_layer_shard_forward(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, B, N, G, rank,
                            d, h, d_ff, causal, dtype, kv_all, out, workspace, workspace_bytes,
                            stream) -> int:
    return load().bpt_layer_shard_forward(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2,
                                          B, N, G, rank, d, h, d_ff, int(bool(causal)), dtype,
                                          kv_all, out, workspace, workspace_bytes, stream)


def bpt_layer_launch_count_opt(B, N, d, h, d_ff, causal, dtype, opts) -> Tuple[int, int]:
    out = ctypes.c_int64(0)
    st = load().bpt_layer_launch_count_opt(B, N, d, h, d_ff, int(bool(causal)), dtype,
                                           _opts_ref(opts), ctypes.byref(out))
    return st, out.value


def bpt_layer_forward(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2,
                      B, N, d, h, d_ff, causal, dtype, out, workspace, workspace_bytes,
                      stream) -> int:
    """Pointer-level call; returns the status code."""
    return load().bpt_layer_forward(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2,
                                    B, N, d, h, d_ff, int(bool(causal)), dtype, out,
                                    workspace, workspace_bytes, stream)


def bpt_layer_forward_bsfa(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2,
                           B, N, d, h, d_ff, causal, dtype, thresholds, block_max, kept, out,
                           workspace, workspace_bytes, stream) -> int:
    """Pointer-level call (block_max, kept may be None); returns the status code."""
    return load().bpt_layer_forward_bsfa(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2,
                                         B, N, d, h, d_ff, int(bool(causal)), dtype, thresholds,
                                         block_max, kept, out, workspace, workspace_bytes, stream)


def bpt_layer_forward_train(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2,
                            B, N, d, h, d_ff, causal, dtype, out, stats, workspace,
                            workspace_bytes, stream) -> int:
    """Pointer-level call; returns the status code."""
    return load().bpt_layer_forward_train(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2,
                                          B, N, d, h, d_ff, int(bool(causal)), dtype, out,
                                          stats, workspace, workspace_bytes, stream)


def bpt_layer_backward_workspace_size(B, N, d, h, d_ff, causal, dtype) -> Tuple[int, int]:
    """Returns (status, bytes)."""
    out = ctypes.c_size_t(0)
    st = load().bpt_layer_backward_workspace_size(B, N, d, h, d_ff, int(bool(causal)), dtype,
                                                  ctypes.byref(out))
    return st, out.value


def bpt_layer_backward(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, stats, dZ,
                       B, N, d, h, d_ff, causal, dtype, dx, d_ln1, dW_Q, dW_K, dW_V, dW_O,
                       d_ln2, dW_1, db_1, dW_2, db_2, workspace, workspace_bytes, stream) -> int:
    """Pointer-level call; returns the status code."""
    return load().bpt_layer_backward(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, stats,
                                     dZ, B, N, d, h, d_ff, int(bool(causal)), dtype, dx, d_ln1,
                                     dW_Q, dW_K, dW_V, dW_O, d_ln2, dW_1, db_1, dW_2, db_2,
                                     workspace, workspace_bytes, stream)


def bpt_read_device_error(workspace, stream) -> Tuple[int, int]:
    """Returns (status, site); workspace None reads the header of the array
    bpt_layer_forward_static uses."""
    site = ctypes.c_uint32(0)
    st = load().bpt_read_device_error(workspace, stream, ctypes.byref(site))
    return st, site.value


def bpt_status_string(status: int) -> str:
    return status_string(status)


def bpt_profile_enable(enable: bool) -> int:
    return load().bpt_profile_enable(int(bool(enable)))


def bpt_profile_read() -> Tuple[int, dict, dict]:
    """Returns (status, ms per kind, launches per kind)."""
    n = len(KINDS)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int64 * n)()
    st = load().bpt_profile_read(ms, cnt, n)
    return st, {k: ms[i] for i, k in enumerate(KINDS)}, {k: cnt[i] for i, k in enumerate(KINDS)}


def bpt_layer_forward_static(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2,
                             B, N, d, h, d_ff, causal, dtype, out, stream) -> int:
    """Pointer-level call of the allocation-free variant; returns the status.

    For callers that may not allocate device memory: the library uses its own
    fixed device array (BPT_STATIC_WORKSPACE_BYTES) as the workspace.
    """
    return load().bpt_layer_forward_static(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2,
                                           B, N, d, h, d_ff, int(bool(causal)), dtype, out,
                                           stream)


def bpt_layer_launch_count(B, N, d, h, d_ff, causal, dtype) -> Tuple[int, int]:
    out = ctypes.c_int64(0)
    st = load().bpt_layer_launch_count(B, N, d, h, d_ff, int(bool(causal)), dtype,
                                       ctypes.byref(out))
    return st, out.value


def bpt_layer_tail_plan(B, N, d, h, d_ff, causal, resident_pairs, rows=None):
    """Returns (status, pairs, shared, plan): plan is a list of
    (whole items, whole items before the shared one, shared item or -1,
    half or -1, partner or -1) per CTA pair, for the first `rows` pairs
    (default: BPT_TAIL_MAX_PAIRS)."""
    rows = BPT_TAIL_MAX_PAIRS if rows is None else rows
    pairs = ctypes.c_int32(0)
    shared = ctypes.c_int32(0)
    buf = (ctypes.c_int32 * (5 * max(rows, 1)))()
    st = load().bpt_layer_tail_plan(B, N, d, h, d_ff, int(bool(causal)), resident_pairs,
                                    ctypes.byref(pairs), ctypes.byref(shared),
                                    buf if rows > 0 else None, rows)
    n = min(pairs.value, rows) if st == BPT_OK else 0
    plan = [tuple(buf[5 * q:5 * q + 5]) for q in range(n)]
    return st, pairs.value, shared.value, plan
