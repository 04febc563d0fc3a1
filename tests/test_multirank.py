"""The multi-process (one rank per GPU) path, exercised with gloo on CPU.

The layer shards by sequence: each rank runs its own batch with the same
weights, and only the timing is reduced (max over ranks).  Two gloo ranks
check the rank inputs, the max reduction and the whole-job throughput; the
reference arm's non-zero ranks exit without work.
"""
import hashlib
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def digest(a):
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


def worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from blockwise_attn_ffn_b200 import dist as bdist
    from blockwise_attn_ffn_b200.inputs import LayerShape, make_inputs
    try:
        r, lr, w = bdist.env_rank()
        bdist.init_process_group("gloo", timeout_s=60)
        cfg = LayerShape("t", B=2, N=64, d=32, h=2, d_ff=64, causal=True, dtype="bf16",
                         block=128, seed=5, ln_scale=0.1)
        inp = bdist.rank_inputs(cfg, r)
        mine = {"w": digest(np.concatenate([inp[k].ravel() for k in
                                            ("W_Q", "W_K", "W_V", "W_O", "W_1", "W_2")])),
                "x": digest(inp["x_bits"])}
        gathered = [None] * w
        dist.all_gather_object(gathered, mine)
        ms = 10.0 + 5.0 * r                     # per-rank device time
        ms_max = bdist.max_over_ranks(ms, dist)
        tput = bdist.weak_scaling_tokens_per_s(cfg, w, ms_max)
        rank0_matches = (r != 0) or digest(inp["x_bits"]) == digest(make_inputs(cfg)["x_bits"])
        dist.barrier()
        dist.destroy_process_group()
        out_q.put((r, gathered, ms_max, tput, rank0_matches, None))
    except Exception as e:  # pragma: no cover - reported to the parent
        out_q.put((rank, None, None, None, None, repr(e)))


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for r, gathered, ms_max, tput, rank0_matches, err in res:
        assert err is None, err
        assert gathered[0]["w"] == gathered[1]["w"]        # same model on every rank
        assert gathered[0]["x"] != gathered[1]["x"]        # each rank its own sequences
        assert ms_max == 15.0                              # slowest rank decides
        assert tput == pytest.approx(2 * 64 * 2 / 15e-3)   # all ranks' tokens
        assert rank0_matches


def test_reference_arm_nonzero_rank_exits_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True,
                       text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
