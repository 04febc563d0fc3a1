"""Sequence sharding, host side (CPU only): the zig-zag partition, the
K | V lookup the attention kernel performs in the all-gathered buffer, and
the all-gather itself with two gloo ranks.

"Blockwise Parallel Transformer — BPT", section "BPT and Ring Attention":
the sequence is split across devices and every device's queries need the
keys and values of all devices; zig-zag chunks (rank r owns chunks r and
2G-1-r) give every rank the same causal work.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from blockwise_attn_ffn_b200 import shard

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("N,G", [(256, 1), (1024, 2), (4096, 4), (65536, 8)])
def test_partition_covers_every_token_once(N, G):
    rows = [shard.token_rows(N, G, r) for r in range(G)]
    assert all(len(r) == N // G for r in rows)
    allr = np.sort(np.concatenate(rows))
    np.testing.assert_array_equal(allr, np.arange(N))
    # chunk r then chunk 2G-1-r, each in token order
    c = N // (2 * G)
    for r in range(G):
        np.testing.assert_array_equal(rows[r][:c], np.arange(r * c, (r + 1) * c))
        np.testing.assert_array_equal(rows[r][c:], np.arange((2 * G - 1 - r) * c,
                                                             (2 * G - r) * c))


@pytest.mark.parametrize("N,G", [(2048, 2), (8192, 4), (65536, 8)])
def test_zigzag_balances_causal_work(N, G):
    """Causal attention of a query block i costs i + 1 key blocks: every
    rank gets the same total."""
    work = []
    for r in range(G):
        blocks = shard.token_rows(N, G, r)[::128] // 128
        work.append(int(np.sum(blocks + 1)))
    assert len(set(work)) == 1


@pytest.mark.parametrize("N,G", [(1024, 2), (4096, 4), (65536, 8)])
def test_kv_lookup_matches_the_gathered_layout(N, G):
    """kv_all[owner, local] built from each rank's rows holds the token
    kv_source names, for every token."""
    kv_all = np.stack([shard.token_rows(N, G, r) for r in range(G)])  # [G, n_loc] token ids
    for t in range(0, N, 37):
        o, l = shard.kv_source(N, G, t)
        assert kv_all[o, l] == t
    # whole key blocks stay contiguous in one rank's rows
    for j in range(N // 128):
        o, l = shard.kv_source(N, G, j * 128)
        np.testing.assert_array_equal(kv_all[o, l:l + 128], np.arange(j * 128, j * 128 + 128))


def test_rejects_unshardable_lengths():
    with pytest.raises(ValueError):
        shard.token_rows(1000, 2, 0)
    with pytest.raises(ValueError):
        shard.token_rows(256 * 3, 2, 0)


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def worker(rank, world, port, N, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    try:
        import torch.distributed as dist
        from blockwise_attn_ffn_b200 import dist as bdist
        from blockwise_attn_ffn_b200 import shard as bshard
        bdist.init_process_group("gloo", timeout_s=60)
        B, d = 2, 4
        rows = torch.from_numpy(bshard.token_rows(N, world, rank))
        # K | V stand-in: every element tagged with (batch, token, column)
        kv_loc = (torch.arange(B)[:, None, None] * 1e6 + rows[None, :, None] * 10 +
                  torch.arange(2 * d)[None, None, :]).to(torch.float32)
        kv_all = torch.empty((world,) + tuple(kv_loc.shape), dtype=torch.float32)
        bshard.gather_kv(kv_loc, kv_all, dist)
        ok = True
        for b in range(B):
            for t in range(N):
                o, l = bshard.kv_source(N, world, t)
                want = b * 1e6 + t * 10 + torch.arange(2 * d, dtype=torch.float32)
                ok &= bool(torch.equal(kv_all[o, b, l], want))
        dist.barrier()
        dist.destroy_process_group()
        out_q.put((rank, ok, None))
    except Exception as e:  # pragma: no cover - reported to the parent
        out_q.put((rank, False, repr(e)))


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_all_gather_gives_every_rank_every_token(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    N = 256 * world * 2
    procs = [ctx.Process(target=worker, args=(r, world, port, N, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    for rank, ok, err in res:
        assert err is None, err
        assert ok, f"rank {rank}: gathered K | V does not match the lookup"
