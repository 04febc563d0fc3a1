"""Throughput of the BPT layer forward (libbpt) on synthetic inputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl bpt|reference] [--no-cpu-baseline]

One step = one full layer forward (LN1, QKV projection, every wave of
attention + W_O + LN2 + FFN) over one batch of the workload, through
bpt_layer_forward with inputs resident in HBM.  The workload defaults to the
long-context layer (B=1, N=65536, d=2048, h=16, d_ff=8192, causal, bf16).
Its per-step traffic (x 256 MiB, QKV 768 MiB, out 512 MiB, scratch 768 MiB)
is far above the 126 MB L2, so no flush is needed between steps.

Multi-GPU (torchrun): each rank runs its own batch of the workload (the outer
loop is data parallel across sequences), no collective on the data path;
value = tokens of all ranks / max-over-ranks time (weak scaling).

Prints one JSON line on rank 0.  `--impl reference` times the fp64 CPU oracle
instead (a bounded row sample per step, on the host cores).
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from blockwise_attn_ffn_b200 import accounting  # noqa: E402
from blockwise_attn_ffn_b200.inputs import WORKLOADS, make_inputs, sample_rows  # noqa: E402

METRIC = "BPT layer fwd tokens/s, TFLOP/s (% bf16 peak) at N=64K; peak live bytes"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one attention
# launch of the default bench command, from a one-kernel, one-launch ncu
# capture with those two metrics only (one pass: nothing saved or replayed;
# profiles/attn_pair_tc_long_n64k_dram.md).  Valid only for the code it was
# taken on: the digest covers the attention kernel, the shared device helpers,
# the host function that configures its launch (grid, head groups, the K/V
# budget) and the fused schedule's call of it; after a change there the bench
# reports null until the one-launch capture is taken again.
ATTN_TRAFFIC = {
    "long_n64k": {"bytes_per_launch": 1437998336, "digest": "7822612978d30784"},
}
TRAFFIC_FILES = ("blockwise_attn_ffn_b200/csrc/attn_pair_tc.cuh",
                 "blockwise_attn_ffn_b200/csrc/common.cuh")
TRAFFIC_API = "blockwise_attn_ffn_b200/csrc/bpt_api.cu"


def sources_digest() -> str:
    import hashlib
    import re
    h = hashlib.sha256()
    for rel in TRAFFIC_FILES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    with open(os.path.join(ROOT, TRAFFIC_API)) as f:
        api = f.read()
    a = api.index("cudaError_t launch_attn(")
    h.update(api[a:api.index("\n}\n", a)].encode())
    a = api.index("// attention over every query block")
    h.update(api[a:api.index("int dummy = 0, pairs_max = 0;", a)].encode())
    h.update(re.search(r"#define BPT_ATTN_KV_BUDGET_MB \d+", api).group(0).encode())
    return h.hexdigest()[:16]


def attn_traffic(workload: str):
    entry = ATTN_TRAFFIC.get(workload)
    if entry is None or entry["digest"] != sources_digest():
        return None
    return entry["bytes_per_launch"]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_config(cfg, world, extra=None):
    c = {"workload": cfg.name, "global_batch": cfg.B * world, "seq_len": cfg.N, "d": cfg.d,
         "h": cfg.h, "d_ff": cfg.d_ff, "causal": cfg.causal, "block": cfg.block,
         "parallelism": f"dp{world}" if world > 1 else "single",
         "l2": "inputs larger than L2 (per-step traffic > 1.5 GiB), no flush"}
    if extra:
        c.update(extra)
    return c


# ------------------------------------------------------------------ clocks --
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"bpt_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------- CPU baseline --
def cpu_oracle_rate(cfg, n_rows: int):
    """Times the fp64 oracle (as it stands) on a sample of rows; tokens/s."""
    import oracle
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        threads = None
    inp = make_inputs(cfg, B=1)
    rows = sample_rows(cfg, n_rows, B=1)
    cores = len(os.sched_getaffinity(0))
    try:  # BLAS threads pinned to the cores this process may use
        from threadpoolctl import threadpool_limits
        limit = threadpool_limits(limits=cores)
        threads = cores
    except Exception:  # pragma: no cover
        limit = None
    t0 = time.perf_counter()
    oracle.layer_rows(inp, cfg.h, cfg.causal, rows)
    dt = time.perf_counter() - t0
    if limit is not None:
        limit.unregister()
    return {"value": len(rows) / dt, "unit": UNIT, "cores": threads or cores,
            "host_cores": cores, "kind": "oracle", "seconds": dt,
            "sample": f"{len(rows)} seeded rows of {cfg.name} (incl. row N-1, so K/V for all "
                      f"{cfg.N} keys) through oracle.layer_rows, fp64"}


# ------------------------------------------------------ training step --
def measure_backward(bpt, cfg, x, p, stream, dev, args, flops, world, peaks, dist):
    """Times bpt_layer_backward (gradients of every parameter and of x from
    the saved (m, l)) and the whole training step (bpt_layer_forward_train +
    bpt_layer_backward), CUDA events on the launching stream, max over ranks.
    Gradient FLOPs are counted as twice the forward's algorithmic FLOPs (the
    usual convention: one product for the data gradient and one for the
    weight gradient of every forward product); the block recomputation adds
    about one forward on top, as the pages state."""
    import torch
    from blockwise_attn_ffn_b200 import dist as bdist
    out, stats, ws = bpt.layer_forward_train(x, p, cfg.h, cfg.causal)
    gen = torch.Generator(device=dev).manual_seed(cfg.seed + 77)
    dZ = torch.randn(x.shape, generator=gen, device=dev, dtype=torch.float32)
    grads, bws = bpt.layer_backward(x, p, cfg.h, cfg.causal, stats, dZ)
    for _ in range(2):
        bpt.layer_backward(x, p, cfg.h, cfg.causal, stats, dZ, workspace=bws)
    torch.cuda.synchronize(dev)
    k = args.backward_steps
    e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    if world > 1:
        dist.barrier()
    e0.record(stream)
    for _ in range(k):
        bpt.layer_backward(x, p, cfg.h, cfg.causal, stats, dZ, workspace=bws)
    e1.record(stream)
    for _ in range(k):
        bpt.layer_forward_train(x, p, cfg.h, cfg.causal, out=out, stats=stats, workspace=ws)
        bpt.layer_backward(x, p, cfg.h, cfg.causal, stats, dZ, workspace=bws)
    e2.record(stream)
    # the same with the attention output kept by the forward (no attention
    # recomputation in the backward; +2 B N d bytes of fp16 activation)
    o = torch.empty(x.shape, dtype=torch.float16, device=dev)
    bpt.layer_forward_train(x, p, cfg.h, cfg.causal, out=out, stats=stats, workspace=ws,
                            keep_o=o)
    bpt.layer_backward(x, p, cfg.h, cfg.causal, stats, dZ, workspace=bws, o=o)
    e3, e4 = (torch.cuda.Event(enable_timing=True) for _ in range(2))
    if world > 1:
        dist.barrier()
    e2b = torch.cuda.Event(enable_timing=True)
    e2b.record(stream)
    for _ in range(k):
        bpt.layer_backward(x, p, cfg.h, cfg.causal, stats, dZ, workspace=bws, o=o)
    e3.record(stream)
    for _ in range(k):
        bpt.layer_forward_train(x, p, cfg.h, cfg.causal, out=out, stats=stats, workspace=ws,
                                keep_o=o)
        bpt.layer_backward(x, p, cfg.h, cfg.causal, stats, dZ, workspace=bws, o=o)
    e4.record(stream)
    torch.cuda.synchronize(dev)
    st, site = bpt.bpt_read_device_error(bws.data_ptr(), stream.cuda_stream)
    if st != bpt.BPT_OK:
        raise SystemExit(f"device error in backward {bpt.status_string(st)} site {site}")
    bwd_ms = bdist.max_over_ranks(e0.elapsed_time(e1), dist, dev) / k
    step_ms = bdist.max_over_ranks(e1.elapsed_time(e2), dist, dev) / k
    bwd_o_ms = bdist.max_over_ranks(e2b.elapsed_time(e3), dist, dev) / k
    step_o_ms = bdist.max_over_ranks(e3.elapsed_time(e4), dist, dev) / k
    grad_tf = 2 * flops["total"] * world / (bwd_ms / 1e3) / 1e12
    tokens = cfg.B * cfg.N * world
    return {"ms_per_step": bwd_ms, "tokens_per_s": tokens / (bwd_ms / 1e3),
            "grad_tflops": grad_tf, "pct_bf16_peak": grad_tf / world / peaks["bf16_tflops"],
            "train_step_ms": step_ms, "train_step_tokens_per_s": tokens / (step_ms / 1e3),
            "train_step_tflops": 3 * flops["total"] * world / (step_ms / 1e3) / 1e12,
            "keep_o": {"ms_per_step": bwd_o_ms,
                       "grad_tflops": 2 * flops["total"] * world / (bwd_o_ms / 1e3) / 1e12,
                       "train_step_ms": step_o_ms,
                       "train_step_tokens_per_s": tokens / (step_o_ms / 1e3),
                       "kept_bytes": int(o.numel() * 2)},
            "steps": k, "workspace_bytes": int(bws.numel()),
            "note": "grad FLOPs = 2 x forward algorithmic FLOPs; train step = forward_train + "
                    "backward (3 x forward FLOPs counted; recomputation not counted); keep_o: "
                    "the forward keeps the attention output and the backward reads it instead "
                    "of recomputing the attention"}


# ---------------------------------------------- gated attention (BSFA) --
def measure_bsfa(bpt, cfg, x, p, out_dense, ms_dense, stream, dev, args, world, dist):
    """Times bpt_layer_forward_bsfa ("Block Sparse Flash Attention": exact
    block maxima, a per-(head, query block) threshold, pruned blocks skip
    their exponentials and PV products).  Thresholds keep the top k
    off-diagonal key blocks per query block, calibrated (package
    ``bsfa.calibrate``) on the block maxima of one other seeded synthetic x
    through the same weights; the timed x is the bench's.  Reports the kept
    fraction, the time per forward (CUDA events, max over ranks), the speed-up
    over the dense forward and the largest output deviation from it."""
    import numpy as np
    import torch
    from blockwise_attn_ffn_b200 import bsfa as bbsfa
    from blockwise_attn_ffn_b200 import dist as bdist
    from blockwise_attn_ffn_b200.inputs import make_inputs
    nb = (cfg.N + 127) // 128
    cal = make_inputs(cfg.with_(seed=cfg.seed + 7919))
    xc = bpt.to_device(cal, cfg.dtype, dev)["x"]  # its weights are dropped: p's are used
    del cal
    none = torch.full((cfg.h, nb), float("-inf"), dtype=torch.float32, device=dev)
    o2 = torch.empty_like(out_dense)
    _, bm, _, ws = bpt.layer_forward_bsfa(xc, p, cfg.h, cfg.causal, none, block_max=True, out=o2)
    del xc
    T = torch.from_numpy(bbsfa.calibrate(bm.cpu().numpy(), args.bsfa_k, cfg.causal)).to(dev)
    _, _, kept, _ = bpt.layer_forward_bsfa(x, p, cfg.h, cfg.causal, T, kept=True, out=o2,
                                           workspace=ws)
    vis = np.tril(np.ones((nb, nb), bool)) if cfg.causal else np.ones((nb, nb), bool)
    off = vis & ~np.eye(nb, dtype=bool)
    kp = kept.cpu().numpy().astype(bool)
    kept_frac = float(kp[:, :, off].mean()) if off.any() else 1.0
    # V tiles the gated kernel loads: a CTA's two query blocks (2q, 2q+1) share
    # each V_j, loaded when either block that visits j keeps it
    v_loaded = v_total = 0
    for q0 in range(0, nb, 2):
        rows = [i for i in (q0, q0 + 1) if i < nb]
        for j in range(nb):
            vis_rows = [i for i in rows if vis[i, j]]
            if not vis_rows:
                continue
            any_keep = np.zeros(kp.shape[:2], bool)
            for i in vis_rows:
                any_keep |= kp[:, :, i, j]
            v_loaded += int(any_keep.sum())
            v_total += any_keep.size
    for _ in range(args.warmup):
        bpt.layer_forward_bsfa(x, p, cfg.h, cfg.causal, T, out=o2, workspace=ws)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        bpt.layer_forward_bsfa(x, p, cfg.h, cfg.causal, T, out=o2, workspace=ws)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    st, site = bpt.bpt_read_device_error(ws.data_ptr(), stream.cuda_stream)
    if st != bpt.BPT_OK:
        raise SystemExit(f"device error in bsfa {bpt.status_string(st)} site {site}")
    ms = bdist.max_over_ranks(e0.elapsed_time(e1), dist, dev) / args.steps
    dev_max = float((o2 - out_dense).abs().max())
    return {"k": args.bsfa_k, "kept_offdiag_frac": kept_frac,
            "v_tiles_loaded_frac": v_loaded / max(1, v_total),
            "v_bytes_skipped_per_forward": int((v_total - v_loaded) * 128 * cfg.d_k * 2),
            "ms_per_step": ms,
            "tokens_per_s": cfg.B * cfg.N * world / (ms / 1e3),
            "speedup_vs_dense": ms_dense / ms, "max_abs_dev_vs_dense": dev_max,
            "max_abs_dense": float(out_dense.abs().max()), "steps": args.steps,
            "calibration": "top-k off-diagonal blocks per query block from the block maxima "
                           "of one other seeded synthetic x (same weights)",
            "note": "approximate attention (the pages' method): synthetic inputs have no "
                    "learned attention sparsity, so the deviation says nothing about model "
                    "quality; a V tile is loaded only when a query block that visits it "
                    "keeps the block"}


# ------------------------------------------------- unfused peak bytes --
def unfused_torch_peak_bytes(cfg, p, dev):
    """Peak device bytes of the plain unfused schedule, measured once outside
    the timed region: LN, Q/K/V matmuls, PyTorch SDPA, W_O matmul + residual,
    LN, W_1 matmul + GELU, W_2 matmul + residual, all materialised in bf16.
    A bench-only measurement of the memory the pages' unfused schedule keeps
    alive; nothing of the library runs here."""
    import torch
    import torch.nn.functional as F
    B, N, d, h = cfg.B, cfg.N, cfg.d, cfg.h
    torch.cuda.synchronize(dev)
    base = torch.cuda.memory_allocated(dev)
    torch.cuda.reset_peak_memory_stats(dev)
    with torch.no_grad():
        x = p["x"].view(B, N, d)
        g1, b1n = p["ln1"][0], p["ln1"][1]
        xn = F.layer_norm(x, (d,), g1, b1n, 1e-5)
        q, k, v = xn @ p["W_Q"], xn @ p["W_K"], xn @ p["W_V"]
        del xn
        def heads(t):
            return t.view(B, N, h, d // h).transpose(1, 2)
        o = F.scaled_dot_product_attention(heads(q), heads(k), heads(v), is_causal=cfg.causal)
        del q, k, v
        o = o.transpose(1, 2).reshape(B, N, d)
        y = x + o @ p["W_O"]
        del o
        yn = F.layer_norm(y, (d,), p["ln2"][0], p["ln2"][1], 1e-5)
        hid = F.gelu(yn @ p["W_1"] + p["b_1"])
        del yn
        z = y + hid @ p["W_2"] + p["b_2"]
        del hid, y, z
    torch.cuda.synchronize(dev)
    return int(torch.cuda.max_memory_allocated(dev) - base)


# ------------------------------------------------------------- reference --
def run_reference(args, cfg, rank, world):
    if rank != 0:
        return 0
    rows = args.ref_rows
    per = []
    for _ in range(args.warmup):
        cpu_oracle_rate(cfg, rows)
    for _ in range(args.steps):
        per.append(cpu_oracle_rate(cfg, rows))
    value = float(np.mean([p["value"] for p in per]))
    cb = dict(per[-1])
    cb["value"] = value
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": float(np.mean([p["seconds"] for p in per]) * 1e3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(cfg, 1),
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ main --
# ----------------------------------------------------------- forward timing --
def time_forward(bpt, cfg, x, p, opts, steps, warmup, stream, dev, dist, world, out=None,
                 ws=None, profile=True, per_step_events=True):
    """Times `steps` forwards (after `warmup`) with CUDA events on the
    launching stream, max over ranks.  Returns a dict with the step time, the
    per-step times, the per-kernel CUDA-event times and the buffers used."""
    import torch
    from blockwise_attn_ffn_b200 import dist as bdist
    out, ws = bpt.layer_forward(x, p, cfg.h, cfg.causal, out=out, workspace=ws, opts=opts)
    torch.cuda.synchronize(dev)
    st, site = bpt.bpt_read_device_error(ws.data_ptr(), stream.cuda_stream)
    if st != bpt.BPT_OK:
        raise SystemExit(f"device error {bpt.status_string(st)} site {site}")
    for _ in range(warmup):
        bpt.layer_forward(x, p, cfg.h, cfg.causal, out=out, workspace=ws, opts=opts)
    torch.cuda.synchronize(dev)
    bpt.bpt_profile_read()  # clear
    bpt.bpt_profile_enable(profile)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1 if per_step_events else 2)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    ev[0].record(stream)
    for i in range(steps):
        bpt.layer_forward(x, p, cfg.h, cfg.causal, out=out, workspace=ws, opts=opts)
        if per_step_events:
            ev[i + 1].record(stream)
    if not per_step_events:
        ev[1].record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    bpt.bpt_profile_enable(False)
    _, kind_ms, kind_n = bpt.bpt_profile_read()
    st, site = bpt.bpt_read_device_error(ws.data_ptr(), stream.cuda_stream)
    if st != bpt.BPT_OK:
        raise SystemExit(f"device error {bpt.status_string(st)} site {site}")
    ms_total = bdist.max_over_ranks(ev[0].elapsed_time(ev[-1]), dist, dev)
    per_step = ([ev[i].elapsed_time(ev[i + 1]) for i in range(steps)] if per_step_events
                else [ms_total / steps])
    return {"ms_step": ms_total / steps, "per_step": per_step, "kind_ms": kind_ms,
            "kind_n": kind_n, "out": out, "ws": ws}


def kernel_table(kind_ms, kind_n, steps, flops):
    """Per-kernel CUDA-event time per step, share and TFLOP/s."""
    total = sum(kind_ms.values())
    flop_kind = {"qkv": flops["qkv"], "attn": flops["attention"], "wo": flops["wo"],
                 "w1": flops["ffn"] / 2, "w2": flops["ffn"] / 2,
                 "tail": flops["wo"] + flops["ffn"]}
    table = {}
    for k, ms in kind_ms.items():
        if kind_n.get(k, 0) == 0:
            continue
        e = {"ms_per_step": ms / steps, "launches_per_step": kind_n[k] / steps,
             "share": ms / total if total else None}
        if k in flop_kind and ms > 0:
            e["tflops"] = flop_kind[k] / (ms / steps / 1e3) / 1e12
        table[k] = e
    return table


def peak_bytes_above(dev, fn):
    """Peak device bytes allocated by fn() above what is allocated before it."""
    import torch
    torch.cuda.synchronize(dev)
    base = torch.cuda.memory_allocated(dev)
    torch.cuda.reset_peak_memory_stats(dev)
    keep = fn()
    torch.cuda.synchronize(dev)
    peak = torch.cuda.max_memory_allocated(dev) - base
    del keep
    return int(peak)


def other_workloads(bpt, args, names, stream, dev, peaks):
    """Each named workload timed on this GPU (fused schedule; waves as well
    for bf16 layers): tokens/s, TFLOP/s and the fraction of the burst peak."""
    import torch
    res = {}
    for name in names:
        cfg = WORKLOADS[name]
        inp = make_inputs(cfg)
        p = bpt.to_device(inp, cfg.dtype, dev)
        del inp
        flops = accounting.layer_flops(cfg.B, cfg.N, cfg.d, cfg.h, cfg.d_ff, cfg.causal)
        steps = max(3, min(args.steps, int(2000.0 / max(1.0, flops["total"] / 1e12 * 1.2))))
        entry = {"B": cfg.B, "N": cfg.N, "d": cfg.d, "h": cfg.h, "d_ff": cfg.d_ff,
                 "dtype": cfg.dtype, "steps": steps, "flops_per_step": flops["total"]}
        schedules = ["fused", "waves"] if cfg.dtype == "bf16" else ["waves"]
        for sched in schedules:
            opts = bpt.make_options(schedule=sched)
            r = time_forward(bpt, cfg, p["x"], p, opts, steps, 3, stream, dev, None, 1,
                             profile=True, per_step_events=False)
            tf = flops["total"] / (r["ms_step"] / 1e3) / 1e12
            entry[sched] = {"ms_per_step": r["ms_step"],
                            "tokens_per_s": cfg.B * cfg.N / (r["ms_step"] / 1e3),
                            "tflops": tf, "pct_bf16_peak": tf / peaks["bf16_tflops"],
                            "kernels": kernel_table(r["kind_ms"], r["kind_n"], steps, flops)}
            del r
        if cfg.dtype == "f32":
            entry["note"] = "fp32 layer on the CUDA cores (FFMA); % of the bf16 tensor peak " \
                            "for reference only"
        res[name] = entry
        del p
        torch.cuda.empty_cache()
    return res


def run_sequence_parallel(args, cfg, rank, world, dev, dist):
    """One sequence split over the ranks (zig-zag chunks; per step: shard
    projection, one NCCL all-gather of K | V into each GPU's own buffer,
    shard attention + layer body).  Strong scaling: the whole job is one
    pass over the workload's batch; value = its tokens / max-over-ranks time."""
    import torch
    import blockwise_attn_ffn_b200 as bpt
    from blockwise_attn_ffn_b200 import dist as bdist
    from blockwise_attn_ffn_b200 import shard
    stream = torch.cuda.current_stream(dev)
    inp = make_inputs(cfg)
    p = bpt.to_device(inp, cfg.dtype, dev)
    del inp
    rows = torch.from_numpy(shard.token_rows(cfg.N, world, rank)).to(dev)
    x_loc = p["x"][:, rows].contiguous()
    x_host = x_loc.cpu().pin_memory()
    del p["x"]
    out, bufs = shard.sequence_parallel_forward(x_loc, p, cfg.h, cfg.causal, cfg.N, dist)
    for _ in range(args.warmup):
        shard.sequence_parallel_forward(x_loc, p, cfg.h, cfg.causal, cfg.N, dist, bufs=bufs)
    torch.cuda.synchronize(dev)
    with ClockSampler(torch.cuda.current_device()) as clk:
        dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            shard.sequence_parallel_forward(x_loc, p, cfg.h, cfg.causal, cfg.N, dist, bufs=bufs)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        dist.barrier()
    st, site = bpt.bpt_read_device_error(bufs["ws"].data_ptr(), stream.cuda_stream)
    if st != bpt.BPT_OK:
        raise SystemExit(f"device error {bpt.status_string(st)} site {site}")
    ms = bdist.max_over_ranks(e0.elapsed_time(e1), dist, dev) / args.steps
    # end to end: the rank's rows up from pinned host memory, its output down
    host_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    dist.barrier()
    e0.record(stream)
    for _ in range(args.steps):
        x_loc.copy_(x_host, non_blocking=True)
        shard.sequence_parallel_forward(x_loc, p, cfg.h, cfg.causal, cfg.N, dist, bufs=bufs)
        host_out.copy_(bufs["out"], non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms_e2e = bdist.max_over_ranks(e0.elapsed_time(e1), dist, dev) / args.steps
    flops = accounting.layer_flops(cfg.B, cfg.N, cfg.d, cfg.h, cfg.d_ff, cfg.causal)
    peaks, peak_src = load_peaks()
    tokens = cfg.B * cfg.N
    tf = flops["total"] / (ms / 1e3) / 1e12
    kv_bytes = int(bufs["kv_loc"].numel() * 2)
    return {
        "metric": METRIC, "value": tokens / (ms / 1e3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic: seeded N(0,1) x, N(0,1/fan_in) weights, LN gamma~1+0.1N, beta~0.1N",
        "config": dict(workload_config(cfg, 1), parallelism=f"sequence{world}",
                       shard="zig-zag chunks r and 2G-1-r; one NCCL all-gather of K|V per step"),
        "tflops": tf, "pct_bf16_peak": tf / world / peaks["bf16_tflops"], "peak_src": peak_src,
        "allgather_bytes_per_rank": kv_bytes * (world - 1),
        "gpu_launches": 5 * args.steps,
        "e2e": {"value": tokens / (ms_e2e / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": int(x_loc.numel() * 2) * world,
                "d2h_bytes_per_step": int(out.numel() * 4) * world, "ms_per_step": ms_e2e},
        "clocks": clk.summary()}


def relaunch_under_torchrun(args) -> int:
    """`bench.py --gpus N` started as a plain process: start the N ranks
    ourselves (one process per GPU) with the same arguments."""
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={args.gpus}", "--master-addr=127.0.0.1",
           f"--master-port={port}", os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


# ------------------------------------------------------------------ main --
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="long_n64k", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="bpt", choices=["bpt", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=1024)
    ap.add_argument("--ref-rows", type=int, default=16)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the training-step (forward_train + backward) measurement")
    ap.add_argument("--backward-steps", type=int, default=10)
    ap.add_argument("--no-unfused-peak", action="store_true",
                    help="skip the bench-only unfused-schedule peak-bytes measurement")
    ap.add_argument("--seq-len", type=int, default=None,
                    help="override the workload's N (profiling runs on a smaller case)")
    ap.add_argument("--no-bsfa", action="store_true",
                    help="skip the gated-attention (BSFA) forward measurement")
    ap.add_argument("--bsfa-k", type=int, default=32,
                    help="off-diagonal key blocks kept per query block by the BSFA thresholds")
    ap.add_argument("--schedule", default="fused", choices=["fused", "waves"],
                    help="layer body after attention: one persistent per-block kernel "
                         "(fused) or wave-level kernels (waves)")
    ap.add_argument("--attn-block", type=int, default=256, choices=[64, 128, 256, 512],
                    help="b, the query rows sharing each K/V tile (256: two 128-row blocks "
                         "per CTA; 128: one block per CTA; 64: one 64-row block per CTA, two "
                         "CTAs per SM; 512: a cluster of two CTAs sharing each tile over DSMEM)")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="skip timing the other four workloads")
    ap.add_argument("--no-alt-schedule", action="store_true",
                    help="skip timing the other schedule on the bench workload")
    ap.add_argument("--parallel", default="data", choices=["data", "sequence"],
                    help="several GPUs: each runs its own batch (data, weak scaling) or one "
                         "sequence is split over them (sequence, strong scaling)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    from blockwise_attn_ffn_b200 import dist as bdist
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return relaunch_under_torchrun(args)
    rank, local_rank, world = bdist.env_rank()
    cfg = WORKLOADS[args.workload]
    if args.seq_len:
        cfg = cfg.with_(N=args.seq_len, name=f"{cfg.name}@N={args.seq_len}")

    if args.impl == "reference":
        return run_reference(args, cfg, rank, world)

    import torch
    import torch.distributed as dist
    import blockwise_attn_ffn_b200 as bpt

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        bdist.init_process_group("nccl", device=dev)
    stream = torch.cuda.current_stream(dev)
    if args.parallel == "sequence" and world > 1:
        line = run_sequence_parallel(args, cfg, rank, world, dev, dist)
        if rank == 0:
            print(json.dumps(line), flush=True)
        dist.barrier()
        dist.destroy_process_group()
        return 0

    # Inputs: the workload's weights on every rank, a rank-seeded x each.
    inp = bdist.rank_inputs(cfg, rank)
    p = bpt.to_device(inp, cfg.dtype, dev)
    x_host = None
    if not args.no_e2e:
        x_host = bpt.to_device(inp, cfg.dtype, dev, pin_x=True)["x"]
    del inp
    x = p["x"]
    opts = bpt.make_options(schedule=args.schedule, attn_block=args.attn_block)
    alt_sched = "waves" if args.schedule == "fused" else "fused"
    alt_opts = bpt.make_options(schedule=alt_sched, attn_block=args.attn_block)

    # Peak device bytes above the resident inputs (x and the parameters), for
    # each schedule: out + workspace of one forward.
    inputs_bytes = int(torch.cuda.memory_allocated(dev))

    def one_forward(o):
        def run():
            r = bpt.layer_forward(x, p, cfg.h, cfg.causal, opts=o)
            torch.cuda.synchronize(dev)
            return r
        return run
    peak_main = peak_bytes_above(dev, one_forward(opts))
    peak_alt = peak_bytes_above(dev, one_forward(alt_opts)) if cfg.dtype == "bf16" else None
    torch.cuda.empty_cache()

    flops = accounting.layer_flops(cfg.B, cfg.N, cfg.d, cfg.h, cfg.d_ff, cfg.causal)
    code = bpt.BPT_BF16 if cfg.dtype == "bf16" else bpt.BPT_F32
    _, launches_per_step = bpt.bpt_layer_launch_count_opt(cfg.B, cfg.N, cfg.d, cfg.h, cfg.d_ff,
                                                          cfg.causal, code, opts)

    # -------- timed region (device time, CUDA events on the launching stream)
    with ClockSampler(local_rank) as clk:
        main_r = time_forward(bpt, cfg, x, p, opts, args.steps, args.warmup, stream, dev, dist,
                              world)
    out, ws = main_r["out"], main_r["ws"]
    ms_step = main_r["ms_step"]
    per_step = main_r["per_step"]
    kind_ms, kind_n = main_r["kind_ms"], main_r["kind_n"]
    tokens_step = cfg.B * cfg.N * world
    value = bdist.weak_scaling_tokens_per_s(cfg, world, ms_step)

    # -------- the other schedule, same workload (no clock record: context)
    alt = None
    if not args.no_alt_schedule and cfg.dtype == "bf16":
        r = time_forward(bpt, cfg, x, p, alt_opts, max(3, args.steps // 2), args.warmup, stream,
                         dev, dist, world)
        alt = {"schedule": alt_sched, "ms_per_step": r["ms_step"],
               "tokens_per_s": bdist.weak_scaling_tokens_per_s(cfg, world, r["ms_step"]),
               "tflops": flops["total"] * world / (r["ms_step"] / 1e3) / 1e12,
               "kernels": kernel_table(r["kind_ms"], r["kind_n"], max(3, args.steps // 2), flops),
               "peak_bytes_above_inputs": peak_alt}
        del r
        torch.cuda.empty_cache()

    # -------- end to end: pinned x -> device, forward, out -> pinned host,
    # every step.  The copies run on their own streams with double-buffered
    # device inputs and outputs, so step i's forward overlaps step i+1's
    # upload and step i-1's download (a serving pipeline); the timed region
    # spans the first upload to the last download.
    e2e = None
    if not args.no_e2e:
        h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        xs = [torch.empty_like(x) for _ in range(2)]
        outs = [out, torch.empty_like(out)]
        hosts = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]

        def pipeline(n, start=None):
            in_free, out_free = [None, None], [None, None]
            if start is not None:
                h2d.wait_event(start)
            for i in range(n):
                b = i & 1
                if in_free[b] is not None:
                    h2d.wait_event(in_free[b])
                with torch.cuda.stream(h2d):
                    xs[b].copy_(x_host, non_blocking=True)
                landed = torch.cuda.Event()
                landed.record(h2d)
                stream.wait_event(landed)
                if out_free[b] is not None:
                    stream.wait_event(out_free[b])
                bpt.layer_forward(xs[b], p, cfg.h, cfg.causal, out=outs[b], workspace=ws,
                                  stream=stream, opts=opts)
                done = torch.cuda.Event()
                done.record(stream)
                in_free[b] = done
                d2h.wait_event(done)
                with torch.cuda.stream(d2h):
                    hosts[b].copy_(outs[b], non_blocking=True)
                out_free[b] = torch.cuda.Event()
                out_free[b].record(d2h)
            for evt in out_free:
                if evt is not None:
                    stream.wait_event(evt)

        pipeline(2)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        pipeline(args.steps, start=e0)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms_e2e = bdist.max_over_ranks(e0.elapsed_time(e1), dist, dev)
        st, site = bpt.bpt_read_device_error(ws.data_ptr(), stream.cuda_stream)
        if st != bpt.BPT_OK:
            raise SystemExit(f"device error in e2e {bpt.status_string(st)} site {site}")
        e2e = {"value": tokens_step / (ms_e2e / args.steps / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": int(x.numel() * x.element_size()),
               "d2h_bytes_per_step": int(out.numel() * out.element_size()),
               "ms_per_step": ms_e2e / args.steps,
               "note": "copies on their own streams, double-buffered, overlapping the "
                       "neighbouring steps' forwards"}
        del xs, hosts

    peaks, peak_src = load_peaks()
    n_attn = max(1, kind_n.get("attn", 0))
    attn_ms_launch = kind_ms["attn"] / n_attn
    attn_flops_launch = flops["attention"] * args.steps / n_attn
    achieved = attn_flops_launch / (attn_ms_launch / 1e3) / 1e12
    attn_bytes_launch = accounting.attention_bytes(cfg.B, cfg.N, cfg.d, cfg.h) * args.steps / n_attn
    peak_burst = peaks["bf16_tflops"]
    peak_sus = peaks["bf16_tflops_sustained"]
    kernels = kernel_table(kind_ms, kind_n, args.steps, flops)
    tflops = flops["total"] * world / (ms_step / 1e3) / 1e12
    # Step a1+a2 (LN1 + QKV projection): x, W_Q|W_K|W_V and QKV touched once.
    esz_in = 2 if cfg.dtype == "bf16" else 4
    kb1_bytes = cfg.B * cfg.N * cfg.d * esz_in + 3 * cfg.d * cfg.d * 2 + cfg.B * cfg.N * 3 * cfg.d * 2
    kb1_ms = (kind_ms.get("ln1", 0.0) + kind_ms.get("qkv", 0.0)) / args.steps
    unfused = accounting.unfused_activation_elems(cfg.N, cfg.d, cfg.h, cfg.d_ff,
                                                  with_logits=False)
    esz = 2 if cfg.dtype == "bf16" else 4

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "f16" if cfg.dtype == "bf16" else "f32",
        "dtype_note": ("bf16 inputs and weights; tensor-core operands fp16 (weights copied "
                       "exactly each call), fp32 accumulation, fp32 residual stream and output")
        if cfg.dtype == "bf16" else "fp32 throughout (CUDA cores)",
        "data": "synthetic: seeded N(0,1) x, N(0,1/fan_in) weights, LN gamma~1+0.1N, beta~0.1N",
        "config": dict(workload_config(cfg, world), attn_block=args.attn_block,
                       schedule=args.schedule),
        "tflops": tflops,
        "pct_bf16_peak": tflops / world / peak_burst,
        "pct_bf16_peak_sustained": tflops / world / peak_sus,
        "pct_nominal_2250": tflops / world / 2250.0,
        "ms_per_step_median": float(np.median(per_step)),
        "ms_per_step_min": float(np.min(per_step)),
        "kb1_hbm": {"algorithmic_bytes": int(kb1_bytes),
                    "achieved_gbs": kb1_bytes / (kb1_ms / 1e3) / 1e9 if kb1_ms > 0 else None,
                    "peak_gbs": peaks["hbm_gbs"],
                    "note": "LN1 + QKV projection kernels: x + W_QKV + QKV once / their time"},
        "peak_src": peak_src,
        "roofline": {"bound": "tensor", "kernel": "attn_pair_tc_kernel", "achieved": achieved,
                     "peak": peak_burst, "unit": "TFLOP/s", "frac": achieved / peak_burst,
                     "peak_kind": f"bf16_tflops burst ({peak_src}); fp16 operands, same "
                                  "dense rate",
                     "frac_of_sustained": achieved / peak_sus,
                     "traffic": attn_traffic(cfg.name),
                     "traffic_unit": "bytes per launch (ncu dram read + write)",
                     "algorithmic_bytes_per_launch": attn_bytes_launch},
        "kernels": kernels,
        "alt_schedule": alt,
        "peak_bytes": {
            "base": "bytes allocated above the resident inputs (x and the parameters) during "
                    "one forward: out + workspace for the library; every activation for the "
                    "unfused torch schedule",
            "inputs_resident": inputs_bytes,
            args.schedule: int(peak_main),
            alt_sched: peak_alt,
            "unfused_activations_analytic": int(cfg.B * unfused["total"] * esz),
            "unfused_ffn_hidden_analytic": int(cfg.B * unfused["ffn_hidden"] * esz)},
        "gpu_launches": int(launches_per_step * args.steps),
        "e2e": e2e,
    }
    line["clocks"] = clk.summary()
    if not args.no_backward and cfg.dtype == "bf16":
        line["backward"] = measure_backward(bpt, cfg, x, p, stream, dev, args, flops, world,
                                            peaks, dist)
    if not args.no_bsfa and cfg.dtype == "bf16":
        line["bsfa"] = measure_bsfa(bpt, cfg, x, p, out, ms_step, stream, dev, args, world, dist)
    if not args.no_unfused_peak and cfg.dtype == "bf16":
        del out, ws, main_r
        torch.cuda.empty_cache()
        line["peak_bytes"]["unfused_torch_measured"] = unfused_torch_peak_bytes(cfg, p, dev)
    if not args.no_other_workloads and world == 1 and args.seq_len is None:
        del p, x
        torch.cuda.empty_cache()
        names = [n for n in ("tiny_f32", "gpt2s_n2k", "mid_n16k", "long_n64k", "wide_n128k")
                 if n != cfg.name]
        line["other_workloads"] = other_workloads(bpt, args, names, stream, dev, peaks)

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_oracle_rate(cfg, args.cpu_rows)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
