#!/usr/bin/env python
"""Decode-step benchmark: single-token MLRA-4 decode over a latent KV cache on B200.

A step is one whole decode call (query absorption -> split-KV decode -> log-sum-exp merge
-> up-projection, four kernels) over one batch of the workload; inputs are resident in HBM when the timed region
starts.  Default workload: MLRA-4, B=64, h=128, T=32768, 64-token pages with a random
page table (2.4 GB of KV cache read per step, larger than L2, so no flush is needed).

    python bench.py [--gpus N --steps K --warmup W] [--workload NAME] [--impl reference]

Multi-GPU (torchrun, one rank per GPU): every rank decodes its own replica batch (the
path has no exchange step); value = all ranks' KV bytes / max-over-ranks step time.
One JSON line is printed by rank 0.

--gpus N without torchrun: bench.py launches itself as N ranks (torch.distributed.run,
rendezvous on 127.0.0.1); under torchrun, --gpus must equal WORLD_SIZE.

--cache int8 (MLRA-4 workloads and their branch shards): the latent cache is int8 with one
fp32 scale per token and 128-column block (K_RoPE stays bf16): 656 instead of 1152 bytes per
token.

--gla 2 (MLA workloads): a rank of GLA-2, MLA's latent split into two 256-wide groups
with half of the heads each (2.5 d_h of cache per token and rank); with one GPU, rank 0's
call is timed alone, with 2 GPUs the ranks' outs are gathered over heads.

--prefill L [--prefill-queries n]: the prefill path instead (causal multi-token MLRA-4 in the
expanded form, h = 128, one sequence of L cached tokens whose last n are the queries), in
TFLOP/s of algorithmic work against the measured tensor peak.

--tp W (W = 2 or 4 for MLRA-4, 2 for MLRA-2): tensor parallelism by branch.  Rank r holds
its W-th of the branches (cache columns + K_RoPE, W_UK / W_UV rows) and a step is its
shard's decode followed by an NCCL all-reduce of out; run it with --gpus W.  With one GPU,
the rank-0 shard's step is timed alone (no all-reduce).  --fused-out replaces the NCCL
call by the fused path: the up-projection adds into every rank's out (symmetric memory),
bracketed by device barriers.
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import hashlib
import json
import math
import os
import pathlib
import statistics
import subprocess
import sys
import time

ROOT = pathlib.Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "MLRA-4 decode µs/step & KV-cache read TB/s (fraction of ~8 TB/s HBM)"
NOMINAL_HBM_GBS = 8000.0
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
# The sources the 128-wide-branch decode kernel (the one whose ncu traffic is recorded) is
# compiled from; a change to any of them invalidates the recorded traffic.
DECODE_SOURCES = ["head_rank_attention_b200/csrc/decode_split_sm100.cu", "head_rank_attention_b200/csrc/sm100.cuh",
                  "head_rank_attention_b200/csrc/schedule.cuh", "head_rank_attention_b200/csrc/decode_sm100.h",
                  "head_rank_attention_b200/csrc/launch.h"]


def tensor_flops_per_token(n_branch: int, heads: int, d_c: int = 512) -> int:
    """Algorithmic tensor-core FLOPs per cached token (shared rope scored once, real heads
    only, one query term): scores over d_c + 64 dims and P.V over d_c columns per head,
    2*(d_c+64)*h + 2*d_c*h.  (The kernels issue more: each slice CTA scores its branch
    for 128 padded head rows, and MLRA-4 scores with two query terms.)"""
    return 2 * (d_c + 64) * heads + 2 * d_c * heads


def peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return d, "measured"
    return dict(FALLBACK), "fallback"


def decode_source_hash() -> str:
    h = hashlib.sha256()
    for f in DECODE_SOURCES:
        h.update((ROOT / f).read_bytes())
    return h.hexdigest()[:16]


def traffic_key(workload: str, tp: int = 0, gla: int = 0, int8: bool = False) -> str:
    """Key of a decode launch's recorded traffic: the workload, the shard or GLA group and the
    cache format (each runs a different kernel or different bytes)."""
    return workload + (f"/tp{tp}" if tp else "") + (f"/gla{gla}" if gla else "") + ("/int8" if int8 else "")


def ncu_traffic(workload: str, path=None):
    """dram bytes per decode launch from the committed ncu summary, if it matches the
    current kernel source; else None."""
    f = ROOT / "profiles" / "decode_dram_traffic.json" if path is None else path
    if not f.exists():
        return None
    d = json.loads(f.read_text())
    entry = d.get(workload)
    if not entry or entry.get("decode_source_sha") != decode_source_hash():
        return None
    return entry.get("dram_bytes_per_launch")


class ClockSampler:
    """SM clock and throttle-reason sampling during the timed region, in-process through
    NVML every 2 ms (a background thread), so short timed regions still get samples."""
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, device: int):
        self.device = device
        self.samples = []
        self.max_mhz = None
        self._stop = None

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(self.device).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            try:
                h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            except Exception:
                h = pynvml.nvmlDeviceGetHandleByIndex(self.device)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception:
            return self
        self._stop = threading.Event()

        def run():
            while not self._stop.is_set():
                try:
                    clk = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                    rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    try:
                        mw = pynvml.nvmlDeviceGetPowerUsage(h)
                    except Exception:
                        mw = None
                    self.samples.append((clk, rs, mw))
                except Exception:
                    pass
                self._stop.wait(0.002)

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._stop is not None:
            self._stop.set()
            self._thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"]}
        clks = sorted(c for c, _, _ in self.samples)
        reasons = sorted({n for _, r, _ in self.samples for n, bit in self.REASONS.items() if r & bit})
        watts = [w / 1000.0 for _, _, w in self.samples if w is not None]
        return {"sm_mhz": statistics.median(clks), "sm_max_mhz": self.max_mhz, "sm_mhz_min": clks[0],
                "reasons": reasons, "power_w": statistics.median(watts) if watts else None,
                "samples": len(clks), "source": "NVML, 2 ms period, timed region only"}


def time_oracle_sample(wl: synth.Workload, n_seqs: int, n_heads: int, tp_world: int = 0, gla: int = 0,
                       int8: bool = False):
    """Run the fp64 oracle (the expanded definition) on n_seqs x n_heads outputs of the
    workload (of its rank-0 branch shard under tp_world-way tensor parallelism, or of rank
    0's group under GLA, if set); return (seconds, the sample's share of the step, threads
    used, sequences, heads)."""
    import oracle
    from head_rank_attention_b200 import tp
    try:
        import threadpoolctl
        threads = max(i.get("num_threads", 1) for i in threadpoolctl.threadpool_info())
    except Exception:  # pragma: no cover
        threads = os.cpu_count()
    w_uk, w_uv = synth.weights(wl)
    q = synth.queries(wl)
    lens = synth.seq_lens(wl)
    seqs = list(range(min(n_seqs, wl.batch)))
    heads = list(range(min(n_heads, wl.heads)))
    rows = {s: synth.seq_rows(wl, s) for s in seqs}  # generation is not timed
    d_c, n_branch = synth.D_C, wl.n_branch
    if tp_world:
        rows = {s: tp.shard_cache(r, 0, tp_world, n_branch) for s, r in rows.items()}
        w_uk, w_uv = tp.shard_weights(w_uk, w_uv, 0, tp_world, n_branch)
        d_c, n_branch = synth.D_C // tp_world, wl.n_branch // tp_world
    n_heads_rank = wl.heads
    if gla:  # group 0: latent columns [0, 512 / gla) and the first h / gla heads
        per = wl.heads // gla
        rows = {s: tp.shard_cache(r, 0, gla, n_branch=gla) for s, r in rows.items()}
        w_uk, w_uv = w_uk[:per, :synth.D_C // gla], w_uv[:per, :synth.D_C // gla]
        q = q[:, :per]
        heads = heads[:per]
        d_c, n_branch, n_heads_rank = synth.D_C // gla, 1, per
    if int8:  # the sample's latent rows as the int8 cache stands for them
        rows = {s: (oracle.dequantize_int8_blocks(*synth.quantize_int8_blocks(r[:, :d_c])), r[:, d_c:])
                for s, r in rows.items()}
    else:
        rows = {s: (r[:, :d_c], r[:, d_c:]) for s, r in rows.items()}
    t0 = time.perf_counter()
    for s in seqs:
        c, kr = rows[s]
        oracle.mlra_decode_expanded(q[s], c, kr, w_uk, w_uv, n_branch,
                                    alpha_q=wl.alpha_q, alpha_kv=wl.alpha_kv,
                                    branch_scale=1.0 if gla else wl.sigma_o,
                                    softmax_scale=wl.softmax_scale, rope_theta=wl.rope_theta, heads=heads)
    dt = time.perf_counter() - t0
    # the sample's share of the full step, by cached tokens x heads
    frac = (sum(int(lens[s]) for s in seqs) * len(heads)) / (int(lens.sum()) * n_heads_rank)
    return dt, frac, threads, len(seqs), len(heads)


def workload_config(wl: synth.Workload, lens, tp_world: int = 0, gla: int = 0) -> dict:
    if gla:
        return dict(workload_config(wl, lens), variant=f"GLA-{gla} rank", d_c=512 // gla, heads=wl.heads // gla,
                    branch_scale=1.0, gla_rank=f"1 of {gla} latent groups, {wl.heads // gla} of {wl.heads} heads")
    return {"workload": wl.name, "variant": {1: "MLA", 2: "MLRA-2", 4: "MLRA-4"}[wl.n_branch],
            "batch": wl.batch, "heads": wl.heads, "seq_len": wl.seq_len,
            "seq_len_min": wl.seq_len_min, "total_tokens": int(np.asarray(lens, dtype=np.int64).sum()),
            "layout": f"paged({wl.page_size})" if wl.page_size else "contiguous",
            "d_c": 512 // tp_world if tp_world else 512, "d_rope": 64,
            **({"tp_shard": f"{wl.n_branch // tp_world} of {wl.n_branch} branches per rank"} if tp_world else {}), "alpha_q": wl.alpha_q, "alpha_kv": wl.alpha_kv, "branch_scale": wl.sigma_o,
            "l2": "inputs larger than L2 (KV cache per step >> 126 MB); no flush"}


def max_over_ranks(values, world: int, device) -> list:
    """Element-wise maximum of `values` over all ranks: the job's time is its slowest
    rank's.  Needs an initialised default process group when world > 1."""
    if world == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def job_tbs(bytes_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job throughput in TB/s: every rank reads bytes_per_rank per step."""
    return world * bytes_per_rank / (ms_per_step * 1e-3) / 1e12


def self_launch(n: int) -> int:
    """Run this script as n ranks (one per GPU) under torch.distributed.run on 127.0.0.1;
    returns the launcher's exit status."""
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", f"--master-port={port}", str(pathlib.Path(__file__).resolve()),
           *sys.argv[1:]]
    return subprocess.call(cmd)


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def run_reference(args, wl, world, rank):
    if rank != 0:
        return
    lens = synth.seq_lens(wl)
    tpw = getattr(args, "tp", 0)
    gla = getattr(args, "gla", 0)
    d_c = synth.D_C // tpw if tpw else synth.D_C // gla if gla else synth.D_C
    int8 = getattr(args, "cache", "bf16") == "int8"
    per_token = d_c + 2 * synth.D_ROPE + 4 * (d_c // 128) if int8 else (d_c + synth.D_ROPE) * 2
    kv = int(np.asarray(lens, dtype=np.int64).sum()) * per_token
    for _ in range(args.warmup):
        time_oracle_sample(wl, 1, 1, tpw, gla, int8)
    times = []
    frac = threads = None
    for _ in range(args.steps):
        dt, frac, threads, ns, nh = time_oracle_sample(wl, args.ref_seqs, args.ref_heads, tpw, gla, int8)
        times.append(dt / frac)  # extrapolated seconds per full decode step
    step_s = statistics.mean(times)
    value = kv / step_s / 1e12
    sample = (f"each step: oracle (expanded fp64 definition) on {args.ref_seqs} sequence(s) x {args.ref_heads} "
              f"head(s) of the workload, extrapolated by cached tokens x heads to the full step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
            "us_per_step": step_s * 1e6, "higher_is_better": True, "scaling": "strong" if tpw else "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(workload_config(wl, lens, tpw, gla), cache="int8" if int8 else "bf16",
                           cache_bytes_per_token=per_token),
            "cpu_baseline": {"value": value, "unit": "TB/s", "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_native(args, wl, world, rank, local):
    import head_rank_attention_b200 as hra
    torch.cuda.set_device(local)
    dev_id = torch.cuda.current_device()
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    inp = synth.make_inputs(wl)
    lens = inp.seq_lens.numpy()
    dev = synth.to_device(inp)
    tpw = args.tp
    all_reduce = tpw > 0 and world > 1
    d_c, n_branch = synth.D_C, wl.n_branch
    cache, w_uk, w_uv = dev.cache, dev.w_uk, dev.w_uv
    host_cache, host_wuk, host_wuv = inp.cache, inp.w_uk, inp.w_uv
    gla = getattr(args, "gla", 0)
    heads = wl.heads
    q_dev, host_q = dev.q, inp.q
    branch_scale = wl.sigma_o
    if gla:  # this rank's GLA-2 group: latent columns [256 g, +256), K_RoPE, heads [h g / 2, +h / 2)
        g = rank if world == gla else 0
        per = wl.heads // gla
        hsl = slice(g * per, (g + 1) * per)
        cols = slice(g * (synth.D_C // gla), (g + 1) * (synth.D_C // gla))
        cache = hra.tp.shard_cache(dev.cache, g, gla, n_branch=gla)
        host_cache = hra.tp.shard_cache(inp.cache, g, gla, n_branch=gla)
        w_uk, w_uv = dev.w_uk[hsl, cols].contiguous(), dev.w_uv[hsl, cols].contiguous()
        host_wuk, host_wuv = inp.w_uk[hsl, cols].contiguous(), inp.w_uv[hsl, cols].contiguous()
        q_dev, host_q = dev.q[:, hsl].contiguous(), inp.q[:, hsl].contiguous()
        dev.cache = dev.w_uk = dev.w_uv = None
        torch.cuda.empty_cache()
        d_c, n_branch, heads, branch_scale = synth.D_C // gla, 1, per, 1.0
    if tpw:  # this rank's branch shard (rank 0's when one GPU stands alone)
        shard = rank if world == tpw else 0
        cache = hra.tp.shard_cache(dev.cache, shard, tpw, wl.n_branch)
        w_uk, w_uv = hra.tp.shard_weights(dev.w_uk, dev.w_uv, shard, tpw, wl.n_branch)
        host_cache = hra.tp.shard_cache(inp.cache, shard, tpw, wl.n_branch)
        host_wuk, host_wuv = hra.tp.shard_weights(inp.w_uk, inp.w_uv, shard, tpw, wl.n_branch)
        dev.cache = dev.w_uk = dev.w_uv = None
        torch.cuda.empty_cache()
        d_c, n_branch = synth.D_C // tpw, wl.n_branch // tpw
    int8 = args.cache == "int8"
    ckv_scale = None
    if int8:  # quantise this rank's latent columns (input preparation, outside the timed region)
        q8, ckv_scale = synth.quantize_int8_blocks(cache[:, :d_c])
        host_q8, host_scale = q8.cpu(), ckv_scale.cpu()  # the same bytes for the end-to-end leg
        krope_dev = cache[:, d_c:].contiguous()
        host_krope = host_cache[:, d_c:].contiguous()
        cache = None
        torch.cuda.empty_cache()
        per_token = d_c + 2 * synth.D_ROPE + 4 * (d_c // 128)
    else:
        per_token = (d_c + synth.D_ROPE) * 2
    kv = int(lens.astype(np.int64).sum()) * per_token  # cache bytes this rank reads
    stream = torch.cuda.current_stream()
    peer_out = None
    if all_reduce and args.fused_out:  # out in symmetric memory, added into by every rank
        peer_out = hra.tp.PeerOut((wl.batch, wl.heads, synth.D_V), device=torch.device("cuda", local))
        out = peer_out.out
    else:
        out = torch.empty(wl.batch, heads, synth.D_V, dtype=torch.float32, device="cuda")
    gathered = (torch.empty(world, wl.batch, heads, synth.D_V, dtype=torch.float32, device="cuda")
                if gla and world > 1 else None)
    ckv_view, krope_view = (q8, krope_dev) if int8 else (cache[:, :d_c], cache[:, d_c:])
    p = hra.make_params(q_dev, ckv_view, krope_view, dev.seq_lens, w_uk, w_uv, out, ckv_scale=ckv_scale,
                        n_branch=n_branch, alpha_q=wl.alpha_q, alpha_kv=wl.alpha_kv, branch_scale=branch_scale,
                        softmax_scale=wl.softmax_scale, rope_theta=wl.rope_theta, block_table=dev.block_table,
                        page_size=wl.page_size, seq_stride=dev.seq_stride, num_splits=args.num_splits,
                        out_accumulate=peer_out is not None, out_peers=peer_out.peers if peer_out else None)
    ws = hra.alloc_workspace(p)

    # per-step stage events: [before absorb, before decode, before combine, after combine]
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for evs in events:  # torch creates the underlying cudaEvent_t on first record
        for e in evs:
            e.record(stream)
    torch.cuda.synchronize()
    handles = [(ctypes.c_void_p * 4)(*[e.cuda_event for e in evs]) for evs in events]
    assert all(h for hs in handles for h in hs), "CUDA events were not created"

    def call():  # one step as a user makes it: the decode call (+ the all-reduce under TP)
        if peer_out is not None:
            peer_out.begin()
            hra.mlra_decode(p, stream)
            peer_out.end()
        else:
            hra.mlra_decode(p, stream)
            if all_reduce:
                hra.tp.all_reduce_out(out)
            elif gathered is not None:  # GLA-2: the ranks' heads side by side
                torch.distributed.all_gather_into_tensor(gathered, out)

    for _ in range(args.warmup):
        call()
    hra.check_device_status(p, stream)

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()

    # Inputs smaller than twice the L2 (126 MB) would stay cached between steps: flush it
    # by writing a 512 MB buffer before every timed step.
    step_bytes = kv + sum(t.numel() * t.element_size() for t in (q_dev, w_uk, w_uv))
    step_bytes_all = step_bytes + out.numel() * 4
    flush = torch.zeros(128 << 20, dtype=torch.float32, device="cuda") if step_bytes < (252 << 20) else None

    # The timed steps: the call as a user makes it (kernels chained by programmatic
    # dependent launch), replayed from a CUDA graph of one call unless --no-graph, so that
    # host-side launch work does not bound the short configurations.
    graph = None
    if not args.no_graph and not all_reduce and gathered is None:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            hra.mlra_decode(p, torch.cuda.current_stream())
        for _ in range(args.warmup):
            graph.replay()
        torch.cuda.synchronize()
        hra.check_device_status(p, stream)
    def one_step():
        if graph is not None:
            graph.replay()
        else:
            call()

    barrier()
    with ClockSampler(dev_id) as clk:
        if flush is None:  # inputs larger than L2: back-to-back steps
            start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            start.record(stream)
            for k in range(args.steps):
                one_step()
            end.record(stream)
            torch.cuda.synchronize()
            elapsed_ms = start.elapsed_time(end)
        else:  # small inputs: L2 flushed before every step, each step timed on its own
            pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                     for _ in range(args.steps)]
            for e0, e1 in pairs:
                flush.add_(1)
                e0.record(stream)
                one_step()
                e1.record(stream)
            torch.cuda.synchronize()
            elapsed_ms = sum(e0.elapsed_time(e1) for e0, e1 in pairs)
    hot_ms = None
    if flush is not None:  # the same steps back to back with a warm L2, reported beside
        h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        h0.record(stream)
        for k in range(args.steps):
            one_step()
        h1.record(stream)
        torch.cuda.synchronize()
        hot_ms = h0.elapsed_time(h1) / args.steps
    hra.check_device_status(p, stream)
    graph_used = graph is not None
    del graph

    # Per-stage breakdown (and the decode kernel's own time for the roofline): the same
    # number of steps again with events between the kernels, which the library then
    # launches without the programmatic overlap so that each event pair brackets whole
    # kernels.
    barrier()
    for k in range(args.steps):
        p.stage_events = ctypes.cast(handles[k], ctypes.c_void_p)
        hra.mlra_decode(p, stream)
    torch.cuda.synchronize()
    p.stage_events = None
    hra.check_device_status(p, stream)
    stage_ms = np.array([[evs[i].elapsed_time(evs[i + 1]) for i in range(3)] for evs in events])
    decode_ms = float(stage_ms[:, 1].mean())

    # end to end through the C ABI with host buffers: H2D of every input, decode, D2H of out
    host_inputs = (dict(q=host_q, ckv=host_q8, scale=host_scale, krope=host_krope) if int8 else
                   dict(q=host_q, cache=host_cache))
    pin = {k: v.pin_memory() for k, v in dict(**host_inputs, seq_lens=inp.seq_lens,
                                               w_uk=host_wuk, w_uv=host_wuv).items()}
    if inp.block_table is not None:
        pin["block_table"] = inp.block_table.pin_memory()
    host_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    dmap = dict(q=q_dev, seq_lens=dev.seq_lens, w_uk=w_uk, w_uv=w_uv,
                **(dict(ckv=q8, scale=ckv_scale, krope=krope_dev) if int8 else dict(cache=cache)),
                block_table=dev.block_table)
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = host_out.numel() * host_out.element_size()
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        for k, t in pin.items():
            dmap[k].copy_(t, non_blocking=True)
        call()
        host_out.copy_(out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    hra.check_device_status(p, stream)
    # the same with the cache and weights resident (as in serving): per step only the
    # query, the lengths (and block table) go host -> device and out comes back
    per_step = [k for k in ("q", "seq_lens", "block_table") if k in pin]
    h2d_res = sum(pin[k].numel() * pin[k].element_size() for k in per_step)
    r_steps = max(1, args.steps)
    barrier()
    r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    r0.record(stream)
    for _ in range(r_steps):
        for k in per_step:
            dmap[k].copy_(pin[k], non_blocking=True)
        call()
        host_out.copy_(out, non_blocking=True)
    r1.record(stream)
    torch.cuda.synchronize()
    res_ms = r0.elapsed_time(r1) / r_steps
    hra.check_device_status(p, stream)

    step_ms = elapsed_ms / args.steps
    step_ms, e2e_ms, decode_ms, res_ms = max_over_ranks([step_ms, e2e_ms, decode_ms, res_ms], world, "cuda")
    clocks = clk.summary()

    if rank == 0:
        pk, pk_src = peaks()
        achieved_gbs = kv / (decode_ms * 1e-3) / 1e9
        flops = tensor_flops_per_token(n_branch, heads, d_c) * int(lens.astype(np.int64).sum())
        achieved_tflops = flops / (decode_ms * 1e-3) / 1e12
        traffic = ncu_traffic(traffic_key(wl.name, tpw, gla, int8))
        if gla:
            parallelism = (f"gla{gla}: head-and-latent groups, outs gathered over heads" if world == gla
                           else f"gla{gla}: rank 0's group alone (no gather)")
        elif tpw:
            if not all_reduce:
                parallelism = f"tp{tpw}: rank 0's branch shard alone (no all-reduce)"
            elif peer_out is not None:
                parallelism = f"tp{tpw}: branch shards, the up-projection adding into every rank's out (fused)"
            else:
                parallelism = f"tp{tpw}: branch shards + NCCL all-reduce of out"
        else:
            parallelism = f"replicas x{world}" if world > 1 else "1 GPU"
        line = {
            "metric": METRIC,
            "value": job_tbs(kv, world, step_ms), "unit": "TB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": step_ms, "us_per_step": step_ms * 1e3,
            "higher_is_better": True, "scaling": "strong" if tpw else "weak", "vs_baseline": None,
            "dtype": "f16",
            "precision": "bf16 inputs; fp16 tensor-core operands (absorbed query fp16, cache tile converted "
                         "bf16 -> fp16 in shared memory, P fp16); fp32 accumulate, softmax, combine",
            "data": "synthetic",
            "config": dict(workload_config(wl, lens, tpw, gla), parallelism=parallelism,
                           cache=("int8, one fp32 scale per token and 128-column block; K_RoPE bf16" if int8
                                  else "bf16"), cache_bytes_per_token=per_token,
                           num_splits=args.num_splits or f"auto (SMs/{d_c // 128})",
                           timing="CUDA-graph replays of one call" if graph_used else "direct calls",
                           **({} if flush is None else
                              {"l2": "inputs smaller than L2: 512 MB written before every step, "
                                     "each step timed on its own"})),
            "kv_frac_of_nominal_8TBs": kv / (step_ms * 1e-3) / 1e9 / NOMINAL_HBM_GBS,
            # every byte a step must move (KV, both weight tensors, q, out) over the measured copy peak
            "step_bytes_frac": step_bytes_all / (step_ms * 1e-3) / 1e9 / peaks()[0]["hbm_gbs"],
            **({} if hot_ms is None else {"us_per_step_hot_l2": hot_ms * 1e3}),
            "stage_us": {"absorb_q": float(stage_ms[:, 0].mean()) * 1e3, "decode": decode_ms * 1e3,
                         "combine_upproj": float(stage_ms[:, 2].mean()) * 1e3},  # merge + up-projection
            "roofline": {"kernel": "decode_split_kernel" if d_c // n_branch == 128 else "decode_kernel",
                         "bound": "hbm", "achieved": achieved_gbs,
                         "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": achieved_gbs / pk["hbm_gbs"],
                         "peak_source": pk_src, "traffic": traffic,
                         "bytes_per_launch": kv,
                         # the same bytes over the whole step (all four kernels)
                         "frac_step": kv / (step_ms * 1e-3) / 1e9 / pk["hbm_gbs"]},
            "roofline_tensor": {"achieved": achieved_tflops, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                                "frac": achieved_tflops / pk["bf16_tflops"],
                                "note": "algorithmic FLOPs (rope scored once, one query term) over the bf16 dense peak"},
            "clocks": clocks,
            "e2e": {"value": job_tbs(kv, world, e2e_ms), "unit": "TB/s", "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps},
            "e2e_resident_cache": {"value": job_tbs(kv, world, res_ms), "unit": "TB/s", "ms_per_step": res_ms,
                                   "h2d_bytes_per_step": h2d_res, "d2h_bytes_per_step": d2h, "steps": r_steps,
                                   "note": "cache and weights resident in HBM; per step the query, lengths "
                                           "(and block table) are copied in and out is copied back"},
            "gpu_launches": 4 * args.steps,  # absorb, decode, merge, up-projection per step
        }
        if world == 1 and not args.no_cpu_baseline:
            dt, frac, threads, ns, nh = time_oracle_sample(wl, args.cpu_seqs, args.cpu_heads, tpw, gla, int8)
            cpu_step = dt / frac
            line["cpu_baseline"] = {
                "value": kv / cpu_step / 1e12, "unit": "TB/s", "cores": threads, "kind": "oracle",
                "us_per_step": cpu_step * 1e6, "seconds_measured": dt,
                "sample": (f"fp64 expanded-definition oracle on {ns} sequence(s) x {nh} head(s), "
                           f"extrapolated by cached tokens x heads to the full step")}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    del ws


def prefill_flops(L: int, n: int, heads: int, n_branch: int = 4) -> int:
    """Algorithmic FLOPs of one expanded-form prefill: forming K_nope and V for every cached
    token (2 products of L x 512 x 128 per head) and, per head and branch, a 192-wide score
    and a 128-wide P.V for every (query, visible key) pair."""
    pairs = n * (L - n) + n * (n + 1) // 2
    return 4 * L * 512 * 128 * heads + 2 * (192 + 128) * pairs * heads * n_branch


def run_cp_bench(args, wl, world, rank, local):
    """One batch of sequences split over `args.cp` devices by token range: each rank decodes
    its range into partial states, the states are all-gathered (NCCL) and every rank merges
    them and finishes the decode.  On one GPU, rank 0 runs alone with its own state standing
    in for the others' (no all-gather)."""
    import head_rank_attention_b200 as hra
    from head_rank_attention_b200 import cp
    torch.cuda.set_device(local)
    W = args.cp
    inp = synth.make_inputs(wl)
    lengths = [int(x) for x in inp.seq_lens]
    starts, counts = cp.token_ranges(lengths, rank, W)
    T = max(max(counts), 1)
    local_cache = torch.zeros(wl.batch * T, inp.cache.shape[1], dtype=inp.cache.dtype, device="cuda")
    for s in range(wl.batch):
        rows = synth.logical_rows(inp, wl, s)[starts[s]:starts[s] + counts[s]]
        local_cache[s * T:s * T + counts[s]] = rows.cuda()
    q = inp.q.cuda()
    w_uk, w_uv = inp.w_uk.cuda(), inp.w_uv.cuda()
    seq_lens = torch.tensor(counts, dtype=torch.int32, device="cuda")
    q_pos = torch.tensor([max(n - 1, 0) for n in lengths], dtype=torch.int32, device="cuda")
    part_o = torch.zeros(wl.batch, wl.heads, synth.D_C, device="cuda")
    part_lse = torch.zeros(wl.batch, wl.heads, synth.D_C // 128, device="cuda")
    kw = dict(n_branch=wl.n_branch, alpha_q=wl.alpha_q, alpha_kv=wl.alpha_kv, branch_scale=wl.sigma_o,
              softmax_scale=wl.softmax_scale, rope_theta=wl.rope_theta)
    p = hra.make_params(q, local_cache[:, :synth.D_C], local_cache[:, synth.D_C:], seq_lens, w_uk, w_uv, None,
                        seq_stride=T, q_positions=q_pos, part_o=part_o, part_lse=part_lse, **kw)
    ws = hra.alloc_workspace(p)
    out = torch.empty(wl.batch, wl.heads, synth.D_V, dtype=torch.float32, device="cuda")
    pc = hra.make_params(q, local_cache[:, :synth.D_C], local_cache[:, synth.D_C:], seq_lens, w_uk, w_uv, out,
                         seq_stride=T, **kw)
    ws_c = hra.alloc_workspace(pc)
    stream = torch.cuda.current_stream()
    if world > 1:
        gather = lambda: cp.gather_partials(part_o, part_lse)  # noqa: E731
    else:
        stand_o = part_o.unsqueeze(0).expand(W, *part_o.shape)
        stand_l = part_lse.unsqueeze(0).expand(W, *part_lse.shape)
        gather = lambda: (stand_o.contiguous(), stand_l.contiguous())  # noqa: E731

    def one_step():
        hra.mlra_decode(p, stream)
        go, gl = gather()
        hra.combine_partials(pc, go, gl, stream)

    for _ in range(args.warmup):
        one_step()
    hra.check_device_status(p, stream)
    hra.check_device_status(pc, stream)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with ClockSampler(torch.cuda.current_device()) as clk:
        for e0, e1, e2 in ev:
            e0.record(stream)
            hra.mlra_decode(p, stream)
            e1.record(stream)
            go, gl = gather()
            hra.combine_partials(pc, go, gl, stream)
            e2.record(stream)
        torch.cuda.synchronize()
    hra.check_device_status(pc, stream)
    step_ms = statistics.median(e0.elapsed_time(e2) for e0, _, e2 in ev)
    range_ms = statistics.median(e0.elapsed_time(e1) for e0, e1, _ in ev)
    step_ms, range_ms = max_over_ranks([step_ms, range_ms], world, "cuda")
    if rank != 0:
        return
    range_bytes = 1152 * sum(counts)
    all_bytes = 1152 * sum(lengths)
    done = all_bytes if world == W else range_bytes  # the tokens this job decoded
    pk, pk_src = peaks()
    line = {
        "metric": f"MLRA decode us/step with each sequence split by token range over {W} devices",
        "value": done / (step_ms * 1e-3) / 1e12, "unit": "TB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "us_per_step": step_ms * 1e3, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": {"workload": wl.name, "split": W, "tokens_per_rank": counts,
                   "parallelism": (f"cp{W}: NCCL all-gather of the partial states" if world == W else
                                   f"cp{W}: rank 0's range alone, its state standing in for the other ranks' "
                                   f"(no all-gather)"),
                   "l2": "the range's cache is larger than L2 (no flush)" if range_bytes > (126 << 20)
                         else "the range's cache fits in L2 (no flush: a lower bound on the time)"},
        "stage_us": {"range_decode": range_ms * 1e3, "gather_and_combine": (step_ms - range_ms) * 1e3},
        "roofline": {"bound": "hbm", "achieved": range_bytes / (range_ms * 1e-3) / 1e9, "peak": pk["hbm_gbs"],
                     "unit": "GB/s", "frac": range_bytes / (range_ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                     "peak_source": pk_src, "traffic": None,
                     "note": "the range's KV bytes over the whole range call (absorb, decode, merge)"},
        "clocks": clk.summary(),
        "e2e": None,
        "gpu_launches": 5 * args.steps,  # absorb, decode, merge; partial combine, up-projection
    }
    print(json.dumps(line), flush=True)


def run_prefill_bench(args, world, rank, local):
    """Prefill of one MLRA-4 sequence (h = 128): the three kernels of mlra_prefill per step."""
    import head_rank_attention_b200 as hra
    torch.cuda.set_device(local)
    L = args.prefill
    n = args.prefill_queries or L
    wl = synth.Workload(f"prefill_mlra4_h128_L{L}_n{n}", 4, 1, 128, L)
    inp = synth.make_inputs(wl)
    q = synth.queries(synth.Workload(wl.name + "_q", 4, n, 128, L, seed=7))
    dev = synth.to_device(inp)
    cache = dev.cache[:L]
    qd = q.cuda()
    out = torch.empty(n, wl.heads, synth.D_V, dtype=torch.float32, device="cuda")
    p = hra.make_prefill_params(qd, cache[:, :512], cache[:, 512:], dev.w_uk, dev.w_uv, out, n_branch=4,
                                branch_scale=wl.sigma_o, softmax_scale=wl.softmax_scale, rope_theta=wl.rope_theta)
    ws = hra.alloc_prefill_workspace(p)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        hra.mlra_prefill(p, stream)
    hra.check_prefill_status(p, stream)
    # the expanded keys and values (2 * 4 * 128 * L_pad * 128 fp16) exceed L2 from L = 512 on;
    # below that, L2 is flushed before every step
    flush = torch.zeros(128 << 20, dtype=torch.float32, device="cuda") if L < 1024 else None
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with ClockSampler(torch.cuda.current_device()) as clk:
        for e0, e1 in pairs:
            if flush is not None:
                flush.add_(1)
            e0.record(stream)
            hra.mlra_prefill(p, stream)
            e1.record(stream)
        torch.cuda.synchronize()
    hra.check_prefill_status(p, stream)
    step_ms = statistics.median(e0.elapsed_time(e1) for e0, e1 in pairs)
    # end to end: host copies of the query, the sequence's cache rows and the weights in, out back
    pin = dict(q=q.pin_memory(), cache=inp.cache[:L].contiguous().pin_memory(), w_uk=inp.w_uk.pin_memory(),
               w_uv=inp.w_uv.pin_memory())
    dmap = dict(q=qd, cache=cache, w_uk=dev.w_uk, w_uv=dev.w_uv)
    host_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = host_out.numel() * host_out.element_size()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    for _ in range(e2e_steps):
        for k, t in pin.items():
            dmap[k].copy_(t, non_blocking=True)
        hra.mlra_prefill(p, stream)
        host_out.copy_(out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    step_ms, e2e_ms = max_over_ranks([step_ms, e2e_ms], world, "cuda")
    if rank != 0:
        return
    flops = prefill_flops(L, n, wl.heads)
    pk, pk_src = peaks()
    tflops = world * flops / (step_ms * 1e-3) / 1e12
    line = {
        "metric": "MLRA-4 prefill TFLOP/s (expanded form)", "value": tflops, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "precision": "bf16 inputs; fp16 tensor-core operands (queries, expanded K/V); fp32 accumulate and softmax",
        "data": "synthetic",
        "config": {"workload": wl.name, "variant": "MLRA-4 prefill", "heads": wl.heads, "seq_len": L,
                   "queries": n, "d_c": 512, "d_rope": 64, "flops_per_step": flops,
                   "l2": "expanded K/V larger than L2; no flush" if flush is None else "512 MB written before every step"},
        "roofline": {"bound": "tensor", "achieved": tflops / world, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": tflops / world / pk["bf16_tflops"], "peak_source": pk_src, "traffic": None,
                     "note": "algorithmic FLOPs of the whole call (expansion + causal attention) over the "
                             "measured dense bf16 peak (fp16 runs at the same rate)"},
        "clocks": clk.summary(),
        "e2e": {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "gpu_launches": 3 * args.steps,  # prep, expand, attend per step
    }
    if world == 1 and not args.no_cpu_baseline:
        # the oracle on a bounded sample (2 heads, the last min(n, 32) queries), scaled by FLOPs
        hs, ns = 2, min(n, 32)
        rows = inp.cache[:L]
        t0 = time.perf_counter()
        oracle_mod = __import__("oracle")
        oracle_mod.mlra_prefill_expanded(q[n - ns:, :hs], rows[:, :512], rows[:, 512:], inp.w_uk[:hs], inp.w_uv[:hs], 4,
                                         branch_scale=wl.sigma_o, softmax_scale=wl.softmax_scale,
                                         rope_theta=wl.rope_theta)
        dt = time.perf_counter() - t0
        sample_flops = prefill_flops(L, ns, hs)
        cpu_tflops = sample_flops / dt / 1e12
        line["cpu_baseline"] = {"value": cpu_tflops, "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
                                "seconds_measured": dt,
                                "sample": f"fp64 expanded prefill oracle on {hs} heads x the last {ns} queries "
                                          f"(its own algorithmic FLOPs over its time)"}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default="paged_b64_t32k_mlra4", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--num-splits", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-seqs", type=int, default=4)
    ap.add_argument("--cpu-heads", type=int, default=16)
    ap.add_argument("--ref-seqs", type=int, default=1)
    ap.add_argument("--ref-heads", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="time direct calls instead of CUDA-graph replays")
    ap.add_argument("--tp", type=int, default=0, choices=[0, 2, 4],
                    help="tensor parallelism by branch over this many ranks (MLRA-4 workloads)")
    ap.add_argument("--fused-out", action="store_true",
                    help="with --tp on several GPUs: the up-projection adds into every rank's out")
    ap.add_argument("--cache", default="bf16", choices=["bf16", "int8"],
                    help="latent cache format (int8: MLRA-4 workloads and their branch shards)")
    ap.add_argument("--gla", type=int, default=0, choices=[0, 2],
                    help="a rank of GLA-2 on an MLA workload (2 latent groups, half the heads each)")
    ap.add_argument("--prefill", type=int, default=0, help="time the prefill path over this many cached tokens")
    ap.add_argument("--cp", type=int, default=0,
                    help="split every sequence over this many devices by token range (rank 0 alone on one GPU)")
    ap.add_argument("--prefill-queries", type=int, default=0, help="query tokens of --prefill (default: all)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        sys.exit(self_launch(args.gpus))
    world, rank, local = dist_setup()
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}: run one rank per GPU")
    wl = synth.WORKLOADS[args.workload]
    if args.tp and (wl.n_branch == 1 or wl.n_branch % args.tp != 0):
        ap.error(f"--tp {args.tp} needs whole branches per rank (MLRA-4: 2 or 4; MLRA-2: 2)")
    if args.fused_out and not (args.tp and world == args.tp > 1):
        ap.error("--fused-out needs --tp W on W > 1 ranks")
    if args.cache == "int8" and (args.gla or (512 // wl.n_branch) != 128):
        ap.error("--cache int8 takes an MLRA-4 workload (128-wide branches)")
    if args.gla and (wl.n_branch != 1 or args.tp):
        ap.error("--gla 2 takes an MLA workload and no --tp")
    if args.gla and world not in (1, args.gla):
        ap.error(f"--gla {args.gla} runs on {args.gla} ranks (or one GPU for a single group), not {world}")
    if args.tp and world not in (1, args.tp):
        ap.error(f"--tp {args.tp} runs on {args.tp} ranks (or one GPU for a single shard), not {world}")
    if args.prefill:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the prefill mode has no reference arm; the oracle "
                                                                  "sample is reported as cpu_baseline"}))
            return
        run_prefill_bench(args, world, rank, local)
    elif args.cp:
        if world not in (1, args.cp) or args.tp or args.gla or args.cache != "bf16" or wl.page_size:
            ap.error(f"--cp {args.cp} runs on {args.cp} ranks (or one GPU), bf16, contiguous, no --tp / --gla")
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the token-range split has no reference arm"}))
            return
        run_cp_bench(args, wl, world, rank, local)
    elif args.impl == "reference":
        run_reference(args, wl, world, rank)
    else:
        run_native(args, wl, world, rank, local)


if __name__ == "__main__":
    main()
