"""The N > 1 host path of bench.py on CPU: two gloo ranks (one process each, rendezvous
on 127.0.0.1).  Every rank decodes its own replica, so the only cross-rank steps are the
maximum of the per-rank times and the whole-job throughput; both are checked here."""
import datetime
import io
import os
import socket
import sys
import contextlib

import pytest
import torch
import torch.multiprocessing as mp

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

WORLD = 2


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, queue) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        setup = bench.dist_setup()
        # rank r reports times (1 + r, 10 - r, r / 2): the job's are the maxima
        times = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 0.5 * rank], world, "cpu")
        tbs = bench.job_tbs(10 ** 12, world, 1000.0)  # 1 TB per rank per 1 s step
        queue.put((rank, setup, times, tbs))
        torch.distributed.barrier()
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_sum_the_bytes():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, WORLD, port, queue)) for r in range(WORLD)]
    for p in procs:
        p.start()
    try:
        results = sorted(queue.get(timeout=120) for _ in range(WORLD))
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert [p.exitcode for p in procs] == [0] * WORLD
    for rank, setup, times, tbs in results:
        assert setup == (WORLD, rank, rank)
        assert times == [float(WORLD), 10.0, 0.5 * (WORLD - 1)]
        assert tbs == pytest.approx(float(WORLD))


def test_single_rank_reduction_is_the_identity():
    import bench
    assert bench.max_over_ranks([3, 1.5], 1, "cpu") == [3.0, 1.5]
    assert bench.job_tbs(6 * 10 ** 9, 1, 1.0) == pytest.approx(6.0)


def test_reference_arm_prints_nothing_on_other_ranks():
    """Under torchrun only rank 0 times the oracle; the other ranks exit without work."""
    import argparse

    import bench
    import synth
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        bench.run_reference(argparse.Namespace(steps=1, warmup=3, ref_seqs=1, ref_heads=1),
                            synth.WORKLOADS["small_mlra4_h16_t2k"], 2, 1)
    assert out.getvalue() == ""


def test_reference_arm_for_a_branch_shard_reports_the_shard():
    """--tp 4 on the reference arm times the oracle on rank 0's shard: one 128-wide branch
    plus the rope key per token, strong scaling, and the shard's latent width in config."""
    import argparse
    import json

    import bench
    import synth
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        bench.run_reference(argparse.Namespace(steps=1, warmup=3, ref_seqs=1, ref_heads=1, tp=4),
                            synth.WORKLOADS["small_mlra4_h16_t2k"], 1, 0)
    line = json.loads(out.getvalue())
    assert line["impl"] == "reference" and line["scaling"] == "strong"
    assert line["config"]["d_c"] == 128 and line["config"]["tp_shard"] == "1 of 4 branches per rank"
    tokens = 2048
    assert line["value"] == pytest.approx(tokens * (128 + 64) * 2 / (line["ms_per_step"] * 1e-3) / 1e12)
    assert line["cpu_baseline"]["value"] == line["value"] and line["e2e"]["value"] == line["value"]


def test_tensor_flops_per_token_of_a_shard():
    import bench
    assert bench.tensor_flops_per_token(4, 128) == 2176 * 128
    assert bench.tensor_flops_per_token(1, 128, 128) == (2 * 192 + 2 * 128) * 128


def _bench_cmd(*extra):
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    return [sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "1", "--warmup", "3",
            "--ref-seqs", "1", "--ref-heads", "1", "--workload", "small_mlra4_h16_t2k", *extra]


def test_gpus_flag_launches_that_many_ranks():
    """bench.py --gpus 2 run by hand (no torchrun) launches itself as two ranks; rank 0
    alone prints the line, which reports both ranks."""
    import json
    import subprocess
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run(_bench_cmd("--gpus", "2"), env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    assert lines[0]["n_gpus"] == 2 and lines[0]["impl"] == "reference"


def test_gpus_flag_must_match_the_launcher():
    """Under a launcher, --gpus must equal WORLD_SIZE."""
    import subprocess
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run(_bench_cmd("--gpus", "2"), env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 2 and "WORLD_SIZE=1" in r.stderr


def test_reference_arm_for_a_gla2_rank_reports_the_group():
    """--gla 2 on an MLA workload: rank 0's group is 256 latent columns, the rope key and
    half of the heads; 2.5 d_h of cache per token."""
    import argparse
    import json

    import bench
    import synth
    wl = synth.Workload("gla_small", 1, 1, 16, 2048)
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        bench.run_reference(argparse.Namespace(steps=1, warmup=3, ref_seqs=1, ref_heads=1, tp=0, gla=2), wl, 1, 0)
    line = json.loads(out.getvalue())
    assert line["config"]["d_c"] == 256 and line["config"]["heads"] == 8
    assert line["config"]["variant"] == "GLA-2 rank"
    assert line["value"] == pytest.approx(2048 * (256 + 64) * 2 / (line["ms_per_step"] * 1e-3) / 1e12)


def test_prefill_flop_count_matches_a_brute_count():
    """The prefill bench's algorithmic FLOPs: K and V for every cached token, and per head and
    branch a 192-wide score and a 128-wide P.V for every visible (query, key) pair."""
    import bench
    L, n, h, nb = 9, 4, 3, 4
    pairs = sum(1 for j in range(n) for t in range(L) if t <= L - n + j)
    assert bench.prefill_flops(L, n, h, nb) == 4 * L * 512 * 128 * h + 2 * 320 * pairs * h * nb


def test_recorded_traffic_is_keyed_by_shard_group_and_cache_format(tmp_path):
    """A launch reads the traffic recorded for its own kernel and bytes: the int8 cache, a
    branch shard or a GLA group never picks up the bf16 whole-model figure, and a record
    taken from other kernel sources is ignored."""
    import json
    import bench
    assert bench.traffic_key("paged_b64_t32k_mlra4") == "paged_b64_t32k_mlra4"
    keys = {bench.traffic_key("w", tp=4), bench.traffic_key("w", gla=2), bench.traffic_key("w", int8=True),
            bench.traffic_key("w", tp=4, int8=True), bench.traffic_key("w")}
    assert len(keys) == 5
    sha = bench.decode_source_hash()
    rec = {"w": {"decode_source_sha": sha, "dram_bytes_per_launch": 123},
           "w/int8": {"decode_source_sha": "0" * 16, "dram_bytes_per_launch": 45}}
    f = tmp_path / "traffic.json"
    f.write_text(json.dumps(rec))
    assert bench.ncu_traffic(bench.traffic_key("w"), f) == 123
    assert bench.ncu_traffic(bench.traffic_key("w", int8=True), f) is None   # stale source
    assert bench.ncu_traffic(bench.traffic_key("w", tp=4), f) is None        # not recorded


@pytest.mark.parametrize("extra", [["--tp", "4"], ["--workload", "paged_b64_t32k_mlra4"], ["--cache", "int8"]])
def test_token_range_split_mode_refuses_other_layouts(extra):
    """--cp W takes contiguous bf16 workloads without --tp / --gla; the rest is refused
    before any device work."""
    import subprocess
    args = ["--cp", "2", "--workload", "long_mlra4_b4_t64k_128k"] + extra
    r = subprocess.run(_bench_cmd(*args), capture_output=True, text=True, timeout=300)
    assert r.returncode == 2 and "--cp 2" in r.stderr, r.stderr[-300:]


def test_token_range_split_has_no_reference_arm():
    import json
    import subprocess
    r = subprocess.run(_bench_cmd("--cp", "2", "--workload", "long_mlra4_b4_t64k_128k", "--impl", "reference"),
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    line = json.loads([x for x in r.stdout.splitlines() if x.startswith("{")][0])
    assert line["impl"] == "reference" and "unavailable" in line
