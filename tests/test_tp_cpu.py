"""Tensor parallelism by branch ("Multi-Head Low-Rank Attention", 核心方法: under 4-way TP
each device holds one MLRA-4 branch), on the CPU.

* The shard layout of head_rank_attention_b200.tp, fed to the fp64 oracle shard by shard
  (each shard an MLRA call with d_c = 128 * branches held and the full model's branch
  scale), sums to the oracle's MLRA-4 output.  A wrong column range, a shard that drops
  or repeats K_RoPE, or weights sliced on the wrong axis fails this.
* Two gloo ranks each produce their shard's output and sum it with tp.all_reduce_out: the
  host side of the multi-GPU path.
"""
import datetime
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from head_rank_attention_b200 import tp  # noqa: E402


def _case(seed=0, h=3, L=19):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(h, 192, generator=g).to(torch.bfloat16)
    cache = torch.randn(L, 576, generator=g).to(torch.bfloat16)
    w_uk = (torch.randn(h, 512, 128, generator=g) / math.sqrt(128)).to(torch.bfloat16)
    w_uv = (torch.randn(h, 512, 128, generator=g) / math.sqrt(128)).to(torch.bfloat16)
    return q, cache, w_uk, w_uv


def _shard_out(q, cache, w_uk, w_uv, rank, world):
    local = tp.shard_cache(cache, rank, world)
    luk, luv = tp.shard_weights(w_uk, w_uv, rank, world)
    d = local.shape[1] - 64
    return oracle.mlra_decode_expanded(q, local[:, :d], local[:, d:], luk, luv, 4 // world,
                                       alpha_q=1.3, alpha_kv=0.7, branch_scale=0.5)


def test_shard_columns():
    assert tp.shard_columns(512, 4, 0, 4) == (0, 128)
    assert tp.shard_columns(512, 4, 3, 4) == (384, 512)
    assert tp.shard_columns(512, 4, 1, 2) == (256, 512)
    assert tp.shard_columns(512, 4, 0, 1) == (0, 512)
    for bad in [(512, 4, 0, 3), (512, 4, 4, 4), (512, 4, -1, 2), (510, 4, 0, 2)]:
        with pytest.raises(ValueError):
            tp.shard_columns(*bad)


def test_peer_ranks():
    assert tp.peer_ranks(0, 1) == []
    assert tp.peer_ranks(2, 4) == [0, 1, 3]
    assert tp.peer_ranks(1, 2) == [0]
    with pytest.raises(ValueError):
        tp.peer_ranks(4, 4)


def test_shard_layout():
    _, cache, w_uk, w_uv = _case()
    local = tp.shard_cache(cache, 2, 4)
    assert local.shape == (cache.shape[0], 192) and local.is_contiguous()
    assert torch.equal(local[:, :128], cache[:, 256:384])
    assert torch.equal(local[:, 128:], cache[:, 512:])
    luk, luv = tp.shard_weights(w_uk, w_uv, 1, 2)
    assert torch.equal(luk, w_uk[:, 256:]) and torch.equal(luv, w_uv[:, 256:])


@pytest.mark.parametrize("world", [2, 4])
def test_branch_shards_sum_to_the_mlra4_output(world):
    q, cache, w_uk, w_uv = _case(seed=world)
    full = oracle.mlra_decode_expanded(q, cache[:, :512], cache[:, 512:], w_uk, w_uv, 4,
                                       alpha_q=1.3, alpha_kv=0.7, branch_scale=0.5)
    parts = [_shard_out(q, cache, w_uk, w_uv, r, world) for r in range(world)]
    total = sum(parts)
    assert np.abs(total - full).max() <= 1e-12 * np.abs(full).max()
    # no shard alone is the answer (each carries only its branches)
    assert all(np.abs(p - full).max() > 1e-3 * np.abs(full).max() for p in parts)


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, queue) -> None:
    torch.distributed.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                                         world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        q, cache, w_uk, w_uv = _case(seed=7)
        out = torch.from_numpy(_shard_out(q, cache, w_uk, w_uv, rank, world)).to(torch.float32)
        tp.all_reduce_out(out)
        queue.put((rank, out.numpy()))
        torch.distributed.barrier()
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_all_reduce_their_shards():
    world = 2
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, queue)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        results = sorted((queue.get(timeout=120) for _ in range(world)), key=lambda x: x[0])
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert [p.exitcode for p in procs] == [0] * world
    q, cache, w_uk, w_uv = _case(seed=7)
    full = oracle.mlra_decode_expanded(q, cache[:, :512], cache[:, 512:], w_uk, w_uv, 4,
                                       alpha_q=1.3, alpha_kv=0.7, branch_scale=0.5)
    for _, out in results:
        assert np.abs(out - full).max() <= 1e-5 * np.abs(full).max()
    assert np.array_equal(results[0][1], results[1][1])
