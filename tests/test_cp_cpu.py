"""A sequence split by token range over two gloo ranks (CPU): each rank takes its range
(head_rank_attention_b200.cp), computes the oracle's partial state of it with the query at
the sequence's last position, the ranks all-gather the states in rank order, and merging
them gives the oracle's decode of the whole sequence on every rank.  This covers the host
side of the split (ranges, gather, order); the GPU path is tested by test_cp_gpu.py."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from head_rank_attention_b200 import cp


def test_token_ranges_partition_every_sequence():
    for L in (0, 1, 2, 3, 7, 64, 1000):
        for world in (1, 2, 3, 4, 8):
            ranges = [cp.token_range(L, r, world) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == L
            assert all(a <= b for a, b in ranges)
            assert all(ranges[r][1] == ranges[r + 1][0] for r in range(world - 1))
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1
    starts, counts = cp.token_ranges([10, 3], 1, 2)
    assert (starts, counts) == ([5, 1], [5, 2])
    with pytest.raises(ValueError):
        cp.token_range(10, 2, 2)


def _case():
    rng = np.random.default_rng(11)
    h, L = 3, 37
    return (rng.standard_normal((h, 192)), rng.standard_normal((L, 512)), rng.standard_normal((L, 64)),
            rng.standard_normal((h, 512, 128)) / 16, rng.standard_normal((h, 512, 128)) / 16)


def _rank(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        qv, C, KR, wk, wv = _case()
        L = C.shape[0]
        a, b = cp.token_range(L, rank, world)
        o, lse = oracle.mlra_partial_state(qv, C[a:b], KR[a:b], wk, 4, L - 1, alpha_q=1.1, alpha_kv=0.9)
        po = torch.from_numpy(o.reshape(1, o.shape[0], -1))          # [B = 1, h, d_c]
        pl = torch.from_numpy(lse.reshape(1, lse.shape[0], -1))      # [B = 1, h, d_c / 128]
        go, gl = cp.gather_partials(po, pl)
        states = [(go[r, 0].numpy().reshape(o.shape), gl[r, 0].numpy()) for r in range(world)]
        mo, _ = oracle.combine_partial_states(states)
        got = oracle.upproject_latent(mo, wv, alpha_kv=0.9)
        ref = oracle.mlra_decode_expanded(qv, C, KR, wk, wv, 4, alpha_q=1.1, alpha_kv=0.9)
        q.put((rank, float(np.abs(got - ref).max())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ranks_merge_their_ranges_into_the_whole_sequence_decode(world):
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    errs = dict(q.get(timeout=10) for _ in range(world))
    assert sorted(errs) == list(range(world))
    assert max(errs.values()) < 1e-12, errs
