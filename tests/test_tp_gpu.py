"""GPU parity of branch shards (tensor parallelism by branch, "Multi-Head Low-Rank
Attention", 核心方法: under 4-way TP each device holds one MLRA-4 branch).

Every rank of a 2- or 4-way split runs here in turn on the one GPU: each call holds its
shard of the cache (its 128-wide branches + K_RoPE, laid out by head_rank_attention_b200.tp)
and of W_UK / W_UV, and the shard outputs are summed on the device as the all-reduce
would.  Each shard is compared with the oracle on the same shard, and the sum with the
oracle's MLRA-4 output, under the parity bar.
"""
import numpy as np
import pytest
import torch

import head_rank_attention_b200 as hra
from head_rank_attention_b200 import tp
import oracle
import synth
from gpu_cases import assert_parity

pytestmark = pytest.mark.gpu


def _wl(name, lengths, heads=128, page_size=0, **kw):
    return synth.Workload(name, 4, len(lengths), heads, max(lengths), page_size=page_size,
                          lengths=tuple(lengths), **kw)


CASES = [
    (_wl("tails", (1, 31, 32, 33, 127, 128, 129, 1000)), 4, 0),
    (_wl("tails", (1, 31, 32, 33, 127, 128, 129, 1000)), 2, 0),
    (_wl("paged64", (5, 64, 65, 700), page_size=64), 4, 0),
    (_wl("paged32", (5, 64, 65, 700), page_size=32), 2, 0),
    (_wl("h16", (2048,), heads=16, alpha_q=2048 ** 0.5 / 1536 ** 0.5, alpha_kv=2.0, branch_scale=0.5), 4, 0),
    (_wl("stress", (3000, 17), alpha_q=synth.A_Q_V3, alpha_kv=synth.A_KV_V3), 4, 0),
    (_wl("splits1", (1, 130, 2000, 64)), 4, 1),
    (_wl("splits200", (1, 130, 2000, 64)), 2, 200),
]


def _run_shard(dev, wl, rank, world, num_splits):
    local = tp.shard_cache(dev.cache, rank, world)
    w_uk, w_uv = tp.shard_weights(dev.w_uk, dev.w_uv, rank, world)
    d = local.shape[1] - synth.D_ROPE
    out = torch.empty(wl.batch, wl.heads, synth.D_V, dtype=torch.float32, device="cuda")
    p = hra.make_params(dev.q, local[:, :d], local[:, d:], dev.seq_lens, w_uk, w_uv, out,
                        n_branch=4 // world, alpha_q=wl.alpha_q, alpha_kv=wl.alpha_kv,
                        branch_scale=wl.sigma_o, softmax_scale=wl.softmax_scale, rope_theta=wl.rope_theta,
                        block_table=dev.block_table, page_size=wl.page_size, seq_stride=dev.seq_stride,
                        num_splits=num_splits)
    assert p.d_c == d == 512 // world
    ws = hra.alloc_workspace(p)
    ws.fill_(0xFF)  # NaN bytes: a read of a slot the call did not write shows up
    hra.mlra_decode(p)
    hra.check_device_status(p)
    return out


def _shard_ref(inp, wl, rank, world, seqs=None):
    w_uk, w_uv = tp.shard_weights(inp.w_uk, inp.w_uv, rank, world)
    res = []
    for s in range(wl.batch) if seqs is None else seqs:
        local = tp.shard_cache(synth.logical_rows(inp, wl, s), rank, world)
        d = local.shape[1] - synth.D_ROPE
        res.append(oracle.mlra_decode_absorbed(inp.q[s], local[:, :d], local[:, d:], w_uk, w_uv, 4 // world,
                                               alpha_q=wl.alpha_q, alpha_kv=wl.alpha_kv, branch_scale=wl.sigma_o,
                                               softmax_scale=wl.softmax_scale, rope_theta=wl.rope_theta))
    return np.stack(res)


@pytest.mark.parametrize("wl,world,num_splits", CASES,
                         ids=[f"{c[0].name}-tp{c[1]}-splits{c[2]}" for c in CASES])
def test_branch_shards_match_the_oracle_and_sum_to_mlra4(wl, world, num_splits):
    inp = synth.make_inputs(wl)
    dev = synth.to_device(inp)
    total = torch.zeros(wl.batch, wl.heads, synth.D_V, dtype=torch.float32, device="cuda")
    for r in range(world):
        out = _run_shard(dev, wl, r, world, num_splits)
        assert_parity(out.cpu().numpy(), _shard_ref(inp, wl, r, world), f"{wl.name} shard {r}/{world}")
        total += out
    ref = oracle.decode_batch(inp, wl, form="absorbed")
    assert_parity(total.cpu().numpy(), ref, f"{wl.name} sum of {world} shards")


def test_zero_length_sequence_gives_zero_row_in_every_shard():
    wl = _wl("zero", (0, 300, 0, 33))
    inp = synth.make_inputs(wl)
    dev = synth.to_device(inp)
    for world in (4, 2):
        for r in range(world):
            out = _run_shard(dev, wl, r, world, 0).cpu()
            assert (out[0] == 0).all() and (out[2] == 0).all()
            assert_parity(out[[1, 3]].numpy(), _shard_ref(inp, wl, r, world, seqs=[1, 3]),
                          f"zero-length neighbours, shard {r}/{world}")


def test_shard_bf16_output():
    wl = _wl("bf16", (700, 33))
    inp = synth.make_inputs(wl)
    dev = synth.to_device(inp)
    local = tp.shard_cache(dev.cache, 3, 4)
    w_uk, w_uv = tp.shard_weights(dev.w_uk, dev.w_uv, 3, 4)
    out = torch.empty(wl.batch, wl.heads, synth.D_V, dtype=torch.bfloat16, device="cuda")
    p = hra.make_params(dev.q, local[:, :128], local[:, 128:], dev.seq_lens, w_uk, w_uv, out, n_branch=1,
                        branch_scale=wl.sigma_o, seq_stride=dev.seq_stride)
    ws = hra.alloc_workspace(p)
    hra.mlra_decode(p)
    hra.check_device_status(p)
    assert_parity(out.float().cpu().numpy(), _shard_ref(inp, wl, 3, 4), "bf16 out, shard 3/4")
    del ws


def test_shard_graph_replay_and_determinism():
    """A shard call replayed from a CUDA graph, and called again directly, gives the same bits."""
    wl = _wl("graph", (1500, 40))
    dev = synth.to_device(synth.make_inputs(wl))
    ref = _run_shard(dev, wl, 1, 4, 0)
    assert torch.equal(_run_shard(dev, wl, 1, 4, 0), ref)
    local = tp.shard_cache(dev.cache, 1, 4)
    w_uk, w_uv = tp.shard_weights(dev.w_uk, dev.w_uv, 1, 4)
    out = torch.zeros_like(ref)
    p = hra.make_params(dev.q, local[:, :128], local[:, 128:], dev.seq_lens, w_uk, w_uv, out, n_branch=1,
                        branch_scale=wl.sigma_o, seq_stride=dev.seq_stride)
    ws = hra.alloc_workspace(p)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        hra.mlra_decode(p, torch.cuda.current_stream())
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    hra.check_device_status(p)
    del g, ws


def test_shard_paged_equals_contiguous_bitwise():
    lens = (100, 640, 33)
    outs = []
    for page_size in (0, 32):
        wl = _wl("layout", lens, page_size=page_size)
        outs.append(_run_shard(synth.to_device(synth.make_inputs(wl)), wl, 2, 4, 0))
    assert torch.equal(outs[0], outs[1])


# --- one 256-wide latent per call: MLRA-2 split by branch, and GLA-2 ranks -------------------

def _wl2(name, lengths, heads=128, page_size=0, **kw):
    return synth.Workload(name, 2, len(lengths), heads, max(lengths), page_size=page_size,
                          lengths=tuple(lengths), **kw)


CASES_256 = [
    _wl2("tails", (1, 31, 32, 33, 63, 64, 65, 1000)),
    _wl2("paged32", (5, 64, 65, 700), page_size=32),
    _wl2("stress", (3000, 17), alpha_q=synth.A_Q_V3, alpha_kv=synth.A_KV_V3),
]


def _call(q, local, w_uk, w_uv, dev, wl, n_branch, branch_scale):
    d = local.shape[1] - synth.D_ROPE
    out = torch.empty(q.shape[0], q.shape[1], synth.D_V, dtype=torch.float32, device="cuda")
    p = hra.make_params(q, local[:, :d], local[:, d:], dev.seq_lens, w_uk, w_uv, out, n_branch=n_branch,
                        alpha_q=wl.alpha_q, alpha_kv=wl.alpha_kv, branch_scale=branch_scale,
                        softmax_scale=wl.softmax_scale, rope_theta=wl.rope_theta, block_table=dev.block_table,
                        page_size=wl.page_size, seq_stride=dev.seq_stride)
    ws = hra.alloc_workspace(p)
    ws.fill_(0xFF)
    hra.mlra_decode(p)
    hra.check_device_status(p)
    return out


@pytest.mark.parametrize("wl", CASES_256, ids=lambda w: w.name)
def test_mlra2_branch_shards_sum_to_mlra2(wl):
    """2-way tensor parallelism of MLRA-2: each rank holds one 256-wide branch (d_c = 256,
    n_branch = 1, branch_scale 1/sqrt(2)); the ranks' outputs sum to MLRA-2's."""
    inp = synth.make_inputs(wl)
    dev = synth.to_device(inp)
    total = torch.zeros(wl.batch, wl.heads, synth.D_V, dtype=torch.float32, device="cuda")
    for r in range(2):
        local = tp.shard_cache(dev.cache, r, 2, n_branch=2)
        w_uk, w_uv = tp.shard_weights(dev.w_uk, dev.w_uv, r, 2, n_branch=2)
        out = _call(dev.q, local, w_uk, w_uv, dev, wl, 1, wl.sigma_o)
        h_uk, h_uv = tp.shard_weights(inp.w_uk, inp.w_uv, r, 2, n_branch=2)
        ref = np.stack([oracle.mlra_decode_absorbed(
            inp.q[s], *(lambda x: (x[:, :256], x[:, 256:]))(tp.shard_cache(synth.logical_rows(inp, wl, s), r, 2,
                                                                           n_branch=2)),
            h_uk, h_uv, 1, alpha_q=wl.alpha_q, alpha_kv=wl.alpha_kv, branch_scale=wl.sigma_o,
            softmax_scale=wl.softmax_scale, rope_theta=wl.rope_theta) for s in range(wl.batch)])
        assert_parity(out.cpu().numpy(), ref, f"{wl.name} MLRA-2 shard {r}/2")
        total += out
    assert_parity(total.cpu().numpy(), oracle.decode_batch(inp, wl, form="absorbed"), f"{wl.name} MLRA-2 sum")


@pytest.mark.parametrize("wl", CASES_256[:2], ids=lambda w: w.name)
def test_gla2_ranks_match_the_oracle(wl):
    """GLA-2 (研究动机: MLA's latent split into two groups): rank g holds latent group g and
    the heads of group g; its call is MLA over a 256-wide latent.  Head i's weights are the
    group's rows of the seeded [h, 512, 128] weights."""
    inp = synth.make_inputs(wl)
    dev = synth.to_device(inp)
    h, per = wl.heads, wl.heads // 2
    w_uk = torch.stack([inp.w_uk[i, (i // per) * 256:(i // per + 1) * 256] for i in range(h)])
    w_uv = torch.stack([inp.w_uv[i, (i // per) * 256:(i // per + 1) * 256] for i in range(h)])
    outs = []
    for g in range(2):
        heads = slice(g * per, (g + 1) * per)
        local = tp.shard_cache(dev.cache, g, 2, n_branch=2)
        outs.append(_call(dev.q[:, heads].contiguous(), local, w_uk[heads].cuda().contiguous(),
                          w_uv[heads].cuda().contiguous(), dev, wl, 1, 1.0))
    got = torch.cat(outs, dim=1).cpu().numpy()
    ref = np.stack([oracle.gla_decode(inp.q[s], (r := synth.logical_rows(inp, wl, s))[:, :512], r[:, 512:],
                                      w_uk, w_uv, 2, alpha_q=wl.alpha_q, alpha_kv=wl.alpha_kv,
                                      softmax_scale=wl.softmax_scale, rope_theta=wl.rope_theta)
                    for s in range(wl.batch)])
    assert_parity(got, ref, f"{wl.name} GLA-2")


# --- the up-projection adding into every rank's out (fused all-reduce) ---------------------

def _shard_params(dev, wl, rank, world, out, **kw):
    local = tp.shard_cache(dev.cache, rank, world)
    w_uk, w_uv = tp.shard_weights(dev.w_uk, dev.w_uv, rank, world)
    d = local.shape[1] - synth.D_ROPE
    p = hra.make_params(dev.q, local[:, :d], local[:, d:], dev.seq_lens, w_uk, w_uv, out, n_branch=4 // world,
                        alpha_q=wl.alpha_q, alpha_kv=wl.alpha_kv, branch_scale=wl.sigma_o,
                        softmax_scale=wl.softmax_scale, rope_theta=wl.rope_theta, block_table=dev.block_table,
                        page_size=wl.page_size, seq_stride=dev.seq_stride, **kw)
    return p, (local, w_uk, w_uv)


@pytest.mark.parametrize("wl", [_wl("tails", (1, 31, 129, 1000)), _wl("paged64", (5, 64, 65, 700), page_size=64)],
                         ids=lambda w: w.name)
def test_accumulating_shards_into_one_out_gives_mlra4(wl):
    """out_accumulate: the 4 ranks' calls add into one zeroed buffer; the sum is MLRA-4."""
    inp = synth.make_inputs(wl)
    dev = synth.to_device(inp)
    out = torch.zeros(wl.batch, wl.heads, synth.D_V, dtype=torch.float32, device="cuda")
    keep = []
    for r in range(4):
        p, k = _shard_params(dev, wl, r, 4, out, out_accumulate=True)
        keep.append((hra.alloc_workspace(p), k))
        hra.mlra_decode(p)
        hra.check_device_status(p)
    assert_parity(out.cpu().numpy(), oracle.decode_batch(inp, wl, form="absorbed"), f"{wl.name} accumulated")


def test_accumulate_of_one_call_equals_the_stored_output():
    wl = _wl("acc1", (700, 33))
    dev = synth.to_device(synth.make_inputs(wl))
    stored = _run_shard(dev, wl, 1, 4, 0)
    out = torch.zeros_like(stored)
    p, keep = _shard_params(dev, wl, 1, 4, out, out_accumulate=True)
    ws = hra.alloc_workspace(p)
    hra.mlra_decode(p)
    hra.check_device_status(p)
    assert torch.equal(out, stored)
    del ws, keep


@pytest.mark.parametrize("world", [4, 2])
def test_every_rank_out_receives_every_shard(world):
    """out_peers: rank r writes into its own out and the other ranks' (here buffers on the
    same GPU standing in for peer memory); run in rank order, every out ends with the same
    bits, the MLRA-4 output."""
    wl = _wl("peers", (1, 300, 2000))
    inp = synth.make_inputs(wl)
    dev = synth.to_device(inp)
    outs = [torch.zeros(wl.batch, wl.heads, synth.D_V, dtype=torch.float32, device="cuda") for _ in range(world)]
    keep = []
    for r in range(world):
        p, k = _shard_params(dev, wl, r, world, outs[r], out_accumulate=True,
                             out_peers=[outs[q] for q in tp.peer_ranks(r, world)])
        keep.append((hra.alloc_workspace(p), k))
        hra.mlra_decode(p)
        hra.check_device_status(p)
    for q in range(1, world):
        assert torch.equal(outs[q], outs[0])
    assert_parity(outs[0].cpu().numpy(), oracle.decode_batch(inp, wl, form="absorbed"), f"peers x{world}")


@pytest.mark.parametrize("n_branch,world", [(4, 4), (2, 2)])
def test_branch_shards_at_the_maximum_batch(n_branch, world):
    """B = 1024 with zero lengths, 8 heads: shards of 128-wide (MLRA-4 / 4) and 256-wide
    (MLRA-2 / 2) branches at the largest batch; their sum is the model's output."""
    rng = np.random.default_rng(13)
    lens = rng.integers(0, 300, size=1024)
    lens[rng.integers(0, 1024, size=20)] = 0
    wl = synth.Workload(f"maxbatch_tp{world}", n_branch, 1024, 8, int(lens.max()), lengths=tuple(int(x) for x in lens))
    inp = synth.make_inputs(wl)
    dev = synth.to_device(inp)
    total = torch.zeros(wl.batch, wl.heads, synth.D_V, dtype=torch.float32, device="cuda")
    for r in range(world):
        local = tp.shard_cache(dev.cache, r, world, n_branch=n_branch)
        w_uk, w_uv = tp.shard_weights(dev.w_uk, dev.w_uv, r, world, n_branch=n_branch)
        total += _call(dev.q, local, w_uk, w_uv, dev, wl, n_branch // world, wl.sigma_o)
    got = total.cpu().numpy()
    zero = lens == 0
    assert np.all(got[zero] == 0)
    ref = oracle.decode_batch(inp, wl, seqs=[int(s) for s in np.flatnonzero(~zero)], form="absorbed")
    assert_parity(got[~zero], ref, wl.name)
