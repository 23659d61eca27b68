"""GPU parity of one sequence split by token range (context parallelism).

Each of `world` ranks holds a contiguous token range of every sequence
(head_rank_attention_b200.cp.token_range) in a cache of its own, decodes it with the
query at the sequence's last position (q_positions) and writes its partial state
(part_o, part_lse); the stacked states go through hra_combine_partials into out, which
must match the fp64 oracle's decode of the whole sequences.  The ranks run one after
another on this GPU: their calls are independent, and the all-gather between them is
host-side plumbing tested on gloo ranks in test_cp_cpu.py."""
import numpy as np
import pytest
import torch

import head_rank_attention_b200 as hra
import oracle
import synth
from gpu_cases import assert_parity, run_gpu
from head_rank_attention_b200 import cp

pytestmark = pytest.mark.gpu


def _case(name, n_branch, lengths, heads=128, **kw):
    return synth.Workload(name, n_branch, len(lengths), heads, max(lengths), lengths=tuple(lengths), **kw)


def _rank_params(inp, wl, rank, world, dev_full):
    """Rank `rank`'s cache (its token range of every sequence, contiguous) and partial-mode
    parameters; returns (params, tensors to keep alive, part_o, part_lse)."""
    lengths = [int(x) for x in inp.seq_lens]
    starts, counts = cp.token_ranges(lengths, rank, world)
    T = max(max(counts), 1)
    local = torch.zeros(wl.batch, T, inp.cache.shape[1], dtype=inp.cache.dtype)
    for s in range(wl.batch):
        rows = synth.logical_rows(inp, wl, s)
        local[s, :counts[s]] = rows[starts[s]:starts[s] + counts[s]]
    local = local.view(wl.batch * T, -1).cuda()
    seq_lens = torch.tensor(counts, dtype=torch.int32, device="cuda")
    q_pos = torch.tensor([max(n - 1, 0) for n in lengths], dtype=torch.int32, device="cuda")
    h = wl.heads
    part_o = torch.full((wl.batch, h, synth.D_C), float("nan"), device="cuda")
    part_lse = torch.full((wl.batch, h, synth.D_C // 128), float("nan"), device="cuda")
    p = hra.make_params(dev_full.q, local[:, :synth.D_C], local[:, synth.D_C:], seq_lens, dev_full.w_uk,
                        dev_full.w_uv, None, n_branch=wl.n_branch, alpha_q=wl.alpha_q, alpha_kv=wl.alpha_kv,
                        branch_scale=wl.sigma_o, softmax_scale=wl.softmax_scale, rope_theta=wl.rope_theta,
                        seq_stride=T, q_positions=q_pos, part_o=part_o, part_lse=part_lse)
    ws = hra.alloc_workspace(p)
    ws.fill_(0xFF)
    return p, (local, seq_lens, q_pos, ws), part_o, part_lse


def _split_decode(inp, wl, world, out_dtype=torch.float32):
    dev = synth.to_device(inp)
    parts_o, parts_lse, keep = [], [], []
    for r in range(world):
        p, k, po, pl = _rank_params(inp, wl, r, world, dev)
        hra.mlra_decode(p)
        hra.check_device_status(p)
        keep.append(k)
        parts_o.append(po)
        parts_lse.append(pl)
    out = torch.empty(wl.batch, wl.heads, synth.D_V, dtype=out_dtype, device="cuda")
    pf = hra.make_params(dev.q, dev.ckv, dev.krope, dev.seq_lens, dev.w_uk, dev.w_uv, out, n_branch=wl.n_branch,
                         alpha_q=wl.alpha_q, alpha_kv=wl.alpha_kv, branch_scale=wl.sigma_o,
                         softmax_scale=wl.softmax_scale, rope_theta=wl.rope_theta, seq_stride=dev.seq_stride)
    ws = hra.alloc_workspace(pf)
    hra.combine_partials(pf, torch.stack(parts_o), torch.stack(parts_lse))
    hra.check_device_status(pf)
    torch.cuda.synchronize()
    return out, dev, pf, ws


CASES = [
    (1, _case("cp1_mlra4", 4, (300,))),
    (2, _case("cp2_mlra4", 4, (300, 77))),
    (3, _case("cp3_mlra4_empty_ranges", 4, (1000, 5, 2))),   # rank 0 holds no token of the last one
    (4, _case("cp4_mla", 1, (513, 130))),
    (2, _case("cp2_mlra2", 2, (700,))),
    (4, _case("cp4_h16", 4, (2048,), heads=16, alpha_q=2048 ** 0.5 / 1536 ** 0.5, alpha_kv=2.0, branch_scale=0.5)),
    (8, _case("cp8_outliers", 4, (5000,), outlier_frac=0.01)),
]


@pytest.mark.parametrize("world,wl", CASES, ids=[c[1].name for c in CASES])
def test_token_range_split_matches_the_whole_sequence(world, wl):
    inp = synth.make_inputs(wl)
    out, _, _, _ = _split_decode(inp, wl, world)
    assert_parity(out.cpu().numpy(), oracle.decode_batch(inp, wl, form="absorbed"), f"{wl.name} over {world}")


def test_one_range_and_combine_equal_the_decode_bitwise():
    """One range covering every token: the partial state through hra_combine_partials gives
    the same bits as mlra_decode (the merged rows reach the up-projection unchanged)."""
    wl = _case("cp1_bitwise", 4, (900, 130))
    inp = synth.make_inputs(wl)
    out, dev, _, _ = _split_decode(inp, wl, 1)
    ref, _, _ = run_gpu(dev, wl)
    assert torch.equal(out, ref)


def test_bf16_out_and_query_positions():
    wl = _case("cp2_bf16", 4, (640, 33))
    inp = synth.make_inputs(wl)
    out, dev, _, _ = _split_decode(inp, wl, 2, out_dtype=torch.bfloat16)
    assert_parity(out.float().cpu().numpy(), oracle.decode_batch(inp, wl, form="absorbed"), "bf16 out")
    # q_positions = L - 1 on a whole-sequence call changes nothing
    ref, _, _ = run_gpu(dev, wl)
    o2 = torch.empty_like(ref)
    pos = (dev.seq_lens - 1).to(torch.int32)
    p = hra.make_params(dev.q, dev.ckv, dev.krope, dev.seq_lens, dev.w_uk, dev.w_uv, o2, n_branch=4,
                        alpha_q=wl.alpha_q, alpha_kv=wl.alpha_kv, branch_scale=wl.sigma_o,
                        softmax_scale=wl.softmax_scale, rope_theta=wl.rope_theta, seq_stride=dev.seq_stride,
                        q_positions=pos)
    ws = hra.alloc_workspace(p)
    hra.mlra_decode(p)
    hra.check_device_status(p)
    assert torch.equal(o2, ref)
    del ws
