"""GPU parity of the split merge and up-projection for small batches.

Batches of up to four sequences whose (head, latent slice) grid fits on the SMs at once,
with up to 64 split groups, take one fused merge + up-projection kernel (a cluster of the
latent slices of one head); the others take the merge kernel and the tensor-core
up-projection.  Both are checked against the fp64 oracle on either side of the boundary
(batch 4 / 5; 32 / 128 heads; 37 / 100 groups), with every output
mode (fp32, bf16, accumulate into a buffer), empty sequences, many splits per sequence and
the latent widths of branch shards."""
import numpy as np
import pytest
import torch

import head_rank_attention_b200 as hra
import oracle
import synth
from gpu_cases import assert_parity, run_gpu

pytestmark = pytest.mark.gpu

LENGTHS = (2000, 1, 0, 700, 129)  # the first B of these


def _wl(B, n_branch=4, heads=32, lengths=LENGTHS, **kw):
    lens = tuple(lengths[:B])
    return synth.Workload(f"combine_b{B}_nb{n_branch}", n_branch, B, heads, max(max(lens), 1), lengths=lens, **kw)


@pytest.mark.parametrize("B,heads,splits", [(1, 32, 37), (2, 32, 37), (3, 32, 37), (4, 32, 37), (5, 32, 37),
                                             (4, 32, 100), (4, 128, 37), (1, 16, 64)])
@pytest.mark.parametrize("n_branch", [4, 1])
def test_small_and_large_batch_paths(B, heads, splits, n_branch):
    wl = _wl(B, n_branch, heads)
    inp = synth.make_inputs(wl)
    out, _, _ = run_gpu(synth.to_device(inp), wl, num_splits=splits)
    got = out.cpu().numpy()
    live = [s for s in range(B) if wl.lengths[s] > 0]
    for s in range(B):
        if wl.lengths[s] == 0:
            assert np.all(got[s] == 0), f"B={B}: empty sequence {s} is not zero"
    assert_parity(got[live], oracle.decode_batch(inp, wl, seqs=live, form="absorbed"), f"B={B}")


@pytest.mark.parametrize("num_splits", [1, 64, 200])
def test_small_batch_any_split_count(num_splits):
    """1 and 64 splits (the fused kernel; 64 groups over four sequences take two load
    rounds per thread set) and 200 (the merge kernel)."""
    wl = _wl(4, lengths=(6000, 130, 2, 4000))
    inp = synth.make_inputs(wl)
    out, _, _ = run_gpu(synth.to_device(inp), wl, num_splits=num_splits)
    assert_parity(out.cpu().numpy(), oracle.decode_batch(inp, wl, form="absorbed"), f"splits={num_splits}")


def test_small_batch_bf16_output():
    wl = _wl(3, heads=16)
    inp = synth.make_inputs(wl)
    out, _, _ = run_gpu(synth.to_device(inp), wl, out_dtype=torch.bfloat16, num_splits=37)
    got = out.float().cpu().numpy()
    assert np.all(got[2] == 0)
    assert_parity(got[:2], oracle.decode_batch(inp, wl, seqs=[0, 1], form="absorbed"), "bf16 out")


def test_small_batch_accumulates_into_out():
    """out_accumulate adds this call's output into what the buffer holds."""
    wl = _wl(2, lengths=(900, 33))
    inp = synth.make_inputs(wl)
    dev = synth.to_device(inp)
    base = torch.randn(wl.batch, wl.heads, synth.D_V, dtype=torch.float32, device="cuda")
    out = base.clone()
    p = hra.make_params(dev.q, dev.ckv, dev.krope, dev.seq_lens, dev.w_uk, dev.w_uv, out, n_branch=wl.n_branch,
                        alpha_q=wl.alpha_q, alpha_kv=wl.alpha_kv, branch_scale=wl.sigma_o,
                        softmax_scale=wl.softmax_scale, rope_theta=wl.rope_theta, seq_stride=dev.seq_stride,
                        out_accumulate=True, num_splits=37)
    ws = hra.alloc_workspace(p)
    hra.mlra_decode(p)
    hra.check_device_status(p)
    got = (out - base).cpu().numpy()
    assert_parity(got, oracle.decode_batch(inp, wl, form="absorbed"), "accumulated")
    del ws


@pytest.mark.parametrize("world", [4, 2])
def test_small_batch_branch_shards(world):
    """The shards of 4- and 2-way tensor parallelism (latent width 128 or 256: clusters of
    1 or 2 slices; 37 splits), each into its own out: their sum is MLRA-4."""
    from head_rank_attention_b200 import tp
    wl = _wl(3, lengths=(1500, 64, 300))
    inp = synth.make_inputs(wl)
    dev = synth.to_device(inp)
    total = np.zeros((wl.batch, wl.heads, synth.D_V))
    for r in range(world):
        local = tp.shard_cache(dev.cache, r, world)
        w_uk, w_uv = tp.shard_weights(dev.w_uk, dev.w_uv, r, world)
        d = local.shape[1] - synth.D_ROPE
        out = torch.empty(wl.batch, wl.heads, synth.D_V, dtype=torch.float32, device="cuda")
        p = hra.make_params(dev.q, local[:, :d], local[:, d:], dev.seq_lens, w_uk, w_uv, out,
                            n_branch=4 // world, alpha_q=wl.alpha_q, alpha_kv=wl.alpha_kv, branch_scale=wl.sigma_o,
                            softmax_scale=wl.softmax_scale, rope_theta=wl.rope_theta, seq_stride=dev.seq_stride,
                            num_splits=37)
        ws = hra.alloc_workspace(p)
        ws.fill_(0xFF)
        hra.mlra_decode(p)
        hra.check_device_status(p)
        total += out.cpu().numpy()
        del ws
    assert_parity(total, oracle.decode_batch(inp, wl, form="absorbed"), f"{world}-way shards summed")
