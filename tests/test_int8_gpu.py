"""GPU parity for the int8 latent cache (hra.h: cache_dtype = HRA_INT8): the CUDA path
through the C ABI against the oracle on the dequantised cache (oracle.decode_batch_int8),
on int8 bytes and scales written by synth.quantize_int8_blocks from the seeded bf16
cache.  The parity bar is the one for the bf16 cache."""
import numpy as np
import pytest
import torch

import head_rank_attention_b200 as hra
import oracle
import synth
from gpu_cases import assert_parity

pytestmark = pytest.mark.gpu


def _case(name, lengths, heads=128, page_size=0, **kw):
    return synth.Workload(name, 4, len(lengths), heads, max(lengths), page_size=page_size, lengths=tuple(lengths),
                          **kw)


def _run(inp, wl, q8, scale, *, d_c=512, n_branch=4, ckv=None, krope=None, w_uk=None, w_uv=None, num_splits=0,
         nan_unused=False):
    dev = synth.to_device(inp)
    ckv = q8.cuda() if ckv is None else ckv
    krope = dev.cache[:, 512:] if krope is None else krope
    if nan_unused:  # rows no sequence owns: their rope part is NaN (their int8 part is whatever it is)
        used = torch.zeros(krope.shape[0], dtype=torch.bool)
        for s in range(wl.batch):
            L = int(inp.seq_lens[s])
            if inp.block_table is None:
                used[s * inp.seq_stride:s * inp.seq_stride + L] = True
            else:
                t = torch.arange(L)
                used[inp.block_table[s, t // wl.page_size].long() * wl.page_size + t % wl.page_size] = True
        krope = krope.clone()
        krope[~used.cuda()] = float("nan")
    out = torch.empty(wl.batch, wl.heads, synth.D_V, dtype=torch.float32, device="cuda")
    p = hra.make_params(dev.q, ckv, krope, dev.seq_lens, dev.w_uk if w_uk is None else w_uk,
                        dev.w_uv if w_uv is None else w_uv, out, n_branch=n_branch, alpha_q=wl.alpha_q,
                        alpha_kv=wl.alpha_kv, branch_scale=wl.sigma_o, softmax_scale=wl.softmax_scale,
                        rope_theta=wl.rope_theta, block_table=dev.block_table, page_size=wl.page_size,
                        seq_stride=dev.seq_stride, num_splits=num_splits, ckv_scale=scale)
    ws = hra.alloc_workspace(p)
    ws.fill_(0xFF)
    hra.mlra_decode(p)
    hra.check_device_status(p)
    return out.cpu().numpy()


CASES = [
    _case("i8_tails", (1, 31, 32, 33, 127, 128, 129, 1000)),
    _case("i8_paged64", (5, 64, 65, 700), page_size=64),
    _case("i8_paged32", (5, 64, 65, 700), page_size=32),
    _case("i8_h16", (2048,), heads=16, alpha_q=2048 ** 0.5 / 1536 ** 0.5, alpha_kv=2.0, branch_scale=0.5),
    _case("i8_stress", (3000, 17), alpha_q=synth.A_Q_V3, alpha_kv=synth.A_KV_V3),
    _case("i8_outliers", (5000,), outlier_frac=0.01),
]


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_int8_cache_matches_the_oracle(wl):
    inp = synth.make_inputs(wl)
    q8, scale = synth.quantize_int8_blocks(inp.cache[:, :512])
    got = _run(inp, wl, q8, scale.cuda(), nan_unused=True)
    ref = oracle.decode_batch_int8(inp, wl, q8.numpy(), scale.numpy())
    assert_parity(got, ref, wl.name)


@pytest.mark.parametrize("num_splits", [1, 200])
def test_int8_split_counts(num_splits):
    wl = _case("i8_splits", (1, 130, 2000, 64))
    inp = synth.make_inputs(wl)
    q8, scale = synth.quantize_int8_blocks(inp.cache[:, :512])
    got = _run(inp, wl, q8, scale.cuda(), num_splits=num_splits)
    assert_parity(got, oracle.decode_batch_int8(inp, wl, q8.numpy(), scale.numpy()), f"splits={num_splits}")


def test_int8_branch_shards_sum_to_mlra4():
    """4-way tensor parallelism over an int8 cache: rank r holds its 128 int8 columns, its
    column of scales (a strided view) and K_RoPE; the four outputs sum to MLRA-4."""
    from head_rank_attention_b200 import tp
    wl = _case("i8_shards", (1, 129, 1000), page_size=64)
    inp = synth.make_inputs(wl)
    dev = synth.to_device(inp)
    q8, scale = synth.quantize_int8_blocks(inp.cache[:, :512])
    q8d, sd = q8.cuda(), scale.cuda()
    krope = dev.cache[:, 512:].contiguous()
    total = 0
    for r in range(4):
        w_uk, w_uv = tp.shard_weights(dev.w_uk, dev.w_uv, r, 4)
        total = total + _run(inp, wl, q8, sd[:, r:r + 1], d_c=128, n_branch=1, ckv=q8d[:, 128 * r:128 * (r + 1)].contiguous(),
                             krope=krope, w_uk=w_uk, w_uv=w_uv)
    assert_parity(total, oracle.decode_batch_int8(inp, wl, q8.numpy(), scale.numpy()), "int8 shards")


def test_int8_cache_stays_close_to_the_bf16_decode():
    """Quantisation moves the output only a little: the int8 decode against the bf16 oracle
    (not a parity bar, a sanity bound on the format)."""
    wl = _case("i8_vs_bf16", (4000, 300))
    inp = synth.make_inputs(wl)
    q8, scale = synth.quantize_int8_blocks(inp.cache[:, :512])
    got = _run(inp, wl, q8, scale.cuda())
    ref = oracle.decode_batch(inp, wl)
    assert np.abs(got - ref).sum() / np.abs(ref).sum() < 3e-2
