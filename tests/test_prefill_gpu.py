"""GPU parity of the prefill (causal multi-token, expanded form) path through the C ABI
(mlra_prefill) against the pinned fp64 oracle mlra_prefill_expanded, on seeded synth
inputs: ragged query counts, n = L, n = 1 (which must equal the decode), every branch
width, more than one tile of queries, the stress scales and a bf16 output."""
import numpy as np
import pytest
import torch

import head_rank_attention_b200 as hra
import oracle
import synth
from gpu_cases import assert_parity, run_gpu

pytestmark = pytest.mark.gpu


def _case(L, n, nb, h, **kw):
    wl = synth.Workload(f"prefill_L{L}_n{n}_b{nb}_h{h}", nb, 1, h, L, **kw)
    inp = synth.make_inputs(wl)
    q = synth.queries(synth.Workload(wl.name + "_q", nb, n, h, L, seed=7))  # [n, h, 192]
    return wl, inp, q


def _run(wl, inp, q, out_dtype=torch.float32):
    dev = synth.to_device(inp)
    L = int(inp.seq_lens[0])
    cache = dev.cache[:L]
    qd = q.cuda()
    out = torch.empty(q.shape[0], wl.heads, synth.D_V, dtype=out_dtype, device="cuda")
    p = hra.make_prefill_params(qd, cache[:, :512], cache[:, 512:], dev.w_uk, dev.w_uv, out, n_branch=wl.n_branch,
                                alpha_q=wl.alpha_q, alpha_kv=wl.alpha_kv, branch_scale=wl.sigma_o,
                                softmax_scale=wl.softmax_scale, rope_theta=wl.rope_theta)
    ws = hra.alloc_prefill_workspace(p)
    ws.fill_(0xFF)  # NaN bytes everywhere: a slot the call reads before writing shows up
    hra.mlra_prefill(p)
    hra.check_prefill_status(p)
    return out.float().cpu().numpy()


def _oracle(wl, inp, q):
    L = int(inp.seq_lens[0])
    rows = inp.cache[:L]
    return oracle.mlra_prefill_expanded(q, rows[:, :512], rows[:, 512:], inp.w_uk, inp.w_uv, wl.n_branch,
                                        alpha_q=wl.alpha_q, alpha_kv=wl.alpha_kv, branch_scale=wl.sigma_o,
                                        softmax_scale=wl.softmax_scale, rope_theta=wl.rope_theta)


CASES = [
    (300, 300, 4, 8, {}),                 # n = L, three query tiles (128, 128, 44)
    (1000, 37, 4, 16, {}),                # ragged: a few queries at the end of a long context
    (513, 130, 1, 4, {}),                 # MLA (512-wide branch), two query tiles
    (700, 200, 2, 8, {}),                 # MLRA-2
    (2000, 64, 4, 8, dict(alpha_q=synth.A_Q_V3, alpha_kv=synth.A_KV_V3)),  # stress scales
    (1024, 256, 4, 128, {}),              # every head
]


@pytest.mark.parametrize("L,n,nb,h,kw", CASES, ids=lambda x: str(x))
def test_prefill_matches_the_oracle(L, n, nb, h, kw):
    wl, inp, q = _case(L, n, nb, h, **kw)
    assert_parity(_run(wl, inp, q), _oracle(wl, inp, q), wl.name)


def test_prefill_bf16_output():
    wl, inp, q = _case(400, 90, 4, 8)
    assert_parity(_run(wl, inp, q, out_dtype=torch.bfloat16), _oracle(wl, inp, q), "bf16 out")


@pytest.mark.parametrize("nb", [4, 1])
def test_one_query_prefill_is_the_decode(nb):
    """n = 1: the last token attending to the whole sequence is one decode step."""
    wl, inp, q = _case(129, 1, nb, 128)
    got = _run(wl, inp, q)
    # the same query through the decode path
    dwl = synth.Workload(wl.name + "_d", nb, 1, 128, 129)
    dinp = synth.Inputs(q=q, cache=inp.cache, seq_lens=inp.seq_lens, block_table=None, seq_stride=inp.seq_stride,
                        w_uk=inp.w_uk, w_uv=inp.w_uv)
    dec, _, _ = run_gpu(synth.to_device(dinp), dwl)
    ref = oracle.decode_batch(dinp, dwl)
    assert_parity(got, ref, "prefill n=1 vs decode oracle")
    assert_parity(got, dec.cpu().numpy().astype(np.float64), "prefill n=1 vs decode kernel")
