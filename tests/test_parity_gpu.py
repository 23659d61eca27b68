"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the same
seeded inputs.  Small cases are compared element by element over every output; the five
full-size workloads are compared on sampled (sequence, head) outputs in the launch
configuration the benchmark uses (num_splits = 0: one split per 4 SMs, one CTA per SM)."""
import numpy as np
import pytest
import torch

import head_rank_attention_b200 as hra
import oracle
import synth
from gpu_cases import assert_parity, run_gpu

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    torch.backends.cuda.matmul.allow_tf32 = False


def _case(name, n_branch, lengths, heads=128, page_size=0, **kw):
    return synth.Workload(name, n_branch, len(lengths), heads, max(lengths), page_size=page_size,
                          lengths=tuple(lengths), **kw)


TAILS = (1, 31, 32, 33, 127, 128, 129, 1000)

SMALL = [
    _case("tails_mlra4", 4, TAILS),
    _case("tails_mlra2", 2, TAILS),
    _case("tails_mla", 1, TAILS),
    _case("paged64_mlra4", 4, (5, 64, 65, 700), page_size=64),
    _case("paged32_mlra2", 2, (5, 64, 65, 700), page_size=32),
    _case("paged128_mla", 1, (5, 64, 65, 700), page_size=128),
    _case("h1_mlra4", 4, (77, 300), heads=1),
    _case("h16_mlra4", 4, (2048,), heads=16, alpha_q=2048 ** 0.5 / 1536 ** 0.5, alpha_kv=2.0, branch_scale=0.5),
    _case("h100_mla", 1, (513, 9), heads=100),
    _case("stress_mlra4", 4, (3000, 17), alpha_q=synth.A_Q_V3, alpha_kv=synth.A_KV_V3),
    _case("stress_mla", 1, (3000, 17), alpha_q=synth.A_Q_V3, alpha_kv=synth.A_KV_V3),
    _case("outlier_mlra4", 4, (5000,), outlier_frac=0.01),
    # the tile boundaries of the 48-token MLA and 80-token MLRA-2 kernels (16-row TMA boxes)
    _case("tails48_mla", 1, (47, 48, 49, 95, 96, 97)),
    _case("paged32_tails48_mla", 1, (47, 49, 97, 200), page_size=32),
    _case("tails80_mlra2", 2, (79, 80, 81, 159, 160, 161)),
    _case("paged64_tails80_mlra2", 2, (79, 81, 161, 300), page_size=64),
]


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_small_full_parity(wl):
    inp = synth.make_inputs(wl)
    dev = synth.to_device(inp)
    out, _, _ = run_gpu(dev, wl)
    ref = oracle.decode_batch(inp, wl, form="absorbed")
    assert_parity(out.cpu().numpy(), ref, wl.name)


@pytest.mark.parametrize("num_splits", [1, 3, 37, 200])
def test_split_count_invariance(num_splits):
    """Any partition of the token stream across splits gives the same result (LSE combine)."""
    wl = _case("splits", 4, (1, 130, 2000, 64))
    inp = synth.make_inputs(wl)
    dev = synth.to_device(inp)
    ref = oracle.decode_batch(inp, wl, form="absorbed")
    out, _, _ = run_gpu(dev, wl, num_splits=num_splits)
    assert_parity(out.cpu().numpy(), ref, f"splits={num_splits}")


def test_many_sequences():
    """B=300 short sequences: many sequences per split, prefix scan over > 32 lengths."""
    rng = np.random.default_rng(5)
    wl = _case("many", 4, tuple(int(x) for x in rng.integers(1, 200, size=300)), heads=8)
    inp = synth.make_inputs(wl)
    out, _, _ = run_gpu(synth.to_device(inp), wl)
    assert_parity(out.cpu().numpy(), oracle.decode_batch(inp, wl, form="absorbed"), "many")


@pytest.mark.parametrize("n_branch", [4, 2, 1])
def test_maximum_batch(n_branch):
    """B = 1024 (the largest batch the library takes), mixed lengths including zeros,
    8 heads: every sequence-indexed table at its largest, absorb and up-projection over
    8 chunks of 128 sequences."""
    rng = np.random.default_rng(11)
    lens = rng.integers(0, 300, size=1024)
    lens[rng.integers(0, 1024, size=20)] = 0
    wl = _case(f"maxbatch_{n_branch}", n_branch, tuple(int(x) for x in lens), heads=8)
    inp = synth.make_inputs(wl)
    out, _, _ = run_gpu(synth.to_device(inp), wl)
    got = out.cpu().numpy()
    zero = lens == 0
    assert np.all(got[zero] == 0)
    ref = oracle.decode_batch(inp, wl, seqs=[int(s) for s in np.flatnonzero(~zero)], form="absorbed")
    assert_parity(got[~zero], ref, wl.name)


def test_bf16_output():
    wl = _case("bf16out", 4, (700, 33))
    inp = synth.make_inputs(wl)
    out, _, _ = run_gpu(synth.to_device(inp), wl, out_dtype=torch.bfloat16)
    assert_parity(out.float().cpu().numpy(), oracle.decode_batch(inp, wl, form="absorbed"), "bf16 out")


def test_paged_equals_contiguous_bitwise():
    """Same logical cache, paged (random page table) or contiguous: identical bits."""
    lens = (100, 640, 33)
    wl_c = _case("layout", 4, lens)
    wl_p = _case("layout", 4, lens, page_size=32)
    out_c, _, _ = run_gpu(synth.to_device(synth.make_inputs(wl_c)), wl_c)
    out_p, _, _ = run_gpu(synth.to_device(synth.make_inputs(wl_p)), wl_p)
    assert torch.equal(out_c, out_p)


def test_mla_entry_point_and_determinism():
    wl = _case("mla_api", 1, (900, 5))
    dev = synth.to_device(synth.make_inputs(wl))
    a, _, _ = run_gpu(dev, wl, api="mla")
    b, _, _ = run_gpu(dev, wl, api="mlra")
    c, _, _ = run_gpu(dev, wl, api="mlra")
    assert torch.equal(a, b) and torch.equal(b, c)


def test_mlra4_differs_from_mla_on_gpu():
    """Guards against a kernel that sums branch keys before the softmax."""
    lens = (1500,)
    wl4 = _case("neg", 4, lens, branch_scale=1.0)
    wl1 = _case("neg", 1, lens)
    inp = synth.make_inputs(wl4)
    dev = synth.to_device(inp)
    o4, _, _ = run_gpu(dev, wl4)
    o1, _, _ = run_gpu(dev, wl1)
    assert (o4 - o1).abs().max() > 0.1 * o1.abs().max()


def test_zero_length_sequence_gives_zero_row():
    wl = _case("zero", 4, (0, 50))
    inp = synth.make_inputs(wl)
    out, _, _ = run_gpu(synth.to_device(inp), wl)
    assert torch.all(out[0] == 0)
    ref = oracle.decode_batch(inp, wl, seqs=[1], form="absorbed")
    assert_parity(out[1:].cpu().numpy(), ref, "zero-length neighbour")


@pytest.mark.parametrize("n_branch,page_size", [(4, 0), (4, 64), (2, 0), (2, 32), (1, 0), (1, 128)])
def test_cache_rows_past_sequence_end_are_never_used(n_branch, page_size):
    """Every physical cache row that holds no token of any sequence (the tail of a
    sequence's stride or of its last page, unused pages) is NaN: the output must not
    change, since tokens past L do not exist."""
    wl = _case(f"nan_tail_{n_branch}_{page_size}", n_branch, (1, 31, 33, 127, 129, 300), page_size=page_size)
    inp = synth.make_inputs(wl)
    used = torch.zeros(inp.cache.shape[0], dtype=torch.bool)
    for s in range(wl.batch):
        L = int(inp.seq_lens[s])
        idx = torch.arange(L)
        if inp.block_table is None:
            used[s * inp.seq_stride + idx] = True
        else:
            used[inp.block_table[s, idx // page_size].to(torch.int64) * page_size + idx % page_size] = True
    assert not used.all()
    inp.cache[~used] = float("nan")
    out, _, _ = run_gpu(synth.to_device(inp), wl)
    assert_parity(out.cpu().numpy(), oracle.decode_batch(inp, wl, form="absorbed"), wl.name)


def test_back_to_back_calls_sharing_a_workspace():
    """Calls queued back to back on one stream, sharing one workspace, with different
    inputs: each call's kernels may start while the previous call drains, so any write
    of the workspace before the previous call is done with it would change an output."""
    wl_a = _case("b2b_a", 4, (3000, 17, 900))
    wl_b = _case("b2b_b", 4, (40, 2500, 700), seed=7)
    dev_a, dev_b = synth.to_device(synth.make_inputs(wl_a)), synth.to_device(synth.make_inputs(wl_b))
    ref_a, p_a, ws = run_gpu(dev_a, wl_a)
    ref_b, p_b, _ = run_gpu(dev_b, wl_b, workspace=ws)
    outs = []
    for k in range(6):
        dev, wl, p = (dev_a, wl_a, p_a) if k % 2 == 0 else (dev_b, wl_b, p_b)
        out = torch.empty_like(ref_a)
        p.out = out.data_ptr()
        hra.mlra_decode(p)
        outs.append(out)
    torch.cuda.synchronize()
    hra.check_device_status(p_a)
    for k, out in enumerate(outs):
        assert torch.equal(out, ref_a if k % 2 == 0 else ref_b), f"call {k}"


@pytest.mark.parametrize("n_branch", [4, 1])
def test_cuda_graph_replay_matches_direct_call(n_branch):
    """A call captured into a CUDA graph (kernels chained programmatically inside it)
    and replayed gives the bits of a direct call."""
    wl = _case(f"graph_{n_branch}", n_branch, (1500, 40))
    dev = synth.to_device(synth.make_inputs(wl))
    ref, p, ws = run_gpu(dev, wl)
    out = torch.zeros_like(ref)
    p.out = out.data_ptr()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        hra.mlra_decode(p, torch.cuda.current_stream())
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    hra.check_device_status(p)


def test_bounded_wait_reports_timeout_and_context_survives():
    """A wait that nothing satisfies ends with HRA_ERR_DEVICE_TIMEOUT; the next call works."""
    wl = _case("timeout", 4, (200,))
    inp = synth.make_inputs(wl)
    dev = synth.to_device(inp)
    out, p, ws = run_gpu(dev, wl)
    hra.selftest_wait_timeout(ws, limit_us=2000)
    with pytest.raises(hra.HraError) as e:
        hra.check_device_status(p)
    assert e.value.status == hra._binding.HRA_ERR_DEVICE_TIMEOUT
    out2, _, _ = run_gpu(dev, wl, workspace=ws)
    assert torch.equal(out, out2)


# ---- the five workloads at full size -------------------------------------------------------

_FULL_CACHE = {}


def _full_inputs(wl):
    key = (wl.batch, wl.heads, wl.seq_len, wl.seq_len_min, wl.page_size, wl.outlier_frac, wl.n_branch)
    if key not in _FULL_CACHE:
        _FULL_CACHE.clear()
        torch.cuda.empty_cache()
        inp = synth.make_inputs(wl)
        _FULL_CACHE[key] = (inp, synth.to_device(inp))
    return _FULL_CACHE[key]


FULL = [
    ("small_mlra4_h16_t2k", None, None),           # every output, expanded definition
    ("mla_b32_t8k", [0, 13, 31], None),
    ("paged_b64_t32k_mlra4", [0, 37, 63], list(range(0, 128, 8))),
    ("paged_b64_t32k_mlra2", [0, 37, 63], list(range(0, 128, 8))),
    ("paged_b64_t32k_mla", [0, 37, 63], list(range(0, 128, 8))),
    ("long_mlra4_b4_t64k_128k", None, list(range(0, 128, 8))),
    ("vlong_mlra4_b1_t2m", None, list(range(0, 128, 16))),
]


@pytest.mark.parametrize("name,seqs,heads", FULL, ids=[f[0] for f in FULL])
def test_full_size_workload(name, seqs, heads):
    wl = synth.WORKLOADS[name]
    inp, dev = _full_inputs(wl)
    out, _, _ = run_gpu(dev, wl)
    got = out.cpu().numpy()
    assert np.isfinite(got).all()
    seqs = list(range(wl.batch)) if seqs is None else seqs
    heads_idx = list(range(wl.heads)) if heads is None else heads
    form = "expanded" if name == "small_mlra4_h16_t2k" else "absorbed"
    ref = oracle.decode_batch(inp, wl, heads=heads_idx, seqs=seqs, form=form)
    assert_parity(got[np.ix_(seqs, heads_idx)], ref, name)
