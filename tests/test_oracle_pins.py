"""Pins for the fp64 oracle: each test ties it to something other than itself.

The pages print no worked numeric example, so the pins are the identities they state,
closed forms of the definition, a library attention routine on the expanded per-branch
keys/values, and brute force on tiny inputs.  Each test names the mistake it catches.
"""
import json
import math
import pathlib

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = pathlib.Path(__file__).parent / "golden"


def _rand_case(rng, h=3, L=11, d_c=512, d_rope=64, d_nope=128, d_v=128, n_branch=4, bf16=True):
    w = d_c // n_branch
    q = rng.standard_normal((h, d_nope + d_rope))
    c = rng.standard_normal((L, d_c))
    kr = rng.standard_normal((L, d_rope))
    wuk = rng.standard_normal((h, d_c, d_nope)) / math.sqrt(w)
    wuv = rng.standard_normal((h, d_c, d_v)) / math.sqrt(w)
    if bf16:  # the path consumes bf16 values; use such values in the pins too
        q, c, kr, wuk, wuv = (torch.from_numpy(x).to(torch.bfloat16) for x in (q, c, kr, wuk, wuv))
    return q, c, kr, wuk, wuv


def _rel(a, b):
    return np.abs(a - b).max() / np.abs(b).max()


# --- identities the pages state -------------------------------------------------------

@pytest.mark.parametrize("n_branch", [1, 2, 4])
def test_absorbed_equals_expanded(n_branch):
    """QK^T = C_q W_q W_k^T C_kv^T ("ML Revisit: Attention", MLA) and the three decode
    steps of "Multi-Head Low-Rank Attention" (方法步骤详情) reproduce the expanded form.
    Catches: a dropped/misplaced alpha, wrong W_UK/W_UV slicing, transposed weights."""
    rng = np.random.default_rng(10 + n_branch)
    case = _rand_case(rng, h=4, L=37, n_branch=n_branch)
    kw = dict(alpha_q=1.3, alpha_kv=0.7, rope_theta=10000.0)
    a = oracle.mlra_decode_absorbed(*case, n_branch, **kw)
    e = oracle.mlra_decode_expanded(*case, n_branch, **kw)
    assert _rel(a, e) < 1e-12


def test_absorbed_chunking_is_exact():
    """The absorbed form's token chunking only bounds memory. Catches: a chunk-boundary
    bug (dropped or double-counted tokens)."""
    rng = np.random.default_rng(3)
    case = _rand_case(rng, h=2, L=301)
    a = oracle.mlra_decode_absorbed(*case, 4, token_chunk=64)
    b = oracle.mlra_decode_absorbed(*case, 4, token_chunk=1 << 20)
    assert _rel(a, b) < 1e-13


def test_mlra_one_branch_is_mla():
    """MLRA with a single block is MLA ("Multi-Head Low-Rank Attention", 核心方法);
    mla_decode is written from the MLA pages alone. Catches: branch-sum scale not 1 at
    B=1, a branch loop that drops the rope key."""
    rng = np.random.default_rng(4)
    case = _rand_case(rng, h=3, L=29, n_branch=1)
    for kw in (dict(), dict(alpha_q=2.16, alpha_kv=3.74)):
        m = oracle.mla_decode(*case, **kw)
        assert _rel(oracle.mlra_decode_expanded(*case, 1, **kw), m) < 1e-12
        assert _rel(oracle.mlra_decode_absorbed(*case, 1, **kw), m) < 1e-12


@pytest.mark.parametrize("blocks", [2, 4])
def test_mla_key_is_sum_of_block_keys(blocks):
    """K_NoPE^(i) = sum_b C_KV^(b) W_UK^(b),(i) ("Multi-Head Low-Rank Attention", 研究动机).
    Catches: blocks cut along the wrong axis of W_UK."""
    rng = np.random.default_rng(5)
    c = rng.standard_normal((13, 512))
    w = rng.standard_normal((512, 128))
    assert _rel(oracle.mlra_nope_key_blocks(c, w, blocks), oracle.mla_nope_key(c, w)) < 1e-12


def test_mlra4_is_not_mla():
    """MLRA's sum of branch softmaxes differs from MLA's softmax of the summed key
    ("Multi-Head Low-Rank Attention", 核心方法: not equivalent). Catches: summing the
    branch keys before the softmax."""
    rng = np.random.default_rng(6)
    case = _rand_case(rng, h=3, L=64, n_branch=4)
    mlra = oracle.mlra_decode_expanded(*case, 4, branch_scale=1.0)
    mla = oracle.mla_decode(*case)
    assert _rel(mlra, mla) > 0.1


@pytest.mark.parametrize("n_groups", [2, 4])
def test_gla_is_mlra_with_the_other_groups_weights_zeroed(n_groups):
    """GLA (head groups, each on its own latent group; "Multi-Head Low-Rank Attention",
    研究动机) equals MLRA with branch = group, branch-sum scale 1, when each head's W_UK and
    W_UV rows outside its group are zero: the other branches then have value 0.
    Catches: heads assigned to the wrong group, the group's latent columns off by a block,
    a dropped rope key."""
    rng = np.random.default_rng(11)
    h, L, d_c = 4, 23, 512
    w = d_c // n_groups
    q, c, kr, _, _ = _rand_case(rng, h=h, L=L, n_branch=n_groups)
    wuk_g = rng.standard_normal((h, w, 128)) / math.sqrt(w)
    wuv_g = rng.standard_normal((h, w, 128)) / math.sqrt(w)
    wuk, wuv = np.zeros((h, d_c, 128)), np.zeros((h, d_c, 128))
    for i in range(h):
        g = i // (h // n_groups)
        wuk[i, g * w:(g + 1) * w], wuv[i, g * w:(g + 1) * w] = wuk_g[i], wuv_g[i]
    for kw in (dict(), dict(alpha_q=2.16, alpha_kv=3.74)):
        gla = oracle.gla_decode(q, c, kr, wuk_g, wuv_g, n_groups, **kw)
        mlra = oracle.mlra_decode_expanded(q, c, kr, wuk, wuv, n_groups, branch_scale=1.0, **kw)
        assert _rel(gla, mlra) < 1e-12


def test_gla_head_reads_only_its_group():
    """A GLA-2 head's output does not change when the other group's latent columns do."""
    rng = np.random.default_rng(12)
    q, c, kr, _, _ = _rand_case(rng, h=4, L=17, n_branch=2, bf16=False)
    wuk = rng.standard_normal((4, 256, 128)) / 16
    wuv = rng.standard_normal((4, 256, 128)) / 16
    base = oracle.gla_decode(q, c, kr, wuk, wuv, 2)
    c2 = c.copy()
    c2[:, 256:] += rng.standard_normal((17, 256))
    moved = oracle.gla_decode(q, c2, kr, wuk, wuv, 2)
    assert np.array_equal(moved[:2], base[:2])
    assert _rel(moved[2:], base[2:]) > 1e-3


# --- the causal multi-token (prefill) form ---------------------------------------------------

@pytest.mark.parametrize("n_branch", [1, 4])
def test_prefill_rows_are_decodes_of_the_prefix(n_branch):
    """Query j of a prefill over the last n tokens sees exactly the first p_j + 1 tokens at
    position p_j: it equals the (pinned) decode oracle on that prefix ("vllbc02MLA":
    prefill and generation compute the same attention).  Catches: a mask off by one, the
    rope position of the wrong token, branch scales applied per query."""
    rng = np.random.default_rng(21)
    h, L, n = 3, 19, 5
    _, c, kr, wuk, wuv = _rand_case(rng, h=h, L=L, n_branch=n_branch)
    q = torch.from_numpy(rng.standard_normal((n, h, 192))).to(torch.bfloat16)
    kw = dict(alpha_q=1.3, alpha_kv=0.7)
    pre = oracle.mlra_prefill_expanded(q, c, kr, wuk, wuv, n_branch, **kw)
    for j in range(n):
        m = L - n + j + 1
        ref = oracle.mlra_decode_absorbed(q[j], c[:m], kr[:m], wuk, wuv, n_branch, **kw)
        assert _rel(pre[j], ref) < 1e-12


def test_prefill_is_causal_and_matches_library_causal_attention():
    """Changing tokens after a query's position leaves its row unchanged, and one branch
    of one head equals torch's scaled_dot_product_attention with a causal (bottom-right)
    mask on the expanded keys and values (library routine, fp64)."""
    rng = np.random.default_rng(22)
    h, L, n = 2, 13, 4
    _, c, kr, wuk, wuv = _rand_case(rng, h=h, L=L, n_branch=1, bf16=False)
    q = rng.standard_normal((n, h, 192))
    pre = oracle.mlra_prefill_expanded(q, c, kr, wuk, wuv, 1)
    c2 = c.copy()
    c2[L - 2:] += 1.0  # only the last two tokens change: rows of queries before them stay
    pre2 = oracle.mlra_prefill_expanded(q, c2, kr, wuk, wuv, 1)
    assert np.array_equal(pre2[:n - 2], pre[:n - 2])
    assert _rel(pre2[n - 1], pre[n - 1]) > 1e-6
    i = 1
    K = np.concatenate([c @ wuk[i], kr], axis=1)
    V = c @ wuv[i]
    pos = np.arange(L - n, L)
    Q = np.stack([np.concatenate([q[j, i, :128], oracle.rope_rotate(q[j, i, 128:], int(pos[j]))]) for j in range(n)])
    mask = torch.from_numpy(np.arange(L)[None, :] <= pos[:, None])
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q)[None], torch.from_numpy(K)[None], torch.from_numpy(V)[None], attn_mask=mask[None],
        scale=1 / math.sqrt(192))[0].numpy()
    assert _rel(pre[:, i], ref) < 1e-12


# --- RoPE --------------------------------------------------------------------------------

def test_rope_relative_position():
    """q.k scores under RoPE depend only on the offset m - n ("Multi-Head Low-Rank
    Attention", 前置知识 RoPE), up to positions of 2^21."""
    rng = np.random.default_rng(7)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    for m, n in [(5, 3), (2097151, 17), (1000003, 999999)]:
        base = oracle.rope_rotate(q, m) @ oracle.rope_rotate(k, n)
        for delta in (1, 4096, 2 ** 20):
            s = oracle.rope_rotate(q, m + delta) @ oracle.rope_rotate(k, n + delta)
            assert abs(s - base) <= 1e-9 * (1 + abs(base))
        direct = oracle.rope_rotate(q, m - n) @ k
        assert abs(direct - base) <= 1e-9 * (1 + abs(base))


def test_rope_is_complex_rotation():
    """Each pair (x_j, x_{j+32}) seen as x_j + i x_{j+32} is multiplied by
    exp(i pos theta^(-2j/64)) (textbook complex form, numpy complex exp). Catches: a
    wrong sign, adjacent-pair instead of half pairing, wrong frequency exponent."""
    rng = np.random.default_rng(8)
    x = rng.standard_normal(64)
    pos = 123457
    z = (x[:32] + 1j * x[32:]) * np.exp(1j * pos * 10000.0 ** (-np.arange(32) / 32.0))
    r = oracle.rope_rotate(x, pos)
    np.testing.assert_allclose(r[:32], z.real, atol=1e-9)
    np.testing.assert_allclose(r[32:], z.imag, atol=1e-9)
    # theta_0 = 1: the first pair turns by exactly pos radians
    assert abs(r[0] - (x[0] * math.cos(pos) - x[32] * math.sin(pos))) < 1e-9


# --- library routine: scaled-dot-product attention per branch ---------------------------

@pytest.mark.parametrize("n_branch", [1, 2, 4])
def test_matches_library_sdpa(n_branch):
    """Each branch is ordinary attention of the query over keys [K_nope^(b); K_R] and
    values V^(b); torch's scaled_dot_product_attention (float64, explicit scale) over
    those, summed with sigma_o, must equal the oracle. Catches: wrong softmax scale,
    missing rope term, alpha_q on the rope part, wrong value projection."""
    rng = np.random.default_rng(20 + n_branch)
    q, c, kr, wuk, wuv = _rand_case(rng, h=5, L=41, n_branch=n_branch)
    aq, akv, sig = 1.1547, 2.0, 0.5
    qd, cd, krd = (x.to(torch.float64) for x in (q, c, kr))
    wukd, wuvd = wuk.to(torch.float64), wuv.to(torch.float64)
    L, w = cd.shape[0], 512 // n_branch
    q_r = torch.from_numpy(oracle.rope_rotate(qd[:, 128:].numpy(), L - 1))
    qq = torch.cat([aq * qd[:, :128], q_r], dim=1)                   # [h, 192]
    out = torch.zeros(5, 128, dtype=torch.float64)
    for b in range(n_branch):
        cb = cd[:, b * w:(b + 1) * w]
        K = torch.cat([akv * torch.einsum("lw,hwd->hld", cb, wukd[:, b * w:(b + 1) * w]),
                       krd.expand(5, L, 64)], dim=2)                 # [h, L, 192]
        V = akv * torch.einsum("lw,hwd->hld", cb, wuvd[:, b * w:(b + 1) * w])
        o = torch.nn.functional.scaled_dot_product_attention(
            qq[:, None, :], K, V, scale=1.0 / math.sqrt(192.0))
        out += o[:, 0, :]
    out = (sig * out).numpy()
    kw = dict(alpha_q=aq, alpha_kv=akv, branch_scale=sig)
    assert _rel(oracle.mlra_decode_expanded(q, c, kr, wuk, wuv, n_branch, **kw), out) < 1e-12
    assert _rel(oracle.mlra_decode_absorbed(q, c, kr, wuk, wuv, n_branch, **kw), out) < 1e-12


# --- closed forms --------------------------------------------------------------------------

@pytest.mark.parametrize("n_branch", [1, 2, 4])
def test_single_token_closed_form(n_branch):
    """T=1: every branch's softmax is [1], so out = sigma_o alpha_kv c W_UV[i] (the full
    latent contraction, since the branches partition the latent)."""
    rng = np.random.default_rng(30 + n_branch)
    q, c, kr, wuk, wuv = _rand_case(rng, h=3, L=1, n_branch=n_branch)
    ref = 0.5 * 1.7 * np.einsum("c,hcv->hv", c.to(torch.float64).numpy()[0], wuv.to(torch.float64).numpy())
    for fn in (oracle.mlra_decode_expanded, oracle.mlra_decode_absorbed):
        got = fn(q, c, kr, wuk, wuv, n_branch, alpha_kv=1.7, branch_scale=0.5)
        assert _rel(got, ref) < 1e-13


def test_uniform_attention_closed_form():
    """q = 0: all scores are 0, every weight is 1/L, so out = sigma_o alpha_kv mean_t(C_t) W_UV."""
    rng = np.random.default_rng(40)
    _, c, kr, wuk, wuv = _rand_case(rng, h=2, L=50, n_branch=4)
    q = torch.zeros(2, 192, dtype=torch.bfloat16)
    mean = c.to(torch.float64).numpy().mean(axis=0)
    ref = 0.5 * 3.0 * np.einsum("c,hcv->hv", mean, wuv.to(torch.float64).numpy())
    for fn in (oracle.mlra_decode_expanded, oracle.mlra_decode_absorbed):
        assert _rel(fn(q, c, kr, wuk, wuv, 4, alpha_kv=3.0, branch_scale=0.5), ref) < 1e-13


def test_two_token_sigmoid_weights():
    """T=2: branch b's weight on token 1 is sigmoid(s_1 - s_0), with s_t computed from the
    definition's score formula for one head."""
    rng = np.random.default_rng(41)
    q, c, kr, wuk, wuv = _rand_case(rng, h=1, L=2, n_branch=4, bf16=False)
    aq, akv, tau = 0.9, 1.2, 1 / math.sqrt(192)
    qr = oracle.rope_rotate(q[0, 128:], 1)
    out = np.zeros(128)
    for b in range(4):
        sl = slice(128 * b, 128 * b + 128)
        s = [tau * (aq * q[0, :128] @ (akv * c[t, sl] @ wuk[0, sl]) + qr @ kr[t]) for t in range(2)]
        p1 = 1.0 / (1.0 + math.exp(s[0] - s[1]))
        out += akv * ((1 - p1) * c[0, sl] + p1 * c[1, sl]) @ wuv[0, sl]
    got = oracle.mlra_decode_expanded(q, c, kr, wuk, wuv, 4, alpha_q=aq, alpha_kv=akv, branch_scale=1.0)
    assert _rel(got[0], out) < 1e-13


def test_linearity_and_permutation():
    """out is linear in W_UV and sigma_o, and invariant to permuting cached tokens (key
    and value rows together)."""
    rng = np.random.default_rng(42)
    q, c, kr, wuk, wuv = _rand_case(rng, h=2, L=33, n_branch=4, bf16=False)
    base = oracle.mlra_decode_absorbed(q, c, kr, wuk, wuv, 4)
    assert _rel(oracle.mlra_decode_absorbed(q, c, kr, wuk, 2 * wuv, 4), 2 * base) < 1e-13
    assert _rel(oracle.mlra_decode_absorbed(q, c, kr, wuk, wuv, 4, branch_scale=1.0), 2 * base) < 1e-13
    perm = rng.permutation(33)
    assert _rel(oracle.mlra_decode_absorbed(q, c[perm], kr[perm], wuk, wuv, 4), base) < 1e-12


# --- brute force on tiny inputs ---------------------------------------------------------------

def _brute(q, c, kr, wuk, wuv, nb, aq, akv, sig, theta):
    """Scalar-loop evaluation with math.exp/cos/sin only."""
    h, dqk = len(q), len(q[0])
    L, dc, dr = len(c), len(c[0]), len(kr[0])
    dn, dv, w = dqk - dr, len(wuv[0][0]), dc // nb
    pos, half = L - 1, dr // 2
    res = []
    for i in range(h):
        qr = [0.0] * dr
        for j in range(half):
            a = pos * theta ** (-2.0 * j / dr)
            x1, x2 = q[i][dn + j], q[i][dn + half + j]
            qr[j] = x1 * math.cos(a) - x2 * math.sin(a)
            qr[half + j] = x1 * math.sin(a) + x2 * math.cos(a)
        o = [0.0] * dv
        for b in range(nb):
            scores, vals = [], []
            for t in range(L):
                kn = [akv * sum(c[t][b * w + r] * wuk[i][b * w + r][d] for r in range(w)) for d in range(dn)]
                vv = [akv * sum(c[t][b * w + r] * wuv[i][b * w + r][d] for r in range(w)) for d in range(dv)]
                s = sum(aq * q[i][d] * kn[d] for d in range(dn)) + sum(qr[d] * kr[t][d] for d in range(dr))
                scores.append(s / math.sqrt(dn + dr))
                vals.append(vv)
            mx = max(scores)
            e = [math.exp(s - mx) for s in scores]
            z = sum(e)
            for t in range(L):
                for d in range(dv):
                    o[d] += e[t] / z * vals[t][d]
        res.append([sig * x for x in o])
    return np.array(res)


@pytest.mark.parametrize("nb", [1, 2, 4])
def test_brute_force_tiny(nb):
    rng = np.random.default_rng(50 + nb)
    h, L, dc, dr, dn, dv = 2, 4, 8, 4, 4, 3
    q = rng.standard_normal((h, dn + dr))
    c = rng.standard_normal((L, dc))
    kr = rng.standard_normal((L, dr))
    wuk = rng.standard_normal((h, dc, dn))
    wuv = rng.standard_normal((h, dc, dv))
    kw = dict(alpha_q=1.5, alpha_kv=0.8, branch_scale=0.6, rope_theta=100.0)
    ref = _brute(q.tolist(), c.tolist(), kr.tolist(), wuk.tolist(), wuv.tolist(), nb, 1.5, 0.8, 0.6, 100.0)
    assert _rel(oracle.mlra_decode_expanded(q, c, kr, wuk, wuv, nb, **kw), ref) < 1e-12
    assert _rel(oracle.mlra_decode_absorbed(q, c, kr, wuk, wuv, nb, **kw), ref) < 1e-12


# --- hand-worked fixtures ----------------------------------------------------------------------

@pytest.mark.parametrize("path", sorted(GOLDEN.glob("hand_*.json")), ids=lambda p: p.stem)
def test_hand_worked_fixture(path):
    """Tiny cases whose result follows by hand from the definition (see each file)."""
    fx = json.loads(path.read_text())
    a = {k: np.array(v, dtype=np.float64) for k, v in fx["inputs"].items()}
    got = oracle.mlra_decode_expanded(a["q"], a["c_kv"], a["k_rope"], a["w_uk"], a["w_uv"],
                                      fx["n_branch"], alpha_q=fx["alpha_q"], alpha_kv=fx["alpha_kv"],
                                      branch_scale=fx["branch_scale"], softmax_scale=fx.get("softmax_scale"),
                                      rope_theta=fx.get("rope_theta", 10000.0))
    expected = eval(fx["expected_expr"], {"math": math, "np": np})  # closed form stated in the file
    np.testing.assert_allclose(got, np.array(expected, dtype=np.float64), rtol=1e-13, atol=1e-13)


def test_oracle_snapshot():
    """Regression snapshot written by tests/golden/make_oracle_snapshot.py (oracle only)."""
    fx = json.loads((GOLDEN / "oracle_snapshot_small.json").read_text())
    wl = synth.WORKLOADS[fx["workload"]]
    inp = synth.make_inputs(wl)
    got = oracle.decode_batch(inp, wl, heads=fx["heads"], seqs=[0], form="expanded")[0]
    np.testing.assert_allclose(got, np.array(fx["out"]), rtol=1e-12, atol=1e-12)


# --- quantised (int8) latent cache --------------------------------------------------------

def test_int8_dequantize_places_each_block_scale_on_its_columns():
    """x[r, c] = q[r, c] * scale[r, c // 128]; distinct power-of-two scales per block make
    any mix-up of blocks, or a division for the product, visible exactly."""
    rng = np.random.default_rng(11)
    q = rng.integers(-127, 128, size=(6, 512)).astype(np.int8)
    scale = np.array([[2.0 ** (b - r) for b in range(4)] for r in range(6)], dtype=np.float32)
    x = oracle.dequantize_int8_blocks(q, scale)
    expect = q.astype(np.float64) * (2.0 ** (np.arange(512)[None, :] // 128 - np.arange(6)[:, None]))
    assert np.array_equal(x, expect)


def test_int8_round_trip_within_half_a_step():
    """The cache format (synth) read back by the oracle: every value is within half a
    quantisation step of the bf16 value it stands for (plus the fp32 rounding of x / scale,
    at most 127 * 2^-24 steps), and each block's largest value maps to +-127."""
    x = (torch.randn(40, 512) * torch.tensor([0.5, 1.0, 4.0, 16.0]).repeat_interleave(128)).to(torch.bfloat16)
    q, s = synth.quantize_int8_blocks(x)
    back = oracle.dequantize_int8_blocks(q, s)
    step = np.repeat(s.double().numpy(), 128, axis=1)
    assert (np.abs(back - x.double().numpy()) <= (0.5 + 1e-4) * step).all()
    assert (q.view(40, 4, 128).abs().amax(dim=2) == 127).all()


@pytest.mark.parametrize("page_size", [0, 32])
def test_int8_decode_on_integer_cache_equals_bf16_decode(page_size):
    """Integer latent values in [-127, 127] with a 127 in every block quantise with scale
    exactly 1, so the int8 decode must equal the bf16 decode of the same values."""
    wl = synth.Workload("int8_pin", 4, 2, 4, 100, lengths=(37, 100), page_size=page_size)
    inp = synth.make_inputs(wl)
    rng = np.random.default_rng(5)
    lat = rng.integers(-127, 128, size=(inp.cache.shape[0], 512)).astype(np.float32)
    lat[:, ::128] = 127.0
    inp.cache[:, :512] = torch.from_numpy(lat).to(torch.bfloat16)
    q8, s = synth.quantize_int8_blocks(inp.cache[:, :512])
    assert (s == 1.0).all()
    got = oracle.decode_batch_int8(inp, wl, q8.numpy(), s.numpy())
    ref = oracle.decode_batch(inp, wl)
    assert _rel(got, ref) < 1e-12


# ---- a sequence split by token range (partial states and their combination) ---------------

def _cp_case(seed=5, h=3, L=61):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((h, 192))
    C = rng.standard_normal((L, 512))
    KR = rng.standard_normal((L, 64))
    wk = rng.standard_normal((h, 512, 128)) / 16
    wv = rng.standard_normal((h, 512, 128)) / 16
    return q, C, KR, wk, wv


@pytest.mark.parametrize("n_branch", [1, 2, 4])
@pytest.mark.parametrize("cuts", [(0, 61), (0, 20, 61), (0, 1, 30, 30, 60, 61), (0, 15, 31, 46, 61)])
def test_partial_states_combine_to_the_whole_sequence_decode(n_branch, cuts):
    """Decoding disjoint token ranges against the query at the sequence's last position and
    merging the states by their log-sum-exp gives the decode of the whole sequence (the
    softmax denominator is the sum of the ranges' denominators); empty ranges included."""
    q, C, KR, wk, wv = _cp_case()
    L = C.shape[0]
    full = oracle.mlra_decode_expanded(q, C, KR, wk, wv, n_branch, alpha_q=1.2, alpha_kv=0.8)
    parts = [oracle.mlra_partial_state(q, C[a:b], KR[a:b], wk, n_branch, L - 1, alpha_q=1.2, alpha_kv=0.8)
             for a, b in zip(cuts[:-1], cuts[1:])]
    o, lse = oracle.combine_partial_states(parts)
    np.testing.assert_allclose(oracle.upproject_latent(o, wv, alpha_kv=0.8), full, rtol=0, atol=1e-12)
    whole = oracle.mlra_partial_state(q, C, KR, wk, n_branch, L - 1, alpha_q=1.2, alpha_kv=0.8)
    np.testing.assert_allclose(lse, whole[1], rtol=0, atol=1e-12)


def test_partial_state_of_one_token_closed_form():
    """Over a single token t the softmax is 1: o^(b) = C_t^(b), and lse^(b) is the token's
    score in log2 units, tau (q~ . k_t) / ln 2, computed here from the expanded key."""
    q, C, KR, wk, _ = _cp_case(h=2)
    L, t, tau = C.shape[0], 17, 1.0 / math.sqrt(192)
    o, lse = oracle.mlra_partial_state(q, C[t:t + 1], KR[t:t + 1], wk, 4, L - 1)
    for i in range(2):
        q_r = oracle.rope_rotate(q[i, 128:], L - 1)
        for b in range(4):
            cols = slice(128 * b, 128 * b + 128)
            np.testing.assert_array_equal(o[i, b], C[t, cols])
            k = np.concatenate([C[t, cols] @ wk[i, cols, :], KR[t]])
            assert abs(lse[i, b] - tau * (k @ np.concatenate([q[i, :128], q_r])) / math.log(2.0)) < 1e-12


def test_empty_partial_state_carries_no_weight():
    q, C, KR, wk, wv = _cp_case()
    L = C.shape[0]
    empty = oracle.mlra_partial_state(q, C[:0], KR[:0], wk, 4, L - 1)
    assert np.all(empty[1] == -np.inf) and np.all(empty[0] == 0)
    whole = oracle.mlra_partial_state(q, C, KR, wk, 4, L - 1)
    o, lse = oracle.combine_partial_states([empty, whole, empty])
    np.testing.assert_allclose(o, whole[0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, whole[1], rtol=0, atol=1e-15)
