"""fp64 CPU oracle for single-token decode over a compressed latent KV cache.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference arm of ``bench.py`` may import this module.  It shares
no code with the CUDA path (``head_rank_attention_b200``); the only module both
sides use is the seeded input generator ``synth``.

Everything here is plain numpy in float64 on the bf16 input values (converted
exactly).  Sources, by page title and section:

* "Multi-Head Low-Rank Attention" (digest of arXiv 2603.02188):
  - 研究动机: MLA's no-position key K_NoPE^(i) = sum_{b=0..3} C_KV^(b) W_UK^(b),(i);
  - 核心方法: MLA is O = Softmax(Q (sum_b K_b)^T)(sum_b V_b), MLRA is
    O = sum_b Softmax(Q K_b^T) V_b (not equal, the softmax is nonlinear);
  - 方法步骤详情: three decode steps (absorb W_UK into the query, MQA-style
    decode over [C_KV | K_RoPE], up-project with W_UV), MLRA-4 = 4 branches each on
    a quarter of C_KV, summed; scales alpha_q = sqrt(d/d_c'), alpha_kv = sqrt(d/d_c)
    and a scale on the branch sum;
  - 前置知识 (RoPE): scores depend only on relative position.
* "ML Revisit: Attention", section Multi-Head Latent Attention: Q K^T =
  C_q W_q W_k^T C_kv^T (absorption) and the decoupled RoPE branch whose key K_R is
  shared by all heads and concatenated to the content key.
* "vllbc02MLA" (blog.vllbc.top/mla), DeepseekV2Attention.__init__:
  qk_head_dim = qk_nope_head_dim + qk_rope_head_dim, scaling = qk_head_dim ** -0.5,
  kv_b_proj yields the no-position key and the value together.

Readings where the pages are silent (each also listed in the design notes):
* alpha_q multiplies q_nope only; alpha_kv multiplies the kv_b_proj outputs, i.e.
  both K_nope and V; K_R is not scaled.
* The branch-sum scale sigma_o multiplies the sum of branch outputs.
* The softmax scale is tau = 1/sqrt(d_nope + d_rope) for every branch.
* RoPE pairs dimension j with j + d_rope/2 ("rotate half"), theta_j =
  rope_theta^(-2j/d_rope); the cache holds K_R already rotated at its position, the
  query's rope part is rotated here at pos = L - 1.
* Branch b owns latent columns [b*w, (b+1)*w), w = d_c / n_branch, and the matching
  rows of W_UK and W_UV; every branch uses the same per-head query.

Parity pins for every function live in tests/test_oracle_pins.py.
"""
from __future__ import annotations

import math

import numpy as np


def _f64(x) -> np.ndarray:
    """bf16/fp32 torch tensor or array -> float64 numpy (exact)."""
    if hasattr(x, "detach"):
        import torch
        return x.detach().to(torch.float64).cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def rope_rotate(x, pos, theta: float = 10000.0) -> np.ndarray:
    """Rotate the last dimension of x at integer position(s) pos.

    Rotary embedding ("Multi-Head Low-Rank Attention", 前置知识, RoPE): each pair
    (x_j, x_{j+d/2}) is turned by the angle pos * theta^(-2j/d), computed in
    float64.  ``pos`` broadcasts against x's leading dimensions.
    """
    x = _f64(x)
    d = x.shape[-1]
    half = d // 2
    j = np.arange(half, dtype=np.float64)
    inv_freq = theta ** (-2.0 * j / d)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * inv_freq
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x1 * s + x2 * c], axis=-1)


def _softmax(score: np.ndarray) -> np.ndarray:
    p = np.exp(score - score.max())
    return p / p.sum()


def mlra_decode_expanded(q, c_kv, k_rope, w_uk, w_uv, n_branch: int,
                         alpha_q: float = 1.0, alpha_kv: float = 1.0,
                         branch_scale: float | None = None,
                         softmax_scale: float | None = None,
                         rope_theta: float = 10000.0, heads=None) -> np.ndarray:
    """Non-absorbed MLRA decode for ONE sequence (the definition).

    q [h, d_nope + d_rope] (rope part not rotated); c_kv [L, d_c]; k_rope [L, d_rope]
    (already rotated); w_uk [h, d_c, d_nope]; w_uv [h, d_c, d_v].  Returns float64
    [len(heads), d_v].  ``n_branch`` = 1 is MLA.

    For each head i and branch b ("Multi-Head Low-Rank Attention", 核心方法 and
    方法步骤详情):
      K_nope^(b) = alpha_kv * C^(b) W_UK^(b),(i);  V^(b) = alpha_kv * C^(b) W_UV^(b),(i)
      score_t = tau * ([alpha_q q_nope ; RoPE(q_rope)] . [K_nope,t^(b) ; K_R,t])
      o^(b) = softmax(score) V^(b)
    out = sigma_o * sum_b o^(b).
    """
    q, c_kv, k_rope = _f64(q), _f64(c_kv), _f64(k_rope)
    w_uk, w_uv = _f64(w_uk), _f64(w_uv)
    h_all, d_qk = q.shape
    L, d_c = c_kv.shape
    d_rope = k_rope.shape[1]
    d_nope = d_qk - d_rope
    d_v = w_uv.shape[2]
    w = d_c // n_branch
    tau = 1.0 / math.sqrt(d_nope + d_rope) if softmax_scale is None else softmax_scale
    sigma = 1.0 / math.sqrt(n_branch) if branch_scale is None else branch_scale
    heads = range(h_all) if heads is None else heads
    pos = L - 1

    out = np.zeros((len(heads), d_v))
    for row, i in enumerate(heads):
        q_n = alpha_q * q[i, :d_nope]
        q_r = rope_rotate(q[i, d_nope:], pos, rope_theta)
        for b in range(n_branch):
            cols = slice(b * w, (b + 1) * w)
            C_b = c_kv[:, cols]
            K_nope = alpha_kv * (C_b @ w_uk[i, cols, :])        # [L, d_nope]
            V = alpha_kv * (C_b @ w_uv[i, cols, :])             # [L, d_v]
            K = np.concatenate([K_nope, k_rope], axis=1)         # [L, d_nope + d_rope]
            score = tau * (K @ np.concatenate([q_n, q_r]))       # [L]
            out[row] += _softmax(score) @ V
    return sigma * out


def mlra_decode_absorbed(q, c_kv, k_rope, w_uk, w_uv, n_branch: int,
                         alpha_q: float = 1.0, alpha_kv: float = 1.0,
                         branch_scale: float | None = None,
                         softmax_scale: float | None = None,
                         rope_theta: float = 10000.0, heads=None,
                         token_chunk: int = 1 << 16) -> np.ndarray:
    """Weight-absorbed MLRA decode for ONE sequence, in the three steps of
    "Multi-Head Low-Rank Attention", 方法步骤详情:

    1. query-side absorption: q~^(b),(i) = alpha_q alpha_kv W_UK^(b),(i) q_nope^(i)
       (a w-vector per head and branch), RoPE on q_rope;
    2. MQA-style decode over the shared key [C_KV | K_RoPE] and value C_KV:
       score_t^(b) = tau (C_t^(b) . q~^(b) + K_R,t . RoPE(q_rope)),
       o_lat^(b) = softmax(score^(b)) C^(b);
    3. output up-projection: out = sigma_o * sum_b alpha_kv o_lat^(b) W_UV^(b),(i).

    Same arguments and result as :func:`mlra_decode_expanded` ("ML Revisit:
    Attention", Multi-Head Latent Attention: Q K^T = C_q W_q W_k^T C_kv^T).
    The scores of all tokens are formed first (in token chunks only to bound
    memory; every score is the same dot product), then the softmax over all of
    them, then the weighted sum of latent rows.
    """
    q = _f64(q)
    w_uk, w_uv = _f64(w_uk), _f64(w_uv)
    h_all, d_qk = q.shape
    L, d_c = c_kv.shape
    d_rope = k_rope.shape[1]
    d_nope = d_qk - d_rope
    d_v = w_uv.shape[2]
    w = d_c // n_branch
    tau = 1.0 / math.sqrt(d_nope + d_rope) if softmax_scale is None else softmax_scale
    sigma = 1.0 / math.sqrt(n_branch) if branch_scale is None else branch_scale
    heads = list(range(h_all)) if heads is None else list(heads)
    hs = len(heads)
    pos = L - 1

    # step 1: absorbed queries [hs, d_c] (branch b in columns b*w:(b+1)*w) and rotated rope
    q_tilde = alpha_q * alpha_kv * np.einsum("hcn,hn->hc", w_uk[heads], q[heads, :d_nope])
    q_r = rope_rotate(q[heads, d_nope:], pos, rope_theta)            # [hs, d_rope]

    # step 2a: every score, per branch: [n_branch, hs, L]
    score = np.empty((n_branch, hs, L))
    for t0 in range(0, L, token_chunk):
        t1 = min(L, t0 + token_chunk)
        C = _f64(c_kv[t0:t1])
        KR = _f64(k_rope[t0:t1])
        s_rope = q_r @ KR.T                                          # [hs, n]
        for b in range(n_branch):
            cols = slice(b * w, (b + 1) * w)
            score[b, :, t0:t1] = tau * (q_tilde[:, cols] @ C[:, cols].T + s_rope)
    # step 2b: softmax per (branch, head) over all L tokens
    score -= score.max(axis=2, keepdims=True)
    p = np.exp(score)
    p /= p.sum(axis=2, keepdims=True)
    # step 2c: latent outputs o_lat^(b) = sum_t p_t C_t^(b): [hs, d_c]
    o_lat = np.zeros((hs, d_c))
    for t0 in range(0, L, token_chunk):
        t1 = min(L, t0 + token_chunk)
        C = _f64(c_kv[t0:t1])
        for b in range(n_branch):
            cols = slice(b * w, (b + 1) * w)
            o_lat[:, cols] += p[b, :, t0:t1] @ C[:, cols]
    # step 3: up-projection, branch sum and scales
    out = np.zeros((hs, d_v))
    for b in range(n_branch):
        cols = slice(b * w, (b + 1) * w)
        out += alpha_kv * np.einsum("hc,hcv->hv", o_lat[:, cols], w_uv[heads][:, cols, :])
    return sigma * out


def mla_decode(q, c_kv, k_rope, w_uk, w_uv, alpha_q: float = 1.0, alpha_kv: float = 1.0,
               softmax_scale: float | None = None, rope_theta: float = 10000.0,
               heads=None) -> np.ndarray:
    """Plain MLA decode for ONE sequence, written from the MLA pages alone.

    "ML Revisit: Attention" (Multi-Head Latent Attention): content key K = C_kv W_k
    and value V = C_kv W_v per head, plus a RoPE key K_R shared by all heads and
    concatenated to the content key; the query likewise concatenates a content part
    and a rotated part.  "vllbc02MLA" (DeepseekV2Attention.__init__): kv_b_proj maps
    kv_lora_rank to the per-head (nope + v) features, scaling = qk_head_dim ** -0.5.
    The variance-correction scales of "Multi-Head Low-Rank Attention" (方法步骤详情)
    also apply to MLA: alpha_q on the query content part, alpha_kv on kv_b_proj.
    """
    q, c_kv, k_rope = _f64(q), _f64(c_kv), _f64(k_rope)
    w_uk, w_uv = _f64(w_uk), _f64(w_uv)
    h_all, d_qk = q.shape
    L = c_kv.shape[0]
    d_rope = k_rope.shape[1]
    d_nope = d_qk - d_rope
    scale = 1.0 / math.sqrt(d_qk) if softmax_scale is None else softmax_scale
    heads = range(h_all) if heads is None else heads
    rows = []
    for i in heads:
        k_content = alpha_kv * (c_kv @ w_uk[i])
        v = alpha_kv * (c_kv @ w_uv[i])
        k = np.concatenate([k_content, k_rope], axis=1)
        q_full = np.concatenate([alpha_q * q[i, :d_nope], rope_rotate(q[i, d_nope:], L - 1, rope_theta)])
        a = _softmax(scale * (k @ q_full))
        rows.append(a @ v)
    return np.stack(rows)


def mlra_prefill_expanded(q, c_kv, k_rope, w_uk, w_uv, n_branch: int,
                          alpha_q: float = 1.0, alpha_kv: float = 1.0,
                          branch_scale: float | None = None,
                          softmax_scale: float | None = None,
                          rope_theta: float = 10000.0) -> np.ndarray:
    """Causal multi-token (prefill) MLRA for ONE sequence, in the expanded form.

    "vllbc02MLA" contrasts the two phases: prefill is compute-bound and forms the per-head
    keys and values (the expanded form), generation is memory-bound and uses the absorbed
    form.  The n query tokens are the last n of the sequence, at positions
    p_j = L - n + j; query j attends to the tokens t <= p_j with the per-branch softmax of
    "Multi-Head Low-Rank Attention" (核心方法), exactly as :func:`mlra_decode_expanded` would
    for the first p_j + 1 tokens.

    q [n, h, d_nope + d_rope] (rope part not rotated); c_kv [L, d_c]; k_rope [L, d_rope]
    (already rotated); w_uk [h, d_c, d_nope]; w_uv [h, d_c, d_v].  Returns [n, h, d_v].
    """
    q, c_kv, k_rope = _f64(q), _f64(c_kv), _f64(k_rope)
    w_uk, w_uv = _f64(w_uk), _f64(w_uv)
    n, h, d_qk = q.shape
    L, d_c = c_kv.shape
    d_rope = k_rope.shape[1]
    d_nope = d_qk - d_rope
    if n > L:
        raise ValueError(f"{n} query tokens but only {L} cached")
    w = d_c // n_branch
    tau = 1.0 / math.sqrt(d_nope + d_rope) if softmax_scale is None else softmax_scale
    sigma = 1.0 / math.sqrt(n_branch) if branch_scale is None else branch_scale
    pos = np.arange(L - n, L)
    visible = np.arange(L)[None, :] <= pos[:, None]                  # [n, L] causal mask
    out = np.zeros((n, h, w_uv.shape[2]))
    for i in range(h):
        q_n = alpha_q * q[:, i, :d_nope]                               # [n, d_nope]
        q_r = np.stack([rope_rotate(q[j, i, d_nope:], int(pos[j]), rope_theta) for j in range(n)])
        for b in range(n_branch):
            cols = slice(b * w, (b + 1) * w)
            K_nope = alpha_kv * (c_kv[:, cols] @ w_uk[i, cols, :])      # [L, d_nope]
            V = alpha_kv * (c_kv[:, cols] @ w_uv[i, cols, :])           # [L, d_v]
            score = tau * (q_n @ K_nope.T + q_r @ k_rope.T)            # [n, L]
            score = np.where(visible, score, -np.inf)
            score -= score.max(axis=1, keepdims=True)
            p = np.exp(score)
            p /= p.sum(axis=1, keepdims=True)
            out[:, i] += p @ V
    return sigma * out


def gla_decode(q, c_kv, k_rope, w_uk, w_uv, n_groups: int = 2, alpha_q: float = 1.0, alpha_kv: float = 1.0,
               softmax_scale: float | None = None, rope_theta: float = 10000.0) -> np.ndarray:
    """Grouped latent attention (GLA-n) decode for ONE sequence.

    "Multi-Head Low-Rank Attention" (研究动机) describes GLA-2 as MLA's single latent head
    split into two groups, so that each of 2 devices loads 2.5 d_h per token (its 256
    latent columns and the shared rope key).  Reading (the page gives no more): the h
    heads form n_groups contiguous groups of h / n_groups; head i of group g attends
    with the MLA formula over latent columns [g*w, (g+1)*w), w = d_c / n_groups, and the
    shared K_R; its W_UK[i], W_UV[i] are [w, d] (the group's rows only).  No branch sum.

    q [h, d_nope + d_rope]; c_kv [L, d_c]; k_rope [L, d_rope]; w_uk [h, w, d_nope];
    w_uv [h, w, d_v].  Returns float64 [h, d_v].
    """
    h, d_c = int(np.shape(q)[0]), int(np.shape(c_kv)[1])
    if h % n_groups or d_c % n_groups:
        raise ValueError(f"{h} heads / {d_c} latent columns do not split into {n_groups} groups")
    w, per = d_c // n_groups, h // n_groups
    c_kv = _f64(c_kv)
    out = []
    for g in range(n_groups):
        heads = slice(g * per, (g + 1) * per)
        out.append(mla_decode(_f64(q)[heads], c_kv[:, g * w:(g + 1) * w], k_rope, _f64(w_uk)[heads],
                              _f64(w_uv)[heads], alpha_q=alpha_q, alpha_kv=alpha_kv,
                              softmax_scale=softmax_scale, rope_theta=rope_theta))
    return np.concatenate(out)


def mla_nope_key(c_kv, w_uk_i) -> np.ndarray:
    """MLA's per-head no-position key C_KV W_UK^(i) over the whole latent, [L, d_nope]."""
    return _f64(c_kv) @ _f64(w_uk_i)


def mlra_nope_key_blocks(c_kv, w_uk_i, n_blocks: int) -> np.ndarray:
    """sum_b C_KV^(b) W_UK^(b),(i) with the latent split into n_blocks column blocks
    ("Multi-Head Low-Rank Attention", 研究动机)."""
    c_kv, w_uk_i = _f64(c_kv), _f64(w_uk_i)
    w = c_kv.shape[1] // n_blocks
    return sum(c_kv[:, b * w:(b + 1) * w] @ w_uk_i[b * w:(b + 1) * w] for b in range(n_blocks))


def dequantize_int8_blocks(q, scale, block: int = 128) -> np.ndarray:
    """The value an int8 latent cache stands for: x[r, c] = q[r, c] * scale[r, c // block].

    Quantised latent cache ("从MHA到MLA", 部署注意事项: INT8 for inference; "Multi-Head
    Low-Rank Attention", 未来方向: combine MLRA with KV-cache quantisation).  The pages fix
    neither the scheme nor its granularity; read here as symmetric int8 with one scale per
    token and 128-column latent block (one per MLRA-4 branch).  Exact in float64.
    """
    q = _f64(q)
    s = _f64(scale)
    rows, d = q.shape
    return q * np.repeat(s[:, :d // block], block, axis=1)


def decode_batch_int8(inp, wl, q8, scale, heads=None, seqs=None) -> np.ndarray:
    """The absorbed oracle over a batch whose latent cache is int8 (q8 [rows, d_c] and
    scale [rows, d_c / 128], physical rows like inp.cache): each sequence's latent rows are
    dequantised (:func:`dequantize_int8_blocks`) and K_RoPE taken from inp.cache as it is."""
    from synth import D_C
    seqs = range(int(inp.seq_lens.shape[0])) if seqs is None else seqs
    res = []
    for s in seqs:
        L = int(inp.seq_lens[s])
        if inp.block_table is None:
            phys = np.arange(s * inp.seq_stride, s * inp.seq_stride + L)
        else:
            t = np.arange(L)
            P = wl.page_size
            phys = inp.block_table.numpy()[s, t // P].astype(np.int64) * P + t % P
        c = dequantize_int8_blocks(q8[phys], scale[phys])
        res.append(mlra_decode_absorbed(inp.q[s], c, inp.cache[phys][:, D_C:], inp.w_uk, inp.w_uv, wl.n_branch,
                                        alpha_q=wl.alpha_q, alpha_kv=wl.alpha_kv, branch_scale=wl.sigma_o,
                                        softmax_scale=wl.softmax_scale, rope_theta=wl.rope_theta, heads=heads))
    return np.stack(res)


def mlra_partial_state(q, c_kv, k_rope, w_uk, n_branch: int, pos: int, alpha_q: float = 1.0,
                       alpha_kv: float = 1.0, softmax_scale: float | None = None,
                       rope_theta: float = 10000.0, heads=None):
    """The decode's state over a subset of one sequence's cached tokens, for a sequence
    split across devices by token range.

    c_kv [n, d_c] and k_rope [n, d_rope] are the subset's rows (K_R rotated at their own
    positions); ``pos`` is the query's position, the sequence's last token, whatever the
    subset.  For each head i and branch b, with the expanded scores of
    ``mlra_decode_expanded`` restricted to the subset,
      o^(b)   = sum_t softmax_t C_t^(b)        (the branch's latent columns, before W_UV)
      lse^(b) = log2 sum_t exp(score_t)        (-inf for an empty subset, with o = 0)
    Returns (o [len(heads), n_branch, w], lse [len(heads), n_branch]).
    """
    q, c_kv, k_rope, w_uk = _f64(q), _f64(c_kv), _f64(k_rope), _f64(w_uk)
    h_all, d_qk = q.shape
    d_c = w_uk.shape[1]
    d_rope = k_rope.shape[1]
    d_nope = d_qk - d_rope
    w = d_c // n_branch
    tau = 1.0 / math.sqrt(d_nope + d_rope) if softmax_scale is None else softmax_scale
    heads = range(h_all) if heads is None else heads
    o = np.zeros((len(heads), n_branch, w))
    lse = np.full((len(heads), n_branch), -np.inf)
    if c_kv.shape[0] == 0:
        return o, lse
    for row, i in enumerate(heads):
        q_n = alpha_q * q[i, :d_nope]
        q_r = rope_rotate(q[i, d_nope:], pos, rope_theta)
        for b in range(n_branch):
            cols = slice(b * w, (b + 1) * w)
            K_nope = alpha_kv * (c_kv[:, cols] @ w_uk[i, cols, :])
            score = tau * (np.concatenate([K_nope, k_rope], axis=1) @ np.concatenate([q_n, q_r]))
            m = score.max()
            e = np.exp(score - m)
            o[row, b] = e @ c_kv[:, cols] / e.sum()
            lse[row, b] = (m + math.log(e.sum())) / math.log(2.0)
    return o, lse


def combine_partial_states(states):
    """Merge partial states of disjoint token subsets of one sequence: with
    m = max_r lse_r, weight_r = 2^(lse_r - m) (each subset's share of the softmax
    denominator), o = sum_r weight_r o_r / sum_r weight_r and lse = m + log2 sum_r weight_r.
    ``states`` is a list of (o, lse) from ``mlra_partial_state``."""
    o = np.stack([s[0] for s in states])        # [R, h, nb, w]
    lse = np.stack([s[1] for s in states])      # [R, h, nb]
    m = lse.max(axis=0)
    wts = np.where(np.isfinite(lse), 2.0 ** (lse - m), 0.0)
    den = wts.sum(axis=0)
    return (wts[..., None] * o).sum(axis=0) / den[..., None], m + np.log2(den)


def upproject_latent(o, w_uv, alpha_kv: float = 1.0, branch_scale: float | None = None, heads=None):
    """Step 3 of the decode (方法步骤详情) on latent outputs o [len(heads), n_branch, w]:
    out^(i) = sigma_o alpha_kv sum_b o^(b),(i) W_UV^(b),(i)."""
    w_uv = _f64(w_uv)
    n_branch, w = o.shape[1], o.shape[2]
    sigma = 1.0 / math.sqrt(n_branch) if branch_scale is None else branch_scale
    heads = range(w_uv.shape[0]) if heads is None else heads
    out = np.zeros((len(heads), w_uv.shape[2]))
    for row, i in enumerate(heads):
        for b in range(n_branch):
            out[row] += o[row, b] @ w_uv[i, b * w:(b + 1) * w, :]
    return sigma * alpha_kv * out


def decode_batch(inp, wl, heads=None, seqs=None, form: str = "absorbed") -> np.ndarray:
    """Run the oracle over sequences of a synth.Inputs; returns [len(seqs), len(heads), d_v]."""
    from synth import logical_rows, D_C
    seqs = range(int(inp.seq_lens.shape[0])) if seqs is None else seqs
    fn = mlra_decode_absorbed if form == "absorbed" else mlra_decode_expanded
    res = []
    for s in seqs:
        rows = logical_rows(inp, wl, s)
        res.append(fn(inp.q[s], rows[:, :D_C], rows[:, D_C:], inp.w_uk, inp.w_uv, wl.n_branch,
                      alpha_q=wl.alpha_q, alpha_kv=wl.alpha_kv, branch_scale=wl.sigma_o,
                      softmax_scale=wl.softmax_scale, rope_theta=wl.rope_theta, heads=heads))
    return np.stack(res)
