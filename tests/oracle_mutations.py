"""Plausible mistakes planted in the oracle, in memory, for tests/test_oracle_mutations.py.

Each entry replaces one piece of source text in one oracle function and re-defines that
function inside oracle.reference (and the oracle package), so that the pins in
tests/test_oracle_pins.py can be run against a wrong oracle.  Nothing on disk changes.
"""
import inspect
import textwrap

# (function, source text, replacement, the mistake it stands for)
MUTATIONS = [
    ("rope_rotate", "x1 * c - x2 * s", "x1 * c + x2 * s", "rotation sign"),
    ("rope_rotate", "theta ** (-2.0 * j / d)", "theta ** (-1.0 * j / d)", "rotation frequencies"),
    ("mlra_decode_absorbed", "pos = L - 1", "pos = L", "query position off by one"),
    ("mlra_decode_absorbed", "alpha_q * alpha_kv * np.einsum", "alpha_q * np.einsum", "alpha_kv dropped from the key"),
    ("mlra_decode_absorbed", "math.sqrt(d_nope + d_rope) if", "math.sqrt(d_nope) if", "softmax scale"),
    ("mlra_decode_absorbed", "@ C[:, cols].T + s_rope)", "@ C[:, cols].T)", "rope score dropped"),
    ("mlra_decode_absorbed", "out += alpha_kv * np.einsum", "out += np.einsum", "alpha_kv dropped from the value"),
    ("mlra_decode_absorbed", "w_uk[heads], q[heads, :d_nope]", "w_uv[heads], q[heads, :d_nope]", "W_UV used for W_UK"),
    ("mlra_decode_absorbed", "+= p[b, :, t0:t1] @ C[:, cols]", "+= p[0, :, t0:t1] @ C[:, cols]",
     "branch 0's weights for every branch"),
    ("mlra_decode_absorbed", "return sigma * out", "return out", "branch-sum scale dropped"),
    ("mlra_decode_expanded", "q_n = alpha_q * q[i, :d_nope]", "q_n = q[i, :d_nope]", "alpha_q dropped"),
    ("mlra_decode_expanded", "K = np.concatenate([K_nope, k_rope], axis=1)",
     "K = np.concatenate([K_nope, 0 * k_rope], axis=1)", "rope key dropped"),
    ("mla_decode", "1.0 / math.sqrt(d_qk) if", "1.0 / math.sqrt(d_nope) if", "MLA softmax scale"),
    ("gla_decode", "c_kv[:, g * w:(g + 1) * w]", "c_kv[:, 0:w]", "every head group on the first latent group"),
    ("gla_decode", "heads = slice(g * per, (g + 1) * per)", "heads = slice(0, per)", "every group on the first heads"),
    ("mlra_prefill_expanded", "np.arange(L)[None, :] <= pos[:, None]", "np.arange(L)[None, :] < pos[:, None]",
     "causal mask hides the query's own token"),
    ("dequantize_int8_blocks", "np.repeat(s[:, :d // block], block, axis=1)", "np.tile(s[:, :d // block], (1, block))",
     "int8 block scales on the wrong columns"),
    ("dequantize_int8_blocks", "return q * np.repeat", "return q / np.repeat", "int8 scale divided instead of multiplied"),
    ("decode_batch_int8", "astype(np.int64) * P + t % P", "astype(np.int64) * P", "int8 cache page offset dropped"),
    ("mlra_prefill_expanded", "rope_rotate(q[j, i, d_nope:], int(pos[j]), rope_theta)",
     "rope_rotate(q[j, i, d_nope:], L - 1, rope_theta)", "every query rotated to the last position"),
    ("mlra_partial_state", "rope_rotate(q[i, d_nope:], pos, rope_theta)",
     "rope_rotate(q[i, d_nope:], c_kv.shape[0] - 1, rope_theta)", "a range's query rotated at the range's end"),
    ("mlra_partial_state", "(m + math.log(e.sum())) / math.log(2.0)", "m + math.log(e.sum())",
     "partial log-sum-exp in natural-log units"),
    ("combine_partial_states", "2.0 ** (lse - m)", "np.exp(lse - m)", "partial weights taken with exp, not 2^"),
    ("combine_partial_states", "(wts[..., None] * o).sum(axis=0) / den[..., None]", "o.mean(axis=0)",
     "partial states averaged, not weighted"),
]


def apply(index: int) -> None:
    """Plant mutation `index` into the imported oracle."""
    import oracle
    from oracle import reference
    name, old, new, _ = MUTATIONS[index]
    src = textwrap.dedent(inspect.getsource(getattr(reference, name)))
    if src.count(old) != 1:
        raise RuntimeError(f"mutation {index}: {old!r} occurs {src.count(old)} times in {name}")
    exec(compile(src.replace(old, new), f"<mutated {name}>", "exec"), reference.__dict__)
    if hasattr(oracle, name):
        setattr(oracle, name, reference.__dict__[name])
