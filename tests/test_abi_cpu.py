"""CPU checks of the C-ABI library: it loads, exports every symbol include/hra.h declares,
the ctypes mirror of hra_decode_params has the C layout, and argument validation
returns the documented status before any CUDA call.  No compute runs here."""
import ctypes
import pathlib
import re
import subprocess

import pytest

import head_rank_attention_b200 as hra
from head_rank_attention_b200 import _binding as B

ROOT = pathlib.Path(__file__).resolve().parents[1]
HEADER = ROOT / "include" / "hra.h"


def _declared_symbols():
    text = HEADER.read_text()
    return sorted(set(re.findall(r"HRA_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)))


def test_library_loads_and_exports_every_declared_symbol():
    lib = hra.load_library()
    declared = _declared_symbols()
    assert set(declared) == set(B.EXPORTS), declared
    nm = subprocess.run(["nm", "-D", "--defined-only", str(hra.LIB_PATH)], capture_output=True, text=True, check=True)
    exported = {line.split()[-1] for line in nm.stdout.splitlines() if " T " in line}
    for name in declared:
        assert name in exported, name
        assert hasattr(lib, name)
    assert "sm_100a" in hra.version()


@pytest.mark.parametrize("cls,ctype", [(B.HraDecodeParams, "hra_decode_params"),
                                       (B.HraPrefillParams, "hra_prefill_params")])
def test_params_layout_matches_c(tmp_path, cls, ctype):
    fields = [f[0] for f in cls._fields_]
    prog = tmp_path / "layout.c"
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "hra.h"', 'int main(void) {',
             f'  printf("size %zu\\n", sizeof({ctype}));']
    lines += [f'  printf("{f} %zu\\n", offsetof({ctype}, {f}));' for f in fields]
    lines += ['  return 0;', '}']
    prog.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", f"-I{ROOT / 'include'}", str(prog), "-o", str(exe)], check=True)
    out = dict(line.split() for line in subprocess.run([str(exe)], capture_output=True, text=True,
                                                        check=True).stdout.splitlines())
    assert int(out["size"]) == ctypes.sizeof(cls)
    for f in fields:
        assert int(out[f]) == getattr(cls, f).offset, f


def _fake_params(**over):
    """Well-formed parameters with fake (aligned, never dereferenced) device pointers."""
    p = B.HraDecodeParams()
    p.batch, p.num_heads, p.n_branch = 2, 128, 4
    p.d_c, p.d_rope, p.d_nope, p.d_v = 512, 64, 128, 128
    p.q, p.ckv, p.krope, p.seq_lens = 0x10000, 0x20000, 0x20400, 0x30000
    p.w_uk, p.w_uv, p.out = 0x40000, 0x50000, 0x60000
    p.ckv_stride, p.krope_stride, p.cache_rows, p.seq_stride = 576, 576, 4096, 2048
    p.alpha_q = p.alpha_kv = 1.0
    p.branch_scale, p.softmax_scale, p.rope_theta = 0.5, 0.0, 10000.0
    p.out_dtype = B.HRA_F32
    p.num_splits = 37  # explicit: sizing then needs no device query
    for k, v in over.items():
        setattr(p, k, v)
    return p


@pytest.mark.parametrize("d_c,n_branch,splits", [(512, 4, 37), (512, 1, 37), (256, 2, 74), (256, 1, 74),
                                                   (128, 1, 148)])
def test_workspace_size_formula(d_c, n_branch, splits):
    p = _fake_params(d_c=d_c, n_branch=n_branch, num_splits=splits, ckv_stride=d_c + 64, krope_stride=d_c + 64)
    n = hra.workspace_size(p)
    slots, slices = splits + 2, d_c // 128
    expect = 256
    expect = -(-(expect + 2 * 128 * (d_c + 64) * 2) // 256) * 256  # fp16 q~
    expect = -(-(expect + slots * slices * 128 * 128 * 4) // 256) * 256
    expect = -(-(expect + slots * slices * 128 * 8) // 256) * 256
    expect = -(-(expect + 2 * 128 * 2 * d_c * 2) // 256) * 256  # merged latent as two bf16 terms
    expect = -(-(expect + (2 + 1) * 4) // 256) * 256  # tile prefix per sequence
    assert n == expect


@pytest.mark.parametrize("over,status", [
    (dict(q=0), B.HRA_ERR_INVALID_ARG),
    (dict(ckv=0x20008), B.HRA_ERR_INVALID_ARG),          # misaligned
    (dict(n_branch=3), B.HRA_ERR_UNSUPPORTED),
    (dict(d_c=256), B.HRA_ERR_UNSUPPORTED),
    (dict(d_c=128, n_branch=2, ckv_stride=192), B.HRA_ERR_UNSUPPORTED),   # 64-wide branches
    (dict(d_c=384, n_branch=3, ckv_stride=448), B.HRA_ERR_UNSUPPORTED),
    (dict(d_c=128, n_branch=1, ckv_stride=120), B.HRA_ERR_INVALID_ARG),   # stride below d_c
    (dict(num_heads=129), B.HRA_ERR_UNSUPPORTED),
    (dict(batch=0), B.HRA_ERR_UNSUPPORTED),
    (dict(ckv_stride=580), B.HRA_ERR_INVALID_ARG),        # not a multiple of 8
    (dict(cache_rows=0), B.HRA_ERR_INVALID_ARG),
    (dict(block_table=0x70000, max_pages=4, page_size=48), B.HRA_ERR_UNSUPPORTED),
    (dict(out_dtype=7), B.HRA_ERR_INVALID_ARG),
    (dict(rope_theta=0.0), B.HRA_ERR_INVALID_ARG),
    (dict(workspace=0), B.HRA_ERR_WORKSPACE),
    (dict(workspace=0x80000, workspace_bytes=1024), B.HRA_ERR_WORKSPACE),
    (dict(workspace=0x80010, workspace_bytes=1 << 30), B.HRA_ERR_WORKSPACE),  # not 256-aligned
])
def test_validation_rejects_before_launch(over, status):
    p = _fake_params(**over)
    rc = hra.load_library().mlra_decode(ctypes.byref(p), None)
    assert rc == status, hra.last_error()
    assert hra.last_error() != ""


_GOOD_PEERS = (ctypes.c_void_p * 2)(0x90000, 0xA0000)
_BAD_PEERS = (ctypes.c_void_p * 2)(0x90000, 0xA0008)


@pytest.mark.parametrize("over,status", [
    (dict(out_accumulate=2), B.HRA_ERR_INVALID_ARG),
    (dict(out_accumulate=1, out_dtype=B.HRA_BF16), B.HRA_ERR_INVALID_ARG),
    (dict(out_accumulate=1, n_out_peers=8, out_peers=ctypes.addressof(_GOOD_PEERS)), B.HRA_ERR_UNSUPPORTED),
    (dict(n_out_peers=2, out_peers=ctypes.addressof(_GOOD_PEERS)), B.HRA_ERR_INVALID_ARG),  # no accumulate
    (dict(out_accumulate=1, n_out_peers=2, out_peers=None), B.HRA_ERR_INVALID_ARG),
    (dict(out_accumulate=1, n_out_peers=2, out_peers=ctypes.addressof(_BAD_PEERS)), B.HRA_ERR_INVALID_ARG),
    (dict(out_accumulate=1, n_out_peers=2, out_peers=ctypes.addressof(_GOOD_PEERS)), B.HRA_ERR_WORKSPACE),
])
def test_fused_output_fields_are_validated(over, status):
    """The fused tensor-parallel output (out_accumulate, out_peers) is checked before any
    launch; a well-formed one passes validation (and stops at the missing workspace)."""
    p = _fake_params(**over)
    rc = hra.load_library().mlra_decode(ctypes.byref(p), None)
    assert rc == status, hra.last_error()


def test_make_params_fills_the_peer_array():
    import torch
    q = torch.zeros(1, 4, 192, dtype=torch.bfloat16)
    cache = torch.zeros(64, 576, dtype=torch.bfloat16)
    w = torch.zeros(4, 512, 128, dtype=torch.bfloat16)
    out = torch.zeros(1, 4, 128)
    p = hra.make_params(q, cache[:, :512], cache[:, 512:], torch.zeros(1, dtype=torch.int32), w, w, out,
                        n_branch=4, out_accumulate=True, out_peers=[0x1000, 0x2000])
    assert p.out_accumulate == 1 and p.n_out_peers == 2
    assert list((ctypes.c_void_p * 2).from_address(p.out_peers)) == [0x1000, 0x2000]
    p0 = hra.make_params(q, cache[:, :512], cache[:, 512:], torch.zeros(1, dtype=torch.int32), w, w, out, n_branch=4)
    assert p0.out_accumulate == 0 and p0.n_out_peers == 0 and not p0.out_peers


def test_mla_decode_requires_one_branch():
    p = _fake_params(n_branch=4)
    with pytest.raises(hra.HraError) as e:
        hra.mla_decode(p, stream=0)
    assert e.value.status == B.HRA_ERR_INVALID_ARG


def test_workspace_size_zero_on_invalid():
    assert hra.load_library().hra_workspace_size(ctypes.byref(_fake_params(n_branch=5))) == 0


@pytest.mark.parametrize("over,status", [
    (dict(cache_dtype=B.HRA_INT8, n_branch=1, ckv_scale=0x90000, ckv_scale_stride=4), B.HRA_ERR_UNSUPPORTED),
    (dict(cache_dtype=B.HRA_INT8, ckv_scale=None, ckv_scale_stride=4), B.HRA_ERR_INVALID_ARG),
    (dict(cache_dtype=B.HRA_INT8, ckv_scale=0x90002, ckv_scale_stride=4), B.HRA_ERR_INVALID_ARG),  # misaligned
    (dict(cache_dtype=B.HRA_INT8, ckv_scale=0x90000, ckv_scale_stride=3), B.HRA_ERR_INVALID_ARG),
    (dict(cache_dtype=B.HRA_INT8, ckv_scale=0x90000, ckv_scale_stride=4, ckv_stride=584), B.HRA_ERR_INVALID_ARG),
    (dict(cache_dtype=5), B.HRA_ERR_INVALID_ARG),
    (dict(cache_dtype=B.HRA_INT8, ckv_scale=0x90000, ckv_scale_stride=4), B.HRA_ERR_WORKSPACE),
])
def test_int8_cache_fields_are_validated(over, status):
    """An int8 latent cache needs 128-wide branches, 4-byte aligned scales with a row stride
    of at least d_c / 128, and a 16-byte multiple row stride; a well-formed one passes
    validation (and stops at the missing workspace)."""
    p = _fake_params(**over)
    rc = hra.load_library().mlra_decode(ctypes.byref(p), None)
    assert rc == status, hra.last_error()


def test_make_params_selects_the_int8_cache():
    import torch
    q = torch.zeros(1, 4, 192, dtype=torch.bfloat16)
    ckv = torch.zeros(64, 512, dtype=torch.int8)
    krope = torch.zeros(64, 64, dtype=torch.bfloat16)
    scale = torch.ones(64, 4)
    w = torch.zeros(4, 512, 128, dtype=torch.bfloat16)
    out = torch.zeros(1, 4, 128)
    p = hra.make_params(q, ckv, krope, torch.zeros(1, dtype=torch.int32), w, w, out, n_branch=4, ckv_scale=scale)
    assert p.cache_dtype == B.HRA_INT8 and p.ckv_scale == scale.data_ptr() and p.ckv_scale_stride == 4
    assert p.ckv_stride == 512
    with pytest.raises(ValueError):
        hra.make_params(q, ckv, krope, torch.zeros(1, dtype=torch.int32), w, w, out, n_branch=4)


def test_static_entry_refuses_calls_beyond_its_array():
    """The allocation-free entry point's 32 MiB array holds up to 35 sequences at h = 128
    with d_c = 512 and 37 splits: B = 36 is refused before any device call; B = 35 passes
    the size check (and then needs a device, which this host does not have)."""
    big = _fake_params(batch=36, num_heads=128)
    assert hra.load_library().mlra_decode_static(ctypes.byref(big), None) == B.HRA_ERR_WORKSPACE
    assert "static array" in hra.last_error()
    fits = _fake_params(batch=35, num_heads=128)
    assert hra.load_library().mlra_decode_static(ctypes.byref(fits), None) != B.HRA_ERR_WORKSPACE
    bad = _fake_params(n_branch=3)
    assert hra.load_library().mlra_decode_static(ctypes.byref(bad), None) == B.HRA_ERR_UNSUPPORTED



def _fake_prefill(**over):
    """Well-formed prefill parameters with fake (aligned, never dereferenced) pointers."""
    p = B.HraPrefillParams()
    p.num_heads, p.n_branch = 16, 4
    p.d_c, p.d_rope, p.d_nope, p.d_v = 512, 64, 128, 128
    p.seq_len, p.n_query = 1000, 37
    p.q, p.ckv, p.krope, p.w_uk, p.w_uv, p.out = 0x10000, 0x20000, 0x20400, 0x40000, 0x50000, 0x60000
    p.ckv_stride, p.krope_stride = 576, 576
    p.alpha_q = p.alpha_kv = 1.0
    p.branch_scale, p.softmax_scale, p.rope_theta = 0.5, 0.0, 10000.0
    p.out_dtype = B.HRA_F32
    for k, v in over.items():
        setattr(p, k, v)
    return p


@pytest.mark.parametrize("over,status", [
    (dict(n_query=0), B.HRA_ERR_INVALID_ARG),
    (dict(n_query=1001), B.HRA_ERR_INVALID_ARG),          # more queries than cached tokens
    (dict(seq_len=0, n_query=0), B.HRA_ERR_UNSUPPORTED),
    (dict(n_branch=3), B.HRA_ERR_UNSUPPORTED),
    (dict(d_c=256), B.HRA_ERR_UNSUPPORTED),
    (dict(num_heads=129), B.HRA_ERR_UNSUPPORTED),
    (dict(q=0), B.HRA_ERR_INVALID_ARG),
    (dict(ckv=0x20008), B.HRA_ERR_INVALID_ARG),           # misaligned
    (dict(ckv_stride=500), B.HRA_ERR_INVALID_ARG),
    (dict(out_dtype=7), B.HRA_ERR_INVALID_ARG),
    (dict(), B.HRA_ERR_WORKSPACE),                        # well formed: stops at the missing workspace
    (dict(workspace=0x80010, workspace_bytes=1 << 40), B.HRA_ERR_WORKSPACE),  # not 256-aligned
])
def test_prefill_validation_rejects_before_launch(over, status):
    p = _fake_prefill(**over)
    rc = hra.load_library().mlra_prefill(ctypes.byref(p), None)
    assert rc == status, hra.last_error()


def test_prefill_workspace_size_formula():
    p = _fake_prefill()
    r = lambda x: -(-x // 256) * 256
    l_pad = 1024
    expect = 256
    expect = r(expect + 37 * 16 * 192 * 2)
    expect = r(expect + l_pad * 64 * 2)
    expect = r(expect + 4 * 16 * l_pad * 128 * 2)
    expect = r(expect + 4 * 16 * l_pad * 128 * 2)
    assert hra.prefill_workspace_size(p) == expect
    assert hra.load_library().hra_prefill_workspace_size(ctypes.byref(_fake_prefill(n_branch=5))) == 0


@pytest.mark.parametrize("over,status", [
    (dict(part_o=0xB0000), B.HRA_ERR_INVALID_ARG),                        # part_lse missing
    (dict(part_lse=0xC0000), B.HRA_ERR_INVALID_ARG),                      # part_o missing
    (dict(part_o=0xB0008, part_lse=0xC0000), B.HRA_ERR_INVALID_ARG),      # misaligned
    (dict(q_positions=0xD0002), B.HRA_ERR_INVALID_ARG),                   # misaligned
    (dict(part_o=0xB0000, part_lse=0xC0000, out=None), B.HRA_ERR_WORKSPACE),  # well formed: out unused
    (dict(q_positions=0xD0000), B.HRA_ERR_WORKSPACE),
])
def test_token_range_fields_are_validated(over, status):
    """The token-range mode of a split sequence (q_positions, part_o, part_lse) is checked
    before any launch; in it out may be NULL."""
    p = _fake_params(**over)
    rc = hra.load_library().mlra_decode(ctypes.byref(p), None)
    assert rc == status, hra.last_error()


@pytest.mark.parametrize("n_parts,parts_o,parts_lse,over,status", [
    (0, 0xB0000, 0xC0000, {}, B.HRA_ERR_INVALID_ARG),
    (65, 0xB0000, 0xC0000, {}, B.HRA_ERR_INVALID_ARG),
    (2, None, 0xC0000, {}, B.HRA_ERR_INVALID_ARG),
    (2, 0xB0004, 0xC0000, {}, B.HRA_ERR_INVALID_ARG),
    (2, 0xB0000, 0xC0000, dict(out=None), B.HRA_ERR_INVALID_ARG),         # the combine writes out
    (2, 0xB0000, 0xC0000, dict(part_o=0xB0000, part_lse=0xC0000), B.HRA_ERR_WORKSPACE),  # ignored
    (64, 0xB0000, 0xC0000, {}, B.HRA_ERR_WORKSPACE),                      # well formed: stops at the workspace
])
def test_combine_partials_is_validated(n_parts, parts_o, parts_lse, over, status):
    p = _fake_params(**over)
    lib = hra.load_library()
    rc = lib.hra_combine_partials(ctypes.byref(p), n_parts, parts_o, parts_lse, None)
    assert rc == status, hra.last_error()


def test_make_params_sets_the_token_range_fields():
    import torch
    q = torch.zeros(1, 4, 192, dtype=torch.bfloat16)
    cache = torch.zeros(64, 576, dtype=torch.bfloat16)
    w = torch.zeros(4, 512, 128, dtype=torch.bfloat16)
    pos = torch.tensor([99], dtype=torch.int32)
    po = torch.zeros(1, 4, 512)
    pl = torch.zeros(1, 4, 4)
    p = hra.make_params(q, cache[:, :512], cache[:, 512:], torch.tensor([64], dtype=torch.int32), w, w, None,
                        n_branch=4, q_positions=pos, part_o=po, part_lse=pl)
    assert (p.q_positions, p.part_o, p.part_lse) == (pos.data_ptr(), po.data_ptr(), pl.data_ptr())
    assert p.out is None
