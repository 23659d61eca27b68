"""mlra_decode_static: the decode for callers that cannot allocate device memory.

Some callers run inside another runtime's memory pool or on an allocation-free serving
path, or are plain C code without a device allocator; they cannot hand the library a
workspace.  mlra_decode_static takes its scratch from a fixed 32 MiB device array inside
the library instead.  These tests call it through the C ABI and compare its output with
mlra_decode (caller workspace) on two calls in a row, under the same parity bar as the
other GPU tests.  The file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import head_rank_attention_b200 as hra
import synth
from gpu_cases import MAX_REL, MEAN_REL, parity, run_gpu

pytestmark = pytest.mark.gpu


def _case(n_branch, lengths, page_size=0, heads=128):
    return synth.Workload("no_alloc", n_branch, len(lengths), heads, max(lengths), page_size=page_size,
                          lengths=tuple(lengths))


@pytest.mark.parametrize("wl", [_case(4, (700, 129, 64)), _case(4, (300, 1000), page_size=64),
                                _case(1, (513, 40)), _case(2, (257,), heads=16)],
                         ids=["mlra4", "mlra4_paged", "mla", "mlra2_h16"])
def test_static_matches_workspace_entry_point(wl):
    dev = synth.to_device(synth.make_inputs(wl))
    ref, p, _ = run_gpu(dev, wl)                      # mlra_decode with a caller workspace
    lib = hra.load_library()
    for _ in range(2):                                # two calls in a row share the array
        out = torch.full_like(ref, float("nan"))
        p.out = out.data_ptr()
        p.workspace, p.workspace_bytes = None, 0      # ignored by the static entry point
        rc = lib.mlra_decode_static(ctypes.byref(p), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert rc == 0, hra.last_error()
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        assert np.isfinite(got).all()
        max_rel, mean_rel = parity(got, ref.cpu().numpy().astype(np.float64))
        assert max_rel <= MAX_REL and mean_rel <= MEAN_REL, (max_rel, mean_rel)


def test_static_rejects_oversized_calls():
    """A batch whose scratch exceeds the fixed array is refused before any launch."""
    B, h = 256, 128
    q = torch.zeros(B, h, 192, dtype=torch.bfloat16, device="cuda")
    cache = torch.zeros(64, 576, dtype=torch.bfloat16, device="cuda")
    lens = torch.ones(B, dtype=torch.int32, device="cuda")
    w = torch.zeros(h, 512, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(B, h, 128, dtype=torch.float32, device="cuda")
    p = hra.make_params(q, cache[:, :512], cache[:, 512:], lens, w, w, out, n_branch=4, seq_stride=0)
    assert hra.workspace_size(p) > (32 << 20)
    rc = hra.load_library().mlra_decode_static(ctypes.byref(p), None)
    assert rc == hra._binding.HRA_ERR_WORKSPACE
    assert "static array" in hra.last_error()
