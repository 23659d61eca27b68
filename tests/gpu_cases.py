"""Shared helpers for the GPU tests: run the CUDA path through the C ABI on synth inputs
and compare with the fp64 oracle under the parity bar."""
from __future__ import annotations

import numpy as np
import torch

import head_rank_attention_b200 as hra
import synth

# Parity bar for floating-point outputs: bf16 inputs, fp32 accumulation.
MAX_REL = 1e-2      # max|g - r| <= MAX_REL * max|r|
MEAN_REL = 2e-3     # sum|g - r| / sum|r| <= MEAN_REL


def run_gpu(dev: synth.DeviceInputs, wl: synth.Workload, *, out_dtype=torch.float32, num_splits: int = 0,
            api: str = "mlra", workspace=None, poison: bool = True):
    B, h = dev.q.shape[0], dev.q.shape[1]
    out = torch.empty(B, h, synth.D_V, dtype=out_dtype, device=dev.q.device)
    p = hra.make_params(dev.q, dev.ckv, dev.krope, dev.seq_lens, dev.w_uk, dev.w_uv, out,
                        n_branch=wl.n_branch, alpha_q=wl.alpha_q, alpha_kv=wl.alpha_kv,
                        branch_scale=wl.sigma_o, softmax_scale=wl.softmax_scale, rope_theta=wl.rope_theta,
                        block_table=dev.block_table, page_size=wl.page_size, seq_stride=dev.seq_stride,
                        num_splits=num_splits)
    ws = hra.alloc_workspace(p) if workspace is None else workspace
    if workspace is not None:
        p.workspace, p.workspace_bytes = ws.data_ptr(), ws.numel()
    if poison:  # NaN bytes everywhere: any read of a slot the call did not write shows up
        ws.fill_(0xFF)
    (hra.mla_decode if api == "mla" else hra.mlra_decode)(p)
    hra.check_device_status(p)
    return out, p, ws


def parity(got: np.ndarray, ref: np.ndarray):
    err = np.abs(got.astype(np.float64) - ref)
    max_rel = err.max() / np.abs(ref).max()
    mean_rel = err.sum() / np.abs(ref).sum()
    return float(max_rel), float(mean_rel)


def assert_parity(got: np.ndarray, ref: np.ndarray, what: str = ""):
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    max_rel, mean_rel = parity(got, ref)
    assert max_rel <= MAX_REL and mean_rel <= MEAN_REL, f"{what}: max_rel={max_rel:.3e} mean_rel={mean_rel:.3e}"
    return max_rel, mean_rel
