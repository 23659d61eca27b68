"""Seeded synthetic inputs for single-token latent-cache decode.

This module is shared by the tests, the benchmark and the smoke check: it is the
only code that both the fp64 oracle (``oracle/``) and the CUDA path see.  It holds
no attention arithmetic -- only shapes, seeds and random draws.

Every random tensor is drawn from torch's CPU generator, seeded per
(base seed, tensor id, sequence, row block) through a splitmix64 mix, in blocks of
``ROW_BLOCK`` cache rows.  Any row range of any sequence can therefore be
regenerated on its own, which lets the oracle re-create just the sequences it
samples.  Values are drawn in fp32 from N(0, 1) (weights N(0, 1/fan_in)) and
rounded once to bf16 (round-to-nearest-even); both sides consume the identical
bf16 bytes.

Workload shapes follow the five decode workloads of the latent-cache decode
study (MLA and MLRA in "Multi-Head Low-Rank Attention", sections 方法步骤详情 and
实验结果): d_c = 512 latent, d_R = 64 shared RoPE key, qk_nope = v_head = 128.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

D_C = 512       # latent width (kv_lora_rank)
D_ROPE = 64     # shared decoupled-RoPE key width (qk_rope_head_dim)
D_NOPE = 128    # per-head no-position query/key width (qk_nope_head_dim)
D_V = 128       # per-head value width (v_head_dim)
ROW = D_C + D_ROPE  # one cache row: [C_KV (512) | K_RoPE (64)]
ROW_BLOCK = 4096    # rows drawn per generator call

# tensor ids for seed derivation
_T_Q, _T_CACHE, _T_WUK, _T_WUV, _T_LENS, _T_PAGES, _T_OUTLIER = 1, 2, 4, 5, 6, 7, 8

_M64 = (1 << 64) - 1


def _splitmix64(x: int) -> int:
    x = (x + 0x9E3779B97F4A7C15) & _M64
    z = x
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def derive_seed(*parts: int) -> int:
    """Mix integers into one 63-bit seed (splitmix64 chain)."""
    h = 0
    for p in parts:
        h = _splitmix64(h ^ (int(p) & _M64))
    return h & ((1 << 63) - 1)


def _gen(*parts: int) -> torch.Generator:
    return torch.Generator().manual_seed(derive_seed(*parts))


@dataclasses.dataclass(frozen=True)
class Workload:
    """One decode workload: shapes, layout, scales and length distribution."""
    name: str
    n_branch: int                 # 1 = MLA, 2 = two-branch MLRA, 4 = MLRA-4
    batch: int
    heads: int
    seq_len: int                  # uniform length, or the upper end of a range
    seq_len_min: Optional[int] = None   # if set, lengths ~ U[seq_len_min, seq_len] (inclusive)
    page_size: int = 0            # 0 = contiguous [B, T_max, 576]; else pages of this many rows
    alpha_q: float = 1.0
    alpha_kv: float = 1.0
    branch_scale: Optional[float] = None  # None -> 1/sqrt(n_branch)
    outlier_frac: float = 0.0     # fraction of positions whose whole cache row is scaled x8
    rope_theta: float = 10000.0
    seed: int = 0
    lengths: Optional[tuple] = None  # explicit per-sequence lengths (overrides seq_len*)

    @property
    def sigma_o(self) -> float:
        return self.branch_scale if self.branch_scale is not None else 1.0 / math.sqrt(self.n_branch)

    @property
    def softmax_scale(self) -> float:
        # P5 (DeepseekV2Attention.__init__): scaling = (qk_nope + qk_rope) ** -0.5
        return 1.0 / math.sqrt(D_NOPE + D_ROPE)

    @property
    def fan_in(self) -> int:
        return D_C // self.n_branch

    def variant(self, n_branch: int, **kw) -> "Workload":
        return dataclasses.replace(self, n_branch=n_branch, branch_scale=None,
                                   name=f"{self.name}/{_VARIANT_NAMES[n_branch]}", **kw)


_VARIANT_NAMES = {1: "mla", 2: "mlra2", 4: "mlra4"}

# Scales for the 2.9B-model workload: d = h * d_h = 2048, d_c' = 1536 (q_lora_rank), d_c = 512.
_A_Q_2048 = math.sqrt(2048 / 1536)
_A_KV_2048 = math.sqrt(2048 / 512)
# DeepSeek-V3 widths (hidden 7168, q_lora_rank 1536, kv_lora_rank 512) for the stress scales.
A_Q_V3 = math.sqrt(7168 / 1536)
A_KV_V3 = math.sqrt(7168 / 512)

WORKLOADS = {
    # MLRA-4, B=1, h=16, T=2048, variance-correction scales, branch-sum scale 1/2
    "small_mlra4_h16_t2k": Workload("small_mlra4_h16_t2k", 4, 1, 16, 2048,
                                    alpha_q=_A_Q_2048, alpha_kv=_A_KV_2048, branch_scale=0.5),
    # MLA absorbed decode, DeepSeek-V3 attention shape, B=32, T=8192
    "mla_b32_t8k": Workload("mla_b32_t8k", 1, 32, 128, 8192),
    # MLRA-4 / 2-branch / MLA at B=64, T=32768, 64-token pages, random page table
    "paged_b64_t32k_mlra4": Workload("paged_b64_t32k_mlra4", 4, 64, 128, 32768, page_size=64),
    "paged_b64_t32k_mlra2": Workload("paged_b64_t32k_mlra2", 2, 64, 128, 32768, page_size=64),
    "paged_b64_t32k_mla": Workload("paged_b64_t32k_mla", 1, 64, 128, 32768, page_size=64),
    # MLRA-4 long context, B=4, lengths ~ U[65536, 131072]
    "long_mlra4_b4_t64k_128k": Workload("long_mlra4_b4_t64k_128k", 4, 4, 128, 131072, seq_len_min=65536),
    # the paged MLRA-4 layout at 1/8 of the batch (302 MB of cache, still larger than L2): the
    # size of a DRAM-traffic capture of the paged decode
    "paged_b8_t32k_mlra4": Workload("paged_b8_t32k_mlra4", 4, 8, 128, 32768, page_size=64),
    # MLRA-4 very long context, B=1, T=2^21, 1% of positions with key norms x8
    "vlong_mlra4_b1_t2m": Workload("vlong_mlra4_b1_t2m", 4, 1, 128, 2097152, outlier_frac=0.01),
}


def seq_lens(wl: Workload) -> np.ndarray:
    """Per-sequence lengths (int32 [B]); the query sits at position L-1."""
    if wl.lengths is not None:
        assert len(wl.lengths) == wl.batch
        return np.asarray(wl.lengths, dtype=np.int32)
    if wl.seq_len_min is None:
        return np.full(wl.batch, wl.seq_len, dtype=np.int32)
    g = _gen(wl.seed, _T_LENS)
    lens = torch.randint(wl.seq_len_min, wl.seq_len + 1, (wl.batch,), generator=g, dtype=torch.int64)
    return lens.numpy().astype(np.int32)


def _row_block(wl: Workload, s: int, blk: int) -> torch.Tensor:
    """Rows [blk*ROW_BLOCK, (blk+1)*ROW_BLOCK) of sequence s, fp32 before rounding."""
    x = torch.randn(ROW_BLOCK, ROW, generator=_gen(wl.seed, _T_CACHE, s, blk))
    if wl.outlier_frac > 0.0:
        u = torch.rand(ROW_BLOCK, generator=_gen(wl.seed, _T_OUTLIER, s, blk))
        x[u < wl.outlier_frac] *= 8.0
    return x


def seq_rows(wl: Workload, s: int, t0: int = 0, t1: Optional[int] = None) -> torch.Tensor:
    """Logical cache rows [t0, t1) of sequence s as bf16 [t1-t0, 576] = [C_KV | K_RoPE].

    K_RoPE is drawn as already-rotated values (iid Gaussian pairs are rotation
    invariant in distribution), so no rotation is applied to the cache.
    """
    L = int(seq_lens(wl)[s])
    t1 = L if t1 is None else min(t1, L)
    out = torch.empty(max(t1 - t0, 0), ROW, dtype=torch.bfloat16)
    t = t0
    while t < t1:
        blk = t // ROW_BLOCK
        b0 = blk * ROW_BLOCK
        b1 = min(b0 + ROW_BLOCK, t1)
        rows = _row_block(wl, s, blk)[t - b0:b1 - b0]
        out[t - t0:b1 - t0] = rows.to(torch.bfloat16)
        t = b1
    return out


def page_table(wl: Workload) -> Optional[np.ndarray]:
    """int32 [B, max_pages]: a seeded random permutation of the page pool, or None."""
    if wl.page_size == 0:
        return None
    lens = seq_lens(wl)
    max_pages = max(1, int(-(-int(lens.max()) // wl.page_size)))
    n_pages = wl.batch * max_pages
    perm = torch.randperm(n_pages, generator=_gen(wl.seed, _T_PAGES)).numpy().astype(np.int32)
    return perm.reshape(wl.batch, max_pages)


@dataclasses.dataclass
class Inputs:
    """Host-side inputs for one decode step (all torch CPU tensors)."""
    q: torch.Tensor            # bf16 [B, h, 192]: q_nope (128) | q_rope (64, not yet rotated)
    cache: torch.Tensor        # bf16 [rows, 576]: physical cache rows [C_KV | K_RoPE]
    seq_lens: torch.Tensor     # int32 [B]
    block_table: Optional[torch.Tensor]  # int32 [B, max_pages] or None
    seq_stride: int            # rows between sequences (contiguous layout), 0 for paged
    w_uk: torch.Tensor         # bf16 [h, 512, 128]
    w_uv: torch.Tensor         # bf16 [h, 512, 128]


def weights(wl: Workload):
    """W_UK, W_UV bf16 [h, 512, 128] ~ N(0, 1/fan_in), fan_in = branch width 512/n_branch."""
    std = 1.0 / math.sqrt(wl.fan_in)
    w_uk = (torch.randn(wl.heads, D_C, D_NOPE, generator=_gen(wl.seed, _T_WUK)) * std).to(torch.bfloat16)
    w_uv = (torch.randn(wl.heads, D_C, D_V, generator=_gen(wl.seed, _T_WUV)) * std).to(torch.bfloat16)
    return w_uk, w_uv


def queries(wl: Workload) -> torch.Tensor:
    return torch.randn(wl.batch, wl.heads, D_NOPE + D_ROPE, generator=_gen(wl.seed, _T_Q)).to(torch.bfloat16)


def make_inputs(wl: Workload, with_cache: bool = True) -> Inputs:
    """Build every input of one decode step on the host.

    Contiguous layout: physical row of (s, t) is s * T_max + t.
    Paged layout: physical row of (s, t) is block_table[s, t // P] * P + t % P.
    """
    lens = seq_lens(wl)
    bt = page_table(wl)
    w_uk, w_uv = weights(wl)
    q = queries(wl)
    t_max = max(1, int(lens.max()))
    if bt is None:
        rows, seq_stride = wl.batch * t_max, t_max
    else:
        rows, seq_stride = bt.size * wl.page_size, 0
    cache = torch.zeros(rows if with_cache else 0, ROW, dtype=torch.bfloat16)
    if with_cache:
        for s in range(wl.batch):
            L = int(lens[s])
            r = seq_rows(wl, s)
            if bt is None:
                cache[s * t_max:s * t_max + L] = r
            else:
                P = wl.page_size
                for p in range(-(-L // P)):
                    n = min(P, L - p * P)
                    dst = int(bt[s, p]) * P
                    cache[dst:dst + n] = r[p * P:p * P + n]
    return Inputs(q=q, cache=cache, seq_lens=torch.from_numpy(lens),
                  block_table=None if bt is None else torch.from_numpy(bt),
                  seq_stride=seq_stride, w_uk=w_uk, w_uv=w_uv)


def logical_rows(inp: Inputs, wl: Workload, s: int) -> torch.Tensor:
    """Gather sequence s's logical rows back out of the physical cache."""
    L = int(inp.seq_lens[s])
    if inp.block_table is None:
        return inp.cache[s * inp.seq_stride:s * inp.seq_stride + L]
    P = wl.page_size
    idx = torch.arange(L)
    phys = inp.block_table[s, idx // P].to(torch.int64) * P + idx % P
    return inp.cache[phys]


def quantize_int8_blocks(latent: torch.Tensor, block: int = 128):
    """An int8 copy of a latent cache, as a caller would write it: for every row and
    128-column block, scale = max|x| / 127 (fp32) and q = round-to-nearest-even(x / scale)
    (0 where the block is all zero).  Returns (q int8 [rows, d], scale fp32 [rows, d / block]).

    This is the cache format, not decode arithmetic: the decode (and the oracle) only read
    it back as q * scale."""
    x = latent.to(torch.float32)
    rows, d = x.shape
    xb = x.view(rows, d // block, block)
    amax = xb.abs().amax(dim=2)
    scale = amax / 127.0
    safe = torch.where(scale > 0, scale, torch.ones_like(scale))
    q = torch.round(xb / safe[:, :, None]).clamp_(-127, 127)
    q = torch.where(scale[:, :, None] > 0, q, torch.zeros_like(q))
    return q.to(torch.int8).view(rows, d), scale.contiguous()


def kv_bytes(lens) -> int:
    """Algorithmic KV-cache bytes one decode step reads: 576 bf16 per cached token."""
    return int(np.asarray(lens, dtype=np.int64).sum()) * ROW * 2


@dataclasses.dataclass
class DeviceInputs:
    """Inputs copied to one device (same bytes as the host copy)."""
    q: torch.Tensor
    cache: torch.Tensor
    seq_lens: torch.Tensor
    block_table: Optional[torch.Tensor]
    seq_stride: int
    w_uk: torch.Tensor
    w_uv: torch.Tensor

    @property
    def ckv(self) -> torch.Tensor:
        return self.cache[:, :D_C]

    @property
    def krope(self) -> torch.Tensor:
        return self.cache[:, D_C:]


def to_device(inp: Inputs, device="cuda") -> DeviceInputs:
    """Copy every input tensor to `device` unchanged."""
    bt = None if inp.block_table is None else inp.block_table.to(device)
    return DeviceInputs(q=inp.q.to(device), cache=inp.cache.to(device), seq_lens=inp.seq_lens.to(device),
                        block_table=bt, seq_stride=inp.seq_stride, w_uk=inp.w_uk.to(device),
                        w_uv=inp.w_uv.to(device))
