"""Tensor parallelism by branch for MLRA decode.

"Multi-Head Low-Rank Attention" (核心方法) splits the latent head into branches that are
attended to independently and summed, so that under 4-way tensor parallelism each
device holds one branch: its 128 latent columns of the cache, a copy of the shared
K_RoPE, and the matching rows of W_UK and W_UV (the per-device loading row of the
table under 实验结果: 1.5 d_h per token instead of MLA's 4.5 d_h).

A device's share is an ordinary call of the library with d_c = 128 * (branches held)
and the full model's branch_scale; its output is that shard's part of the branch sum,
and one all-reduce (sum) over the tensor-parallel group gives the model's output.  This
module lays the cache and weights out per shard and does that all-reduce; the decode
itself runs in libhra.so.

The same layout serves MLRA-2 split by branch over 2 ranks (n_branch=2: one 256-wide
branch per rank, a d_c = 256, n_branch = 1 call) and the latent side of a GLA-2 rank
(研究动机: MLA's latent split into two groups; the rank also holds only its group's heads,
and the ranks' outputs are concatenated over heads instead of summed).
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch

__all__ = ["shard_columns", "shard_cache", "shard_weights", "all_reduce_out", "peer_ranks", "PeerOut"]


def shard_columns(d_c: int, n_branch: int, rank: int, world: int) -> Tuple[int, int]:
    """Latent columns [c0, c1) that rank `rank` of `world` holds: n_branch / world whole
    branches of width d_c / n_branch, in branch order."""
    if world < 1 or n_branch % world != 0 or d_c % n_branch != 0:
        raise ValueError(f"cannot split {n_branch} branches of a {d_c}-wide latent over {world} ranks")
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside [0, {world})")
    width = (d_c // n_branch) * (n_branch // world)
    return rank * width, (rank + 1) * width


def shard_cache(cache: torch.Tensor, rank: int, world: int, n_branch: int = 4, d_c: int = 512) -> torch.Tensor:
    """Rank `rank`'s cache rows, [rows, c1 - c0 + d_rope]: its latent columns then K_RoPE
    (a new contiguous tensor on cache's device; row indices and the block table are kept).
    Pass the result as the call's fused cache: ckv = [:, :c1-c0], krope = [:, c1-c0:]."""
    c0, c1 = shard_columns(d_c, n_branch, rank, world)
    return torch.cat([cache[:, c0:c1], cache[:, d_c:]], dim=1).contiguous()


def shard_weights(w_uk: torch.Tensor, w_uv: torch.Tensor, rank: int, world: int,
                  n_branch: int = 4) -> Tuple[torch.Tensor, torch.Tensor]:
    """Rank `rank`'s rows of W_UK and W_UV ([h, d_c, 128] each): [h, c1 - c0, 128]."""
    c0, c1 = shard_columns(int(w_uk.shape[1]), n_branch, rank, world)
    return w_uk[:, c0:c1].contiguous(), w_uv[:, c0:c1].contiguous()


def peer_ranks(rank: int, world: int) -> list:
    """The ranks whose out buffers a rank's up-projection adds into besides its own, in
    rank order (the order of hra_decode_params.out_peers)."""
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside [0, {world})")
    return [r for r in range(world) if r != rank]


class PeerOut:
    """Out buffers for the fused up-projection + all-reduce of a branch-sharded decode.

    Every rank allocates its fp32 out [B, h, d_v] in symmetric memory (peer-mapped over
    NVLink) and learns the addresses of the other ranks' buffers.  A step is then

        po.begin()                    # zero this rank's out; barrier: every out is zeroed
        p = make_params(..., out=po.out, out_accumulate=True, out_peers=po.peers)
        mlra_decode(p)                # adds this shard's part into every rank's out
        po.end()                      # barrier: every rank's additions have landed

    after which po.out holds the sum over the shards on every rank.  The barriers are
    torch's symmetric-memory device barriers on the current stream (bounded by
    timeout_ms), so no host synchronisation sits in the step.
    """

    def __init__(self, shape, group=None, device=None, timeout_ms: int = 10000):
        import torch.distributed as dist
        import torch.distributed._symmetric_memory as symm_mem
        group = dist.group.WORLD if group is None else group
        self.out = symm_mem.empty(*shape, dtype=torch.float32, device=device)
        self.handle = symm_mem.rendezvous(self.out, group)
        self.rank, self.world = int(self.handle.rank), int(self.handle.world_size)
        ptrs = list(self.handle.buffer_ptrs)
        self.peers = [int(ptrs[r]) for r in peer_ranks(self.rank, self.world)]
        self.timeout_ms = int(timeout_ms)

    def begin(self) -> None:
        self.out.zero_()
        self.handle.barrier(channel=0, timeout_ms=self.timeout_ms)

    def end(self) -> torch.Tensor:
        self.handle.barrier(channel=1, timeout_ms=self.timeout_ms)
        return self.out


def all_reduce_out(out: torch.Tensor, group: Optional[object] = None) -> torch.Tensor:
    """Sum the shards' partial outputs in place over the tensor-parallel group (NCCL for
    device tensors).  Use an fp32 `out` so that the sum is not rounded per shard."""
    import torch.distributed as dist
    dist.all_reduce(out, op=dist.ReduceOp.SUM, group=group)
    return out
