"""One sequence split across devices by token range (context parallelism) for decode.

The softmax of a decode step is over all of a sequence's cached tokens, but its
denominator is a sum over tokens, so a sequence can be cut into contiguous token ranges
held by different devices.  Each device decodes its range as if it were the whole
sequence, with the query rotated at the sequence's real last position
(``q_positions``), and stops after the split-KV merge: for every (sequence, head,
128-column slice of the latent) it writes the softmax-weighted latent row over its
tokens, normalised, and the log2 of that range's softmax denominator (``part_o``,
``part_lse``).  The devices all-gather those states, and each then finishes the decode
with ``combine_partials``: the states are merged by their log-sum-exp and go through
the up-projection and branch sum.  Over NVSwitch the exchange is one small all-gather
(h * d_c fp32 values and h * d_c / 128 lse values per sequence and device).

This module cuts the ranges and does the all-gather; the decode and the merge run in
libhra.so.
"""
from __future__ import annotations

from typing import Optional, Sequence, Tuple

import torch

__all__ = ["token_range", "token_ranges", "gather_partials"]


def token_range(length: int, rank: int, world: int) -> Tuple[int, int]:
    """Tokens [a, b) of a sequence of `length` tokens held by rank `rank` of `world`:
    contiguous ranges whose sizes differ by at most one (empty when length < world)."""
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    return length * rank // world, length * (rank + 1) // world


def token_ranges(lengths: Sequence[int], rank: int, world: int) -> Tuple[list, list]:
    """Per sequence: the first token and the number of tokens rank `rank` holds."""
    starts, counts = [], []
    for n in lengths:
        a, b = token_range(int(n), rank, world)
        starts.append(a)
        counts.append(b - a)
    return starts, counts


def gather_partials(part_o: torch.Tensor, part_lse: torch.Tensor,
                    group: Optional[object] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """All-gather every rank's partial state (NCCL for device tensors): returns
    ([world, B, h, d_c], [world, B, h, d_c / 128]) in rank order, the layout
    ``combine_partials`` takes."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    # gathered along the first dimension (rank r's rows follow rank r - 1's), then viewed
    # with a leading rank index
    out_o = torch.empty((world * part_o.shape[0],) + tuple(part_o.shape[1:]), dtype=part_o.dtype, device=part_o.device)
    out_l = torch.empty((world * part_lse.shape[0],) + tuple(part_lse.shape[1:]), dtype=part_lse.dtype,
                        device=part_lse.device)
    dist.all_gather_into_tensor(out_o, part_o.contiguous(), group=group)
    dist.all_gather_into_tensor(out_l, part_lse.contiguous(), group=group)
    return out_o.view((world,) + tuple(part_o.shape)), out_l.view((world,) + tuple(part_lse.shape))
