"""Decode attention over a context sharded by position across ranks.

You Only Cache Once (abstract) scales the single cache to 1M tokens, more than
one GPU holds.  Each rank keeps a contiguous slice of every sequence's cached
positions in its own cache (local positions 0..n_r-1).  One decode step is:

  1. every rank: yocopp_decode_attn_partial over its slice -> unnormalised
     (o, m, l) per (sequence, query head), base-2 logits;
  2. one all-gather of those partials (batch * heads * (d + 2) fp32 per rank,
     tiny next to the slice's KV bytes) over NCCL;
  3. every rank: yocopp_decode_combine -> the full attention output.

The exchange is the only collective; the arithmetic is in the kernels.
"""
from __future__ import annotations

from typing import Callable, Optional, Tuple

import torch

from . import yocopp_decode_attn_partial, yocopp_decode_combine


def shard_bounds(length: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous, near-equal slice [start, end) of `length` positions owned by `rank`."""
    base, extra = divmod(length, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def local_lengths(lens, world: int, rank: int):
    """Per-sequence count of positions in this rank's slice."""
    out = []
    for t in lens:
        a, b = shard_bounds(int(t), world, rank)
        out.append(b - a)
    return out


def seq_shard_decode(q: torch.Tensor, cache, local_lens: torch.Tensor, out: torch.Tensor, workspace: torch.Tensor,
                     group=None, scale: float = 0.0,
                     partial_fn: Optional[Callable] = None, combine_fn: Optional[Callable] = None) -> torch.Tensor:
    """Full decode attention for q [B][Hq][d] whose keys/values are split across the ranks
    of `group` (this rank's slice in `cache`, lengths `local_lens`).  `partial_fn` /
    `combine_fn` default to the CUDA entry points."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    B, hq, d = q.shape
    partial = torch.empty((B, hq, d + 2), dtype=torch.float32, device=q.device)
    if partial_fn is None:
        yocopp_decode_attn_partial(q, cache, local_lens, partial, workspace, hq, scale)
    else:
        partial_fn(q, cache, local_lens, partial)
    flat = torch.empty((world * B, hq, d + 2), dtype=torch.float32, device=q.device)
    dist.all_gather_into_tensor(flat, partial, group=group)
    gathered = flat.view(world, B, hq, d + 2)
    if combine_fn is None:
        yocopp_decode_combine(gathered, out)
    else:
        combine_fn(gathered, out)
    return out
