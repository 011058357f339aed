"""Key-range split of one long sequence's cache over G processes (one per
device), the multi-device variant of the decode step: each process holds a
contiguous share of every ring's slots, produces the partial (m, l, o) of its
share with `rswa_decode_step_partial`, the partials are all-gathered, and
`rswa_combine_partials` merges them by log-sum-exp.  Only the partials cross
devices: G x B x H x (d + 2) floats per layer and step.

This module holds the host side: how the prompt is cut into shares, and the
exchange (torch.distributed; NCCL on GPUs, gloo on CPU).
"""
from __future__ import annotations

from typing import List, Tuple

import torch


def share_bounds(prefill_len: int, shares: int) -> List[Tuple[int, int]]:
    """Contiguous prompt slices [lo, hi) of near-equal length, one per share;
    the ring (slots P .. P + W) belongs to the last share."""
    if shares < 1 or prefill_len < 0:
        raise ValueError("shares >= 1 and prefill_len >= 0")
    base, extra = divmod(prefill_len, shares)
    out, lo = [], 0
    for g in range(shares):
        hi = lo + base + (1 if g < extra else 0)
        out.append((lo, hi))
        lo = hi
    return out


def gather_partials(part_ml: torch.Tensor, part_o: torch.Tensor, group=None):
    """All-gather this rank's partial (m, l) [B, H, 2] and o [B, H, d] into
    [G, B, H, 2] and [G, B, H, d], rank order (the merge does not depend on
    the order, but a fixed order keeps the result reproducible)."""
    import torch.distributed as dist
    G = dist.get_world_size(group)
    ml = [torch.empty_like(part_ml) for _ in range(G)]
    o = [torch.empty_like(part_o) for _ in range(G)]
    dist.all_gather(ml, part_ml.contiguous(), group=group)
    dist.all_gather(o, part_o.contiguous(), group=group)
    return torch.stack(ml), torch.stack(o)
