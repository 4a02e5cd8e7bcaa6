"""Head-parallel layout of the SALAD layer over the ranks of a job.

The layer's (b, h) units are independent (each head has its own mask rows,
linear-branch state and output), so G ranks split the Hh heads into G
contiguous ranges and each runs its range with attn_forward_heads: no exchange
in the forward pass.  Where a consumer wants every head on every rank (a DiT's
output projection mixes heads), gather_heads assembles the full [B, N, Hh, d]
output from the ranks' ranges with one all-gather (NCCL over NVLink on GPUs,
any torch.distributed backend works).
"""
from __future__ import annotations

import torch


def head_ranges(num_heads: int, world: int) -> list[tuple[int, int]]:
    """(head_begin, head_count) of every rank: contiguous, in rank order,
    covering each head exactly once; counts differ by at most one (the first
    num_heads % world ranks take one more)."""
    if num_heads < 1 or world < 1:
        raise ValueError("num_heads and world must be positive")
    if world > num_heads:
        raise ValueError(f"{world} ranks for {num_heads} heads: some rank would have none")
    base, extra = divmod(num_heads, world)
    out, h = [], 0
    for r in range(world):
        c = base + (1 if r < extra else 0)
        out.append((h, c))
        h += c
    return out


def gather_heads(out: torch.Tensor, rank: int, world: int, group=None) -> torch.Tensor:
    """Every rank's range of heads of `out` ([B, N, Hh, d], this rank's range
    filled) into a full [B, N, Hh, d] tensor on every rank: each rank contributes
    its range as a contiguous [B, N, count, d] block (padded to the largest
    count so that one all_gather carries all of them)."""
    import torch.distributed as dist
    B, N, Hh, d = out.shape
    ranges = head_ranges(Hh, world)
    cmax = max(c for _, c in ranges)
    h0, c = ranges[rank]
    mine = torch.zeros(B, N, cmax, d, dtype=out.dtype, device=out.device)
    mine[:, :, :c] = out[:, :, h0:h0 + c]
    parts = [torch.empty_like(mine) for _ in range(world)]
    dist.all_gather(parts, mine, group=group)
    full = torch.empty_like(out)
    for r, (b0, cnt) in enumerate(ranges):
        full[:, :, b0:b0 + cnt] = parts[r][:, :, :cnt]
    return full
