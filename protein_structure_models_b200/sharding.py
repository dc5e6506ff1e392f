"""Partition of the fused IPA forward across ranks (one process per GPU).

Page "Invariant point attention (IPA)", Required behavior: every output row of
sample b is a function of that row's query, its frame and all keys of the same
sample.  So samples are independent, and within a sample the query rows are
independent once every rank holds all keys.  Neither split needs a collective
on the data path; the only collectives are the timing barrier and the max of
the per-rank step times.

batch_shards  -- contiguous sample ranges (batches of many short chains)
tile_shards   -- contiguous ranges of 128-residue query tiles, balanced by the
                 number of tiles holding a valid residue (long chains)
max_over_ranks -- the slowest rank's time, the job's step time
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

TILE = 128   # residues per query tile of the core kernel


def batch_shards(B: int, world: int) -> List[Tuple[int, int]]:
    """Split samples 0..B-1 into `world` contiguous ranges whose sizes differ by
    at most one (the first B % world ranges take the extra sample)."""
    if B < 0 or world <= 0:
        raise ValueError("B must be >= 0 and world > 0")
    base, extra = divmod(B, world)
    out, start = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append((start, start + n))
        start += n
    return out


def tile_weights(mask_row: Sequence[bool], tile: int = TILE) -> List[int]:
    """1 for a query tile holding at least one valid residue, else 0 (fully
    masked tiles produce only zero rows and cost nothing)."""
    n = len(mask_row)
    return [1 if any(mask_row[t:min(t + tile, n)]) else 0 for t in range(0, n, tile)]


def tile_shards(weights: Sequence[int], world: int) -> List[Tuple[int, int]]:
    """Split tiles 0..T-1 into `world` contiguous ranges with balanced total
    weight: range r ends at the first tile where the running weight reaches
    (r + 1) / world of the total.  Zero-weight tiles go with the range they
    follow; with no weight at all the tiles are split evenly by count.  With at
    least as many tiles as ranks every range gets at least one tile."""
    T = len(weights)
    if world <= 0:
        raise ValueError("world must be > 0")
    total = sum(weights)
    if total == 0:
        return batch_shards(T, world)
    out, start, acc, t = [], 0, 0, 0
    for r in range(world):
        if r == world - 1:
            out.append((start, T))
            break
        goal = total * (r + 1) / world
        left = world - 1 - r                      # ranges after this one
        while t < T - left and acc + weights[t] <= goal:
            acc += weights[t]
            t += 1
        if t == start and t < T - left:           # never empty while tiles suffice
            acc += weights[t]
            t += 1
        out.append((start, t))
        start = t
    return out


def tile_rows(tiles: Tuple[int, int], N: int, tile: int = TILE) -> Tuple[int, int]:
    """Query rows [start, stop) covered by a tile range."""
    return min(tiles[0] * tile, N), min(tiles[1] * tile, N)


def max_over_ranks(x: float, device=None) -> float:
    """Maximum of `x` over all ranks of the default process group (x itself
    when torch.distributed is not initialised).  `device` is where the
    reduction tensor lives: a CUDA device under NCCL, None (CPU) under gloo."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
