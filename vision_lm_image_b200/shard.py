"""Data-parallel sharding of a preprocessing batch across ranks (one process per GPU).

Images are independent and every output row has exactly one producer, so the
path needs no exchange step: each rank runs the fused kernel on its own
images. This module only decides which images a rank takes. Images go to
ranks by longest-processing-time-first greedy assignment, with the cost of an
image taken as its output bytes (resized pixels; the kernel is bound by HBM
writes). Ties break by image index and then by rank, so every rank computes
the same assignment from the same sizes without communicating.

The batch plan (image_grid_thw, row offsets) stays global: a rank's rows for
image i are rows [row_offsets[i], row_offsets[i+1]) of the batch, so shards
can be reassembled, or consumed in place, without renumbering.

Whole images bound the balance of that assignment by the largest image. The
second plan cuts the batch's merge units instead (unit u = batch rows
4u..4u+3 in merge order) into one contiguous window per rank, equal up to a
single unit: an image larger than a rank's share is split by merge-block
ranges, and each rank runs one mimo_preprocess_units call on its window.
"""
from __future__ import annotations

import heapq
from typing import Sequence

import numpy as np

from . import mimo


def lpt_assign(costs: Sequence[int], world: int) -> list[list[int]]:
    """Greedy LPT: images by decreasing cost, each to the currently least-loaded rank."""
    if world <= 0:
        raise ValueError("world must be positive")
    order = sorted(range(len(costs)), key=lambda i: (-int(costs[i]), i))
    heap = [(0, r) for r in range(world)]
    out: list[list[int]] = [[] for _ in range(world)]
    for i in order:
        load, r = heapq.heappop(heap)
        out[r].append(i)
        heapq.heappush(heap, (load + int(costs[i]), r))
    for r in range(world):
        out[r].sort()
    return out


def shard_plan(heights: Sequence[int], widths: Sequence[int], world: int, params=None):
    """Returns (assignment per rank, grid_thw [n, 3], row_offsets [n + 1]) for a batch."""
    grid, offs = mimo.plan_batch(heights, widths, params)
    rows = np.diff(offs)
    return lpt_assign(rows.tolist(), world), grid, offs


def rank_images(images, rank: int, world: int, params=None):
    """The images (in batch order) that ``rank`` processes, with their batch indices."""
    heights = [int(im.shape[0]) for im in images]
    widths = [int(im.shape[1]) for im in images]
    assign, grid, offs = shard_plan(heights, widths, world, params)
    mine = assign[rank]
    return [images[i] for i in mine], mine, grid, offs


def unit_windows(total_units: int, world: int) -> list[tuple[int, int]]:
    """Contiguous merge-unit windows (first_unit, unit_count), one per rank, tiling [0, total_units) with
    counts that differ by at most one."""
    if world <= 0:
        raise ValueError("world must be positive")
    if total_units < 0:
        raise ValueError("total_units must be non-negative")
    bounds = [r * total_units // world for r in range(world + 1)]
    return [(bounds[r], bounds[r + 1] - bounds[r]) for r in range(world)]


def window_plan(heights: Sequence[int], widths: Sequence[int], world: int, params=None):
    """Returns (windows per rank, grid_thw [n, 3], row_offsets [n + 1]) for a batch cut by merge units."""
    grid, offs = mimo.plan_batch(heights, widths, params)
    return unit_windows(int(offs[-1]) // 4, world), grid, offs


def window_images(offs, first_unit: int, unit_count: int) -> list[int]:
    """Batch indices of the images a window touches (whole or in part)."""
    lo, hi = 4 * first_unit, 4 * (first_unit + unit_count)
    return [i for i in range(len(offs) - 1) if offs[i] < hi and offs[i + 1] > lo]


def gather_windows(local_rows, windows: Sequence[tuple[int, int]], dst: int = 0, group=None, out=None):
    """Collects every rank's window rows on rank ``dst`` in batch row order.

    Each rank passes the rows of its own merge-unit window (``local_rows``: [4 * count, cols], as written by
    mimo_preprocess_units) and the shared window plan. Rank ``dst`` receives the other windows with one
    grouped batch of point-to-point transfers (NCCL send/recv over NVLink for CUDA tensors) straight into
    the matching row ranges of ``out`` ([total_rows, cols], allocated when not given) and returns it; the
    other ranks send theirs and return None. No collective touches the data path before this call."""
    import torch
    import torch.distributed as dist

    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    if len(windows) != world:
        raise ValueError("one window per rank")
    first, count = windows[rank]
    if local_rows.shape[0] != 4 * count:
        raise ValueError(f"rank {rank} holds {local_rows.shape[0]} rows for a window of {count} merge units")
    total = 4 * (windows[-1][0] + windows[-1][1])
    if rank != dst:
        if count:
            dist.send(local_rows.contiguous(), dst=dist.get_global_rank(group, dst) if group else dst, group=group)
        return None
    if out is None:
        out = torch.empty((total,) + tuple(local_rows.shape[1:]), dtype=local_rows.dtype, device=local_rows.device)
    out[4 * first:4 * (first + count)].copy_(local_rows)
    ops = []
    for r, (f, c) in enumerate(windows):
        if r == dst or c == 0:
            continue
        src = dist.get_global_rank(group, r) if group else r
        ops.append(dist.P2POp(dist.irecv, out[4 * f:4 * (f + c)], src, group))
    for w in dist.batch_isend_irecv(ops) if ops else []:
        w.wait()
    return out
