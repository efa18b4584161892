"""Multi-rank sharding on CPU (gloo, world size 2): every image is taken by exactly one rank, the
ranks agree on the assignment without exchanging it, row offsets stay batch-global, and the load
is balanced within the LPT bound."""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import workloads
from vision_lm_image_b200 import build, shard


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, sizes, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        H = [h for h, _ in sizes]
        W = [w for _, w in sizes]
        assign, grid, offs = shard.shard_plan(H, W, world)
        mine = assign[rank]
        gathered = [None] * world
        dist.all_gather_object(gathered, (rank, mine, offs.tolist()))
        q.put(gathered if rank == 0 else None)
    finally:
        dist.destroy_process_group()


def test_lpt_two_ranks_gloo():
    build.build()
    rng = workloads.rng_for(99)
    sizes = workloads.random_sizes(rng, 37) + [(16, 192), (4096, 4096), (1080, 1920)]
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, sizes, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = None
    for _ in range(world):
        item = q.get(timeout=120)
        if item is not None:
            res = item
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res is not None
    sets = [set(m) for _, m, _ in res]
    assert sets[0].isdisjoint(sets[1])
    assert sets[0] | sets[1] == set(range(len(sizes)))
    assert res[0][2] == res[1][2]  # identical global row offsets on both ranks
    offs = np.array(res[0][2])
    rows = np.diff(offs)
    loads = [int(rows[list(s)].sum()) for s in sets]
    assert max(loads) - min(loads) <= rows.max()  # LPT: imbalance below the largest item


def test_lpt_properties():
    rng = np.random.Generator(np.random.PCG64(3))
    for world in (1, 2, 3, 8):
        costs = rng.integers(1, 1000, size=50).tolist()
        a = shard.lpt_assign(costs, world)
        flat = sorted(i for part in a for i in part)
        assert flat == list(range(50))
        loads = [sum(costs[i] for i in part) for part in a]
        assert max(loads) <= sum(costs) / world + max(costs)
    assert shard.lpt_assign([], 4) == [[], [], [], []]
    with pytest.raises(ValueError):
        shard.lpt_assign([1], 0)


def _window_worker(rank, world, port, sizes, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        windows, grid, offs = shard.window_plan([h for h, _ in sizes], [w for _, w in sizes], world)
        first, count = windows[rank]
        gathered = [None] * world
        dist.all_gather_object(gathered, (rank, first, count, offs.tolist(),
                                          shard.window_images(offs, first, count)))
        q.put(gathered if rank == 0 else None)
    finally:
        dist.destroy_process_group()


def _run_ranks(target, world, sizes):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, sizes, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = None
    for _ in range(world):
        item = q.get(timeout=120)
        if item is not None:
            res = item
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


@pytest.mark.parametrize("sizes", [[(4096, 4096)], [(1080, 1920), (4096, 4096), (16, 192), (640, 480)]])
def test_unit_windows_two_ranks_gloo(sizes):
    # one huge image (or a batch dominated by one): the two ranks split it by merge-block ranges
    build.build()
    world = 2
    res = _run_ranks(_window_worker, world, sizes)
    assert res is not None and res[0][3] == res[1][3]
    units = res[0][3][-1] // 4
    covered = np.zeros(units, np.int64)
    for _, first, count, _, _ in res:
        covered[first:first + count] += 1
    assert (covered == 1).all()  # every merge unit exactly once
    counts = [c for _, _, c, _, _ in res]
    assert max(counts) - min(counts) <= 1  # balanced within one merge unit
    # the largest image is shared between the ranks
    offs = np.array(res[0][3])
    big = int(np.argmax(np.diff(offs)))
    assert all(big in imgs for *_, imgs in res)


def test_unit_windows_properties():
    for total in (0, 1, 7, 8100, 522240):
        for world in (1, 2, 3, 8):
            w = shard.unit_windows(total, world)
            assert w[0][0] == 0 and sum(c for _, c in w) == total
            assert all(w[r][0] + w[r][1] == w[r + 1][0] for r in range(world - 1))
            assert max(c for _, c in w) - min(c for _, c in w) <= 1
    with pytest.raises(ValueError):
        shard.unit_windows(5, 0)


def _gather_worker(rank, world, port, units, q):
    import torch

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        windows = shard.unit_windows(units, world)
        first, count = windows[rank]
        # stand-in rows: row r of the batch holds r in every column
        rows = torch.arange(4 * first, 4 * (first + count), dtype=torch.float32).repeat_interleave(6).view(-1, 6)
        out = shard.gather_windows(rows, windows, dst=0)
        q.put(None if out is None else out.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,units", [(2, 8100), (3, 7)])
def test_gather_windows_reassembles_the_batch_gloo(world, units):
    res = _run_ranks(_gather_worker, world, units)
    # _run_ranks keeps the one result that is not None: rank 0's gathered rows
    assert res is not None and res.shape == (4 * units, 6)
    assert np.array_equal(res[:, 0], np.arange(4 * units, dtype=np.float32))
    assert (res == res[:, :1]).all()
