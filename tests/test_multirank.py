"""Multi-rank host logic of bench.py on CPU with gloo (world size 2).

Two ways to use N GPUs, neither with a collective on the data path: every rank solves its
own layer set (weak scaling), or the ranks split ONE layer set by matrix (bench.py --split;
calibration_free_dual_b200/shard.py). The only collectives are the barrier and the
max-over-ranks reduction of the timed region. Checked here: the reduction, disjoint seeds,
and the split (every matrix assigned exactly once, ranks within one largest matrix of each
other, and rank-local oracle solves gathered on rank 0 equal to one rank solving the whole
small layer set).
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import workloads as wl
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world)
        bench.barrier(world)
        mx = bench.reduce_max(10.0 + rank, world)           # each rank's elapsed ms
        # per-rank layer sets: same shapes, different seeds
        cfg = wl.CONFIGS[3]
        seeds = [wl.seed_of(cfg.cid, b, p) + 1_000_000 * rank for b, p, _, _ in cfg.layer_set()]
        gathered = [None] * world
        dist.all_gather_object(gathered, seeds[:5])
        q.put((rank, mx, gathered))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def _split_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import numpy as np
    import workloads as wl
    from calibration_free_dual_b200.shard import assign
    from oracle import formats as F
    from oracle import solver as S
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world)
        layer = _small_layer()
        parts = assign([m * n for _, _, m, n in layer], world)
        mine = {}
        for i in parts[rank]:
            W = _small_matrix(layer[i])
            o = S.solve(W, F.make_format("MXFP4"), 4)
            mine[i] = (o["codes"], o["r_codes"], o["c"], o["mse"])
        gathered = [None] * world
        dist.all_gather_object(gathered, mine)
        q.put((rank, parts, gathered))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def _small_layer():
    """A small layer set of mixed shapes (block, proj, m, n)."""
    shapes = [(64, 128), (32, 128), (32, 128), (64, 128), (160, 128), (160, 128), (64, 320)]
    return [(b, p, m, n) for b in range(3) for p, (m, n) in enumerate(shapes)]


def _small_matrix(entry):
    import numpy as np
    b, p, m, n = entry
    rng = np.random.default_rng(100 * b + p)
    w = rng.standard_t(4, (m, n)) * 0.02
    w[:, rng.choice(n, 2, replace=False)] *= 8.0
    return w.astype(np.float32).astype(np.float64)


def test_layer_set_split_over_ranks():
    import numpy as np
    from calibration_free_dual_b200.shard import assign, loads
    from oracle import formats as F
    from oracle import solver as S
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_split_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    layer = _small_layer()
    sizes = [m * n for _, _, m, n in layer]
    parts = res[0][1]
    assert all(r[1] == parts for r in res)                   # every rank agrees
    flat = sorted(i for part in parts for i in part)
    assert flat == list(range(len(layer)))                  # each matrix exactly once
    ld = loads(sizes, parts)
    assert max(ld) - min(ld) <= max(sizes)                  # within one largest matrix
    merged = {}
    for d in res[0][2]:
        assert not set(d) & set(merged)
        merged.update(d)
    for i, entry in enumerate(layer):                        # = one rank solving everything
        o = S.solve(_small_matrix(entry), F.make_format("MXFP4"), 4)
        codes, rc, c, mse = merged[i]
        np.testing.assert_array_equal(codes, o["codes"])
        np.testing.assert_array_equal(rc, o["r_codes"])
        np.testing.assert_array_equal(c, o["c"])
        np.testing.assert_array_equal(mse, o["mse"])


def test_assignment_rule():
    """Largest first, each to the least-loaded rank (ties: lowest rank); every split of a
    layer set is exhaustive, disjoint and balanced within one largest matrix."""
    from calibration_free_dual_b200.shard import assign, loads
    import workloads as wl
    assert assign([5, 3, 3, 1], 2) == [[0, 3], [1, 2]]
    assert assign([4, 4, 4], 4) == [[0], [1], [2], []]
    for cid in (2, 3, 4):
        sizes = [m * n for _, _, m, n in wl.CONFIGS[cid].layer_set()]
        for world in (1, 2, 3, 4, 8):
            parts = assign(sizes, world)
            assert sorted(i for p in parts for i in p) == list(range(len(sizes)))
            ld = loads(sizes, parts)
            assert max(ld) - min(ld) <= max(sizes)
    with pytest.raises(ValueError):
        assign([1, 2], 0)


def test_max_over_ranks_and_disjoint_seeds():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, gathered in res:
        assert mx == 11.0                                    # the slowest rank's time
        assert set(gathered[0]).isdisjoint(gathered[1])      # independent problems per rank
