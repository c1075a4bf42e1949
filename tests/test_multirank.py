"""Multi-rank host logic of bench.py on CPU with gloo (world size 2).

Every rank solves its own layer set (weak scaling, no collective on the data path); the
only collectives are the barrier and the max-over-ranks reduction of the timed region.
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
