"""The multi-rank plumbing of bench.py, as world-size-2 gloo processes on CPU.

Each rank runs its own tower (weak scaling, no data-path collective); timing is
the max over ranks.  Nothing here touches a GPU.
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
    import workloads
    from datetime import timedelta
    dist.init_process_group("gloo", timeout=timedelta(seconds=60))
    r, w, lr = bench.rank_info()
    seed = bench.rank_base_seed(r)
    cases = workloads.tower_cases(8, seed)          # tiny 8x8 grid: host-side structure only
    elapsed = 10.0 + 5.0 * r                          # stand-in for a per-rank device time
    mx = bench.max_over_ranks(elapsed, dist, "cpu")
    seeds = [None] * w
    dist.all_gather_object(seeds, [c.seed for c in cases])
    dist.barrier()
    dist.destroy_process_group()
    q.put((r, w, lr, mx, seeds))


def test_two_gloo_ranks_weak_scaling_plumbing():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    for r, w, lr, mx, seeds in out:
        assert w == 2 and lr == r
        assert mx == 15.0                      # max over ranks, identical on every rank
        assert seeds[0] != seeds[1]            # independent images per rank
        assert seeds[0][0] == 0 and seeds[1][0] == 1000


def test_single_process_helpers():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.rank_base_seed(0) == 0 and bench.rank_base_seed(3) == 3000
