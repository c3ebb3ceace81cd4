"""World-size-2 gloo run (CPU) of bench.py's multi-rank host logic: replica seeding and the
max-over-ranks timing reduction, with every rank taking the same collective steps."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import datetime
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from workload import configs
        wl = bench.replica_workload(configs.cfg2(), rank, world)
        t = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        seeds = [None] * world
        dist.all_gather_object(seeds, wl.seed)
        q.put((rank, t, seeds, wl.name))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_replicas():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert [r[1] for r in res] == [15.0, 15.0]         # max over ranks on every rank
    seeds = res[0][2]
    assert len(set(seeds)) == world                     # each replica decodes its own batch
    assert res[0][3] != res[1][3]


def test_single_rank_is_identity():
    import bench
    from workload import configs
    wl = configs.cfg2()
    assert bench.replica_workload(wl, 0, 1) is wl
    assert bench.max_over_ranks(3.5, 1) == 3.5
