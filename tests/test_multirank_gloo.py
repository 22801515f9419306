"""The N > 1 path of bench.py on CPU: two gloo ranks pick disjoint planned
owner shares (no collective on the data path) and agree on the max-over-ranks
timing reduction."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    import datetime
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    from synth import workload
    wl = workload("7b_share")
    planned, mats, owns_tail, flops = bench.planned_share(wl.params, wl.world_size, rank,
                                                         bench.product_plan, bench.product_heaviest)
    t = bench.max_over_ranks(float(10 + rank))
    out[rank] = (planned, sorted(p.pid for p in mats), owns_tail, flops, t)
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_take_disjoint_shares():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    (p0, m0, t0, f0, x0), (p1, m1, t1, f1, x1) = res[0], res[1]
    assert p0 != p1
    assert not set(m0) & set(m1)
    assert len(m0) == len(m1) == 28
    assert f0 == f1                      # the 7B plan is balanced
    assert t0 != t1 and (t0 or t1)       # exactly one rank owns the tail
    assert x0 == x1 == 11.0              # max over ranks


def test_single_rank_max_is_identity():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
