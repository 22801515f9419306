"""Checkpoint resharding across world sizes, driven by mfsdp_reshard's routes
over real process-to-process transfers: three gloo ranks on CPU restore the
state two saved ranks held.  Ranks 0 and 1 hold the saved layout's owner-local
buffers; every rank ends up with the buffers of the three-rank layout, moved by
send/recv for each route whose owner rank changes, and checks every parameter
it now owns against the value it was saved with."""

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

OLD_WORLD, NEW_WORLD = 2, 3


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _params():
    """The block workload's parameter list with every side divided by 32, so
    that the buffers stay small while the plan keeps its structure."""
    from synth import workload
    from synth.workloads import ParamSpec
    wl = workload("block")
    return [ParamSpec(p.pid, p.name, max(1, p.rows // 32), max(1, p.cols // 32), p.kind, p.dtype)
            for p in wl.params]


def _value(pid, n):
    # the saved state of parameter pid: distinct per parameter and element
    return (pid * 1000003 + np.arange(n, dtype=np.float64)).astype(np.float32)


def _buffers(params, shards, world, rank, fill):
    """This rank's owner-local buffers (matrix state, packed tail state) for a layout."""
    mat_len = tail_len = 0
    for p, s in zip(params, shards):
        if s.owner != rank:
            continue
        n = p.rows * p.cols
        if s.kind == 0:
            mat_len = max(mat_len, s.owner_offset + n)
        else:
            tail_len = max(tail_len, s.owner_offset + n)
    mb, tb = np.zeros(mat_len, np.float32), np.zeros(tail_len, np.float32)
    if fill:
        for p, s in zip(params, shards):
            if s.owner == rank:
                (mb if s.kind == 0 else tb)[s.owner_offset:s.owner_offset + p.rows * p.cols] = \
                    _value(p.pid, p.rows * p.cols)
    return mb, tb


def _worker(rank, port, out):
    import sys
    import datetime
    import torch
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=NEW_WORLD, timeout=datetime.timedelta(seconds=60))
    from matrix_optimizer_step_nesterov_b200 import _lib
    params = _params()
    descs = [(p.rows, p.cols, p.kind, 1 if p.dtype == "bf16" else 0) for p in params]
    saved, _, _ = _lib.mfsdp_plan(descs, OLD_WORLD)
    shards, routes, moved = _lib.mfsdp_reshard(descs, saved, NEW_WORLD)
    old = _buffers(params, saved, OLD_WORLD, rank, fill=rank < OLD_WORLD)
    new = _buffers(params, shards, NEW_WORLD, rank, fill=False)
    sent = 0
    # every rank walks the routes in the same order; only the two ranks of a route act
    for r in routes:
        k = 0 if r.kind == 0 else 1
        if r.src_rank == r.dst_rank == rank:
            new[k][r.dst_offset:r.dst_offset + r.elems] = old[k][r.src_offset:r.src_offset + r.elems]
        elif rank == r.src_rank:
            dist.send(torch.from_numpy(old[k][r.src_offset:r.src_offset + r.elems].copy()), dst=r.dst_rank)
            sent += r.elems
        elif rank == r.dst_rank:
            buf = torch.empty(r.elems, dtype=torch.float32)
            dist.recv(buf, src=r.src_rank)
            new[k][r.dst_offset:r.dst_offset + r.elems] = buf.numpy()
    ok = True
    owned = 0
    for p, s in zip(params, shards):
        if s.owner != rank:
            continue
        n = p.rows * p.cols
        got = new[0 if s.kind == 0 else 1][s.owner_offset:s.owner_offset + n]
        ok = ok and np.array_equal(got, _value(p.pid, n))
        owned += 1
    out[rank] = (ok, owned, sent, moved)
    dist.barrier()
    dist.destroy_process_group()


def test_three_ranks_restore_a_two_rank_checkpoint():
    from matrix_optimizer_step_nesterov_b200 import build
    build.build()
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, port, out)) for r in range(NEW_WORLD)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(180)
            assert p.exitcode == 0
        res = dict(out)
    assert all(res[r][0] for r in range(NEW_WORLD)), res
    assert sum(res[r][1] for r in range(NEW_WORLD)) == len(_params())   # every parameter owned once
    assert sum(res[r][2] for r in range(NEW_WORLD)) > 0                 # some state crossed ranks
    assert len({res[r][3] for r in range(NEW_WORLD)}) == 1              # all ranks computed one plan
