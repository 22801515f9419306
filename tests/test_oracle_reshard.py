"""Pins of the owner-shard checkpoint resharding oracle.

The data-level pins build each saved rank's owner-local buffers from the saved
layout, move every parameter's state by its route, and read every parameter
back from the new ranks' buffers through the new layout alone.
"""

import numpy as np
import pytest

from oracle import plan_owners, reshard, state_bytes
from oracle.plan import MATRIX as PMATRIX, TAIL as PTAIL
from synth.workloads import ParamSpec, MATRIX, TAIL, workload


def mat(pid, r, c, dtype="bf16"):
    return ParamSpec(pid, f"m{pid}", r, c, MATRIX, dtype)


def tail(pid, n):
    return ParamSpec(pid, f"t{pid}", n, 1, TAIL, "f32")


def test_state_bytes_hand_values():
    assert state_bytes(10, 20, PMATRIX, "bf16") == 200 * (2 + 4)
    assert state_bytes(10, 20, PMATRIX, "f32") == 200 * (4 + 4)
    assert state_bytes(100, 1, PTAIL, "f32") == 100 * 12


def test_hand_worked_one_to_two_ranks():
    # World 1: everything on rank 0, matrices packed in id order, tail packed.
    # World 2 (the three-matrix plan worked by hand in test_oracle_plan):
    # 4096^2 -> rank 0; both 2048^2 -> rank 1; the tail goes to the rank with
    # fewer bytes: rank 1 holds 2 * 2048^2 * 8 B < 4096^2 * 8 B -> rank 1.
    params = [mat(0, 2048, 2048), mat(1, 4096, 4096), mat(2, 2048, 2048), tail(3, 100)]
    old, _, _ = plan_owners(params, 1)
    new, routes, moved = reshard(params, old, 2)
    assert [r.src_rank for r in routes] == [0, 0, 0, 0]
    assert [r.dst_rank for r in routes] == [1, 0, 1, 1]
    assert [r.src_offset for r in routes] == [0, 2048 * 2048, 2048 * 2048 + 4096 * 4096, 0]
    assert [r.dst_offset for r in routes] == [0, 0, 2048 * 2048, 0]
    # pids 0, 2 and the tail change rank
    assert moved == 2 * 2048 * 2048 * 6 + 100 * 12
    assert [e.owner for e in new] == [r.dst_rank for r in routes]


@pytest.mark.parametrize("name,old_w,new_w", [("7b_share", 8, 16), ("7b_share", 8, 3), ("32b_share", 64, 48),
                                              ("block", 1, 4), ("skew", 4, 7)])
def test_same_world_is_identity_and_round_trip(name, old_w, new_w):
    wl = workload(name)
    old, _, _ = plan_owners(wl.params, old_w)
    same, routes, moved = reshard(wl.params, old, old_w)
    assert same == old and moved == 0
    assert all(r.src_rank == r.dst_rank and r.src_offset == r.dst_offset for r in routes)
    mid, _, _ = reshard(wl.params, old, new_w)
    back, _, _ = reshard(wl.params, mid, old_w)
    assert back == old


def _saved_buffers(params, entries, world, seed=0):
    """Each rank's owner-local buffers (matrix state, packed tail state),
    filled with per-parameter values, and the values themselves."""
    rng = np.random.default_rng(seed)
    vals = {p.pid: rng.standard_normal(p.rows * p.cols) for p in params}
    mat_len = [0] * world
    tail_len = [0] * world
    for p, e in zip(params, entries):
        n = p.rows * p.cols
        if e.kind == PMATRIX:
            mat_len[e.owner] = max(mat_len[e.owner], e.owner_offset + n)
        else:
            tail_len[e.owner] = max(tail_len[e.owner], e.owner_offset + n)
    bufs = [(np.full(mat_len[r], np.nan), np.full(tail_len[r], np.nan)) for r in range(world)]
    for p, e in zip(params, entries):
        n = p.rows * p.cols
        bufs[e.owner][0 if e.kind == PMATRIX else 1][e.owner_offset:e.owner_offset + n] = vals[p.pid]
    return bufs, vals


@pytest.mark.parametrize("name,old_w,new_w", [("7b_share", 8, 5), ("block", 2, 3), ("skew", 3, 8),
                                              ("tiny", 1, 2)])
def test_routes_move_every_state_to_where_the_new_layout_reads_it(name, old_w, new_w):
    wl = workload(name)
    if name in ("7b_share",):
        # keep the arrays small: same parameter list with tiny shapes keeps the plan's structure
        params = [ParamSpec(p.pid, p.name, max(1, p.rows // 256), max(1, p.cols // 256), p.kind, p.dtype)
                  for p in wl.params]
    elif name == "skew":
        params = [ParamSpec(p.pid, p.name, max(1, p.rows // 64), max(1, p.cols // 64), p.kind, p.dtype)
                  for p in wl.params]
    else:
        params = list(wl.params)
    old, _, _ = plan_owners(params, old_w)
    bufs, vals = _saved_buffers(params, old, old_w)
    new, routes, moved = reshard(params, old, new_w)
    # the new ranks' buffers, sized from the new layout alone
    mat_len = [0] * new_w
    tail_len = [0] * new_w
    for p, e in zip(params, new):
        n = p.rows * p.cols
        if e.kind == PMATRIX:
            mat_len[e.owner] = max(mat_len[e.owner], e.owner_offset + n)
        else:
            tail_len[e.owner] = max(tail_len[e.owner], e.owner_offset + n)
    nbufs = [(np.full(mat_len[r], np.nan), np.full(tail_len[r], np.nan)) for r in range(new_w)]
    for rt in routes:
        k = 0 if rt.kind == PMATRIX else 1
        nbufs[rt.dst_rank][k][rt.dst_offset:rt.dst_offset + rt.elems] = \
            bufs[rt.src_rank][k][rt.src_offset:rt.src_offset + rt.elems]
    for p, e in zip(params, new):
        n = p.rows * p.cols
        got = nbufs[e.owner][0 if e.kind == PMATRIX else 1][e.owner_offset:e.owner_offset + n]
        np.testing.assert_array_equal(got, vals[p.pid])
    # every slot of every new buffer was filled: the new layout packs without gaps
    for mb, tb in nbufs:
        assert not np.isnan(mb).any() and not np.isnan(tb).any()
    assert moved == sum(state_bytes(p.rows, p.cols, e.kind, p.dtype if e.kind == PMATRIX else "f32")
                        for p, e, o in zip(params, new, old) if e.owner != o.owner)


def test_reshard_rejects_a_layout_of_other_parameters():
    params = [mat(0, 64, 64), mat(1, 32, 64)]
    old, _, _ = plan_owners(params, 2)
    with pytest.raises(ValueError):
        reshard([mat(0, 64, 64), mat(1, 64, 32)], old, 3)
    with pytest.raises(ValueError):
        reshard(params[:1], old, 3)
