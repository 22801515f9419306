"""Pins of the owner-planner oracle: hand-worked plans and invariants."""

import itertools
import random
from collections import Counter

import pytest

from oracle import heaviest_rank, plan_owners
from oracle.plan import ns_flops, resident_bytes
from synth.workloads import ParamSpec, MATRIX, TAIL, workload


def mat(pid, r, c, dtype="bf16"):
    return ParamSpec(pid, f"m{pid}", r, c, MATRIX, dtype)


def test_cost_model_hand_values():
    # 4096^2: 5 (4 * 4096^3 + 2 * 4096^3) = 30 * 4096^3
    assert ns_flops(4096, 4096) == 30 * 4096 ** 3
    # 11008 x 4096 is transposed: r = 4096, c = 11008
    assert ns_flops(11008, 4096) == 5 * (4 * 4096 ** 2 * 11008 + 2 * 4096 ** 3)
    assert ns_flops(4096, 11008) == ns_flops(11008, 4096)
    assert resident_bytes(10, 20, MATRIX, "bf16") == 200 * 8
    assert resident_bytes(10, 20, MATRIX, "f32") == 200 * 12
    assert resident_bytes(100, 1, TAIL, "f32") == 1600


def test_hand_worked_three_matrix_plan():
    # f(4096^2) = 8 f(2048^2), b(4096^2) = 4 b(2048^2); Fbar = 5 f2, Bbar = 3 b2.
    # 4096 first: both ranks score max(8/5, 4/3) = 1.6 -> rank 0 (lowest id).
    # first 2048: rank 0 scores max(9/5, 5/3) = 1.8, rank 1 max(1/5, 1/3) -> rank 1.
    # second 2048: rank 0 1.8, rank 1 max(2/5, 2/3) -> rank 1.
    params = [mat(0, 2048, 2048), mat(1, 4096, 4096), mat(2, 2048, 2048)]
    entries, F, B = plan_owners(params, 2)
    assert [e.owner for e in entries] == [1, 0, 1]
    assert F == [ns_flops(4096, 4096), 2 * ns_flops(2048, 2048)]
    # rank 1 holds pids 0 and 2 in id order
    assert entries[0].owner_offset == 0 and entries[2].owner_offset == 2048 * 2048
    assert entries[1].owner_offset == 0
    assert heaviest_rank(F, B) == 0


def test_hand_worked_tail_placement_and_ties():
    # Two equal matrices on two ranks: the first to rank 0, the second to rank 1
    # (rank 0 would score 2.0).  The tail goes to the rank with fewer bytes:
    # equal bytes -> rank 0.  Heaviest: equal F, rank 0 has more bytes.
    params = [mat(0, 64, 128), mat(1, 64, 128),
              ParamSpec(2, "n1", 100, 1, TAIL, "f32"), ParamSpec(3, "n2", 50, 1, TAIL, "f32")]
    entries, F, B = plan_owners(params, 2)
    assert [e.owner for e in entries] == [0, 1, 0, 0]
    assert entries[2].owner_offset == 0 and entries[3].owner_offset == 100
    assert B[0] == B[1] + 150 * 16
    assert heaviest_rank(F, B) == 0
    assert not entries[0].transposed and entries[0].shape_scale == 1.0


def test_transposed_flag_and_scale():
    entries, _, _ = plan_owners([mat(0, 256, 64), mat(1, 64, 256), mat(2, 64, 64)], 1)
    assert [e.transposed for e in entries] == [True, False, False]
    assert entries[0].shape_scale == 2.0 and entries[1].shape_scale == 1.0


@pytest.mark.parametrize("R", [1, 2, 3, 5])
def test_every_parameter_owned_once_and_deterministic(R):
    rnd = random.Random(R)
    params = [mat(i, 64 * rnd.randint(1, 8), 64 * rnd.randint(1, 8)) for i in range(17)]
    params.append(ParamSpec(17, "tail", 1000, 1, TAIL, "f32"))
    e1, F1, B1 = plan_owners(params, R)
    shuffled = params[:]
    rnd.shuffle(shuffled)
    e2, F2, B2 = plan_owners(shuffled, R)
    own1 = {e.pid: e.owner for e in e1}
    own2 = {e.pid: e.owner for e in e2}
    assert own1 == own2 and F1 == F2 and B1 == B2
    assert all(0 <= o < R for o in own1.values())
    assert sum(F1) == sum(ns_flops(p.rows, p.cols) for p in params if p.kind == MATRIX)
    assert sum(B1) == sum(e.resident_bytes for e in e1)


def test_brute_force_makespan_identical_items():
    # With identical items the greedy deals them round-robin; its FLOP makespan
    # equals the optimum found by enumerating every assignment.
    params = [mat(i, 256, 256) for i in range(7)]
    entries, F, B = plan_owners(params, 3)
    assert sorted(Counter(e.owner for e in entries).values()) == [2, 2, 3]
    best = min(max(sum(ns_flops(256, 256) for j, o in enumerate(a) if o == r) for r in range(3))
               for a in itertools.product(range(3), repeat=7))
    assert max(F) == best


def test_llama_share_plans_are_balanced():
    # 7B: 224 matrices = 8 x (16 square 4096^2, 8 of 11008x4096, 4 of 4096x11008):
    # every rank gets the same NS FLOPs (85.56e12); rank 0 also takes the tail.
    wl = workload("7b_share")
    entries, F, B = plan_owners(wl.params, 8)
    assert len(set(F)) == 1 and abs(F[0] - 85.55574853632e12) < 1.0
    h = heaviest_rank(F, B)
    assert h == 0
    share = Counter((e.rows, e.cols) for e in entries if e.owner == h and e.kind == MATRIX)
    assert share == Counter({(4096, 4096): 16, (11008, 4096): 8, (4096, 11008): 4})
    assert all(e.owner == h for e in entries if e.kind == TAIL)
    # 32B over 64 ranks: 7 matrices per rank, equal FLOPs.
    wl = workload("32b_share")
    entries, F, B = plan_owners(wl.params, 64)
    assert len(set(F)) == 1
    h = heaviest_rank(F, B)
    share = Counter((e.rows, e.cols) for e in entries if e.owner == h and e.kind == MATRIX)
    assert share == Counter({(27648, 5120): 2, (5120, 27648): 1, (5120, 5120): 2, (1024, 5120): 2})
