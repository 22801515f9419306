"""The pages' equivalence invariant, pinned on the fp64 oracle.

Under owner-shaped ZeRO-3 placement the ordinary backward reduction lands the
full gradient of a 2D weight on its one owner; the owner runs the whole-matrix
update locally and the other ranks hold empty shards ("MatrixFSDP:
communication-free matrix optimizers under ZeRO-3 parameter sharding",
arxivlens summary page, Abstract; gist.science French summary, Methodologie
section 1: the owner receives exactly the full gradient and updates with no
optimizer-step communication).  Two consequences are checked bit for bit:

* the owner's step on R data-parallel ranks' gradient contributions, summed
  in rank order into the owner segment, equals the step on the gradient the
  ranks would all-reduce (summed in the same order);
* stepping every planned rank's share separately and putting the results back
  together equals the unsharded update of the whole parameter list.

The packed non-matrix tail (arxivlens Abstract: tail owners stay on AdamW) is
checked the same way: AdamW on the packed buffer equals AdamW per tensor.
"""

import numpy as np
import pytest

import oracle
from oracle import AdamWHParams, MuonHParams
from synth.workloads import MATRIX, TAIL, ParamSpec

HP = MuonHParams()
R = 3


def _model():
    shapes = [(48, 80), (80, 48), (64, 64), (16, 96), (96, 16), (33, 70), (70, 33), (1, 40), (40, 1), (57, 57)]
    params = [ParamSpec(i, f"w{i}", r, c, MATRIX, "f32") for i, (r, c) in enumerate(shapes)]
    params += [ParamSpec(len(shapes) + k, f"n{k}", n, 1, TAIL, "f32", "norm") for k, n in enumerate((64, 17, 80))]
    return params


def _rank_grads(rng, shape):
    """One gradient contribution per data-parallel rank, on its own scale."""
    return [rng.standard_normal(shape) * 10.0 ** rng.uniform(-4, -2) for _ in range(R)]


def _sum_in_rank_order(parts):
    g = parts[0].copy()
    for p in parts[1:]:
        g = g + p
    return g


@pytest.mark.parametrize("shape", [(20, 30), (30, 20), (25, 25), (1, 7)])
@pytest.mark.parametrize("nparts", [1, 2, 5])
def test_owner_step_on_contributions_equals_full_gradient_step(shape, nparts):
    rng = np.random.default_rng(nparts * 100 + shape[0])
    W = rng.standard_normal(shape) * 0.02
    buf = rng.standard_normal(shape) * 1e-3
    parts = [rng.standard_normal(shape) * 1e-3 for _ in range(nparts)]
    owner = oracle.muon_step_parts(W, parts, buf, HP)
    full = oracle.muon_step(W, _sum_in_rank_order(parts), buf, HP)
    for x, y in zip(owner, full):
        assert np.array_equal(x, y)


def test_planned_shares_equal_the_unsharded_update():
    rng = np.random.default_rng(2024)
    params = _model()
    mats = [p for p in params if p.kind == MATRIX]
    W = {p.pid: rng.standard_normal((p.rows, p.cols)) * 0.02 for p in mats}
    buf = {p.pid: rng.standard_normal((p.rows, p.cols)) * 1e-3 for p in mats}
    grads = {p.pid: _rank_grads(rng, (p.rows, p.cols)) for p in mats}

    # unsharded: every rank all-reduces every gradient, then the whole list is updated at once
    Wu, Ou, bu = oracle.muon_step_list([W[p.pid] for p in mats], [_sum_in_rank_order(grads[p.pid]) for p in mats],
                                       [buf[p.pid] for p in mats], HP)
    unsharded = {p.pid: (Wu[k], Ou[k], bu[k]) for k, p in enumerate(mats)}

    # owner-shaped: each matrix has one planned owner, which alone receives the
    # ranks' contributions (in rank order) and steps its share
    entries, F, B = oracle.plan_owners(params, R)
    owner_of = {e.pid: e.owner for e in entries}
    got = {}
    for q in range(R):
        share = [p for p in mats if owner_of[p.pid] == q]
        for p in share:
            assert p.pid not in got, "a matrix stepped by two owners"
            got[p.pid] = oracle.muon_step_parts(W[p.pid], grads[p.pid], buf[p.pid], HP)
    assert sorted(got) == sorted(p.pid for p in mats), "every matrix is stepped by exactly one owner"
    for pid, res in got.items():
        for x, y in zip(res, unsharded[pid]):
            assert np.array_equal(x, y), pid

    # the share-by-share list steps (one call per rank) agree too
    for q in range(R):
        share = [p for p in mats if owner_of[p.pid] == q]
        if not share:
            continue
        Ws, Os, bs = oracle.muon_step_list([W[p.pid] for p in share],
                                           [_sum_in_rank_order(grads[p.pid]) for p in share],
                                           [buf[p.pid] for p in share], HP)
        for k, p in enumerate(share):
            assert np.array_equal(Ws[k], unsharded[p.pid][0])
            assert np.array_equal(Os[k], unsharded[p.pid][1])
            assert np.array_equal(bs[k], unsharded[p.pid][2])


def test_packed_tail_adamw_equals_per_tensor_adamw():
    rng = np.random.default_rng(7)
    params = _model()
    entries, _, _ = oracle.plan_owners(params, R)
    tails = [(p, e) for p, e in zip(params, entries) if p.kind == TAIL]
    owners = {e.owner for _, e in tails}
    assert len(owners) == 1, "the whole tail is one unit on one owner"
    n = sum(p.numel for p, _ in tails)
    packed = {k: np.zeros(n) for k in "pgmv"}
    per = {}
    for p, e in tails:
        vals = {"p": 1.0 + 0.01 * rng.standard_normal(p.numel), "g": rng.standard_normal(p.numel) * 1e-3,
                "m": rng.standard_normal(p.numel) * 1e-4, "v": np.abs(rng.standard_normal(p.numel)) * 1e-7}
        per[p.pid] = vals
        for k in "pgmv":
            packed[k][e.owner_offset:e.owner_offset + p.numel] = vals[k]
    hp = AdamWHParams()
    pn, mn, vn = oracle.adamw_step(packed["p"], packed["g"], packed["m"], packed["v"], 4, hp)
    for p, e in tails:
        v = per[p.pid]
        rp, rm, rv = oracle.adamw_step(v["p"], v["g"], v["m"], v["v"], 4, hp)
        sl = slice(e.owner_offset, e.owner_offset + p.numel)
        assert np.array_equal(pn[sl], rp) and np.array_equal(mn[sl], rm) and np.array_equal(vn[sl], rv)
