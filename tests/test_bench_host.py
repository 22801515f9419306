"""Host-side helpers of bench.py (no GPU): the e2e group split, the planner
balance field and the Newton-Schulz FLOP counts behind the roofline."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402
from synth.workloads import workload  # noqa: E402


def _specs(name):
    return workload(name).matrices


@pytest.mark.parametrize("name", ["tiny", "block", "7b_share", "skew"])
@pytest.mark.parametrize("n_groups", [1, 2, 3, 6, 8])
def test_split_groups_covers_every_matrix_once(name, n_groups):
    specs = _specs(name)
    groups = bench.split_groups(specs, n_groups)
    flat = [i for g in groups for i in g]
    assert sorted(flat) == list(range(len(specs)))
    assert all(groups) and len(groups) <= max(1, n_groups)


def test_split_groups_puts_the_two_smallest_matrices_at_the_ends():
    specs = _specs("7b_share")
    groups = bench.split_groups(specs, 6)
    costs = [bench.ns_flops_dense([s]) for s in specs]
    smallest = sorted(range(len(specs)), key=lambda i: (costs[i], i))[:2]
    assert groups[0] == [smallest[0]] and groups[-1] == [smallest[1]]
    # the middle groups carry about equal work: none above twice the mean
    middle = [sum(costs[i] for i in g) for g in groups[1:-1]]
    assert max(middle) <= 2.0 * sum(middle) / len(middle)


def test_ns_flop_counts_match_their_closed_forms():
    class S:
        def __init__(self, rows, cols):
            self.rows, self.cols = rows, cols

    # square r x r: per iteration r^2 c + r^3 + 2 r^2 c = 4 r^3 algorithmic, 4 r^3 + 2 r^3 dense
    assert bench.ns_flops_algorithmic([S(512, 512)]) == 5 * 4.0 * 512 ** 3
    assert bench.ns_flops_dense([S(512, 512)]) == 5 * 6.0 * 512 ** 3
    # orientation does not matter: r = min, c = max
    assert bench.ns_flops_algorithmic([S(300, 1000)]) == bench.ns_flops_algorithmic([S(1000, 300)])
    # the symmetric phases (GRAM, POLY) count half their dense work; APPLY counts all of it
    r, c = 300, 1000
    saved = 5 * (r * r * c + r ** 3)
    assert bench.ns_flops_dense([S(c, r)]) - bench.ns_flops_algorithmic([S(c, r)]) == saved


def test_plan_balance_reports_the_heaviest_rank_over_the_means():
    wl = workload("7b_share")
    pb = bench.plan_balance(wl.params, wl.world_size)
    shards, F, B = bench.product_plan(wl.params, wl.world_size)
    assert pb["world_size"] == wl.world_size
    assert pb["heaviest_rank"] == bench.product_heaviest(F, B)
    assert pb["imbalance_flops"] == pytest.approx(max(F) / (sum(F) / len(F)), rel=1e-5)
    assert pb["imbalance_bytes"] == pytest.approx(max(B) / (sum(B) / len(B)), rel=1e-5)
    assert pb["imbalance_flops"] >= 1.0 and pb["imbalance_bytes"] >= 1.0
    assert 1 <= pb["ranks_with_matrices"] <= wl.world_size
