"""The five workloads at full size on the GPU against the fp64 C++ oracle.

Each workload's whole owner share is stepped in ONE grouped call, the launch
configuration the benchmark times, once in each GEMM mode; the oracle then
recomputes a sample of the matrices one by one (once, for both modes):
every distinct shape, at least eight seeded picks (all matrices when fewer),
and on the skew workload at least one matrix of each short-side class
r = 128, 256, 384, 512 and r >= 1024 plus both extreme aspect ratios.
Per-matrix errors go to $MFSDP_PARITY_REPORT when it is set.
"""

import random

import numpy as np
import pytest
import torch

from synth import workload
from tests import _harness as H

pytestmark = pytest.mark.gpu

MODES = ("bf16", "fp32")


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def sample_indices(specs, picks, seed, classes=()):
    """Every distinct shape, ``picks`` seeded extra matrices, and one matrix of
    each short-side class [lo, hi) in ``classes``."""
    idx = set()
    seen = set()
    for k, s in enumerate(specs):
        if (s.rows, s.cols) not in seen:
            seen.add((s.rows, s.cols))
            idx.add(k)
    rnd = random.Random(seed)
    for lo, hi in classes:
        members = [k for k, s in enumerate(specs) if lo <= min(s.rows, s.cols) < hi]
        if members and not idx.intersection(members):
            idx.add(rnd.choice(members))
    pool = [k for k in range(len(specs)) if k not in idx]
    idx.update(rnd.sample(pool, min(picks, len(pool))))
    return sorted(idx)


def skew_sample(specs):
    """The skew workload has hundreds of distinct shapes: sample by class
    instead, plus the two extreme aspect ratios and eight seeded picks."""
    rnd = random.Random(1)
    idx = set()
    for lo, hi in ((128, 129), (256, 257), (384, 385), (512, 513), (1024, 1 << 30)):
        members = [k for k, s in enumerate(specs) if lo <= min(s.rows, s.cols) < hi and max(s.rows, s.cols) > 64]
        idx.update(rnd.sample(members, min(2, len(members))))
    idx.update(k for k, s in enumerate(specs) if (s.rows, s.cols) in ((64, 16384), (16384, 64)))
    # one of each extreme is enough: keep the first of each
    extremes = {}
    for k in sorted(idx):
        sh = (specs[k].rows, specs[k].cols)
        if sh in ((64, 16384), (16384, 64)):
            extremes.setdefault(sh, k)
    idx = {k for k in idx if (specs[k].rows, specs[k].cols) not in ((64, 16384), (16384, 64))} | set(extremes.values())
    pool = [k for k in range(len(specs)) if k not in idx]
    idx.update(rnd.sample(pool, 8))
    return sorted(idx)


@pytest.mark.parametrize("name", ["block", "7b_share", "32b_share", "skew"])
def test_workload_parity(name):
    wl = workload(name)
    specs = H.owner_share(wl)
    hs = H.host_state(wl, specs)
    want = skew_sample(specs) if name == "skew" else sample_indices(specs, 8, 1)
    results = {mode: H.gpu_step(hs, mode, want_o=want, keep=want) for mode in MODES}
    failures = []
    worst = {mode: 0.0 for mode in MODES}
    for k in want:
        ref = H.oracle_step(hs, k)
        for mode in MODES:
            m = H.compare_matrix(hs, results[mode], k, mode, ref=ref)
            label = f"{name}[{k}] {specs[k].rows}x{specs[k].cols}"
            try:
                H.assert_parity(m, mode, label)
            except AssertionError as e:
                failures.append(f"{mode}: {e}")
            worst[mode] = max(worst[mode], m["rel_O"])
        del ref
    print(f"{name}: {len(want)} sampled matrices; worst rel_O " +
          ", ".join(f"{mode} {worst[mode]:.3e}" for mode in MODES))
    assert not failures, "\n".join(failures)
