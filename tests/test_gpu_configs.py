"""The five workloads at full size on the GPU against the fp64 oracle.

Each workload's whole owner share is stepped in ONE grouped call, the launch
configuration the benchmark times; the oracle recomputes a sample of the
matrices (every distinct shape, plus seeded picks) one by one.
"""

import random

import numpy as np
import pytest
import torch

from synth import workload
from tests import _harness as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def sample_indices(specs, extra, seed):
    first = {}
    for k, s in enumerate(specs):
        first.setdefault((s.rows, s.cols), k)
    idx = set(first.values()) if len(first) <= 8 else set()
    rnd = random.Random(seed)
    pool = [k for k in range(len(specs)) if k not in idx]
    idx.update(rnd.sample(pool, min(extra, len(pool))))
    return sorted(idx)


_STATES = {}


def state(name):
    if name not in _STATES:
        wl = workload(name)
        specs = H.owner_share(wl)
        _STATES.clear()
        _STATES[name] = (wl, specs, H.host_state(wl, specs))
    return _STATES[name]


@pytest.mark.parametrize("name,extra", [("block", 0), ("7b_share", 1), ("32b_share", 0), ("skew", 6)])
@pytest.mark.parametrize("mode", ["bf16", "fp32"])
def test_workload_parity(name, extra, mode):
    wl, specs, hs = state(name)
    if name == "skew":
        # both extreme aspect ratios are always in the sample
        want = sorted(set(sample_indices(specs, extra, 1)) | {512, 520})
    else:
        want = sample_indices(specs, extra, 1)
    res = H.gpu_step(hs, mode, want_o=want)
    worst = 0.0
    for k in want:
        m = H.compare_matrix(hs, res, k, mode)
        H.assert_parity(m, mode, f"{name} {specs[k].rows}x{specs[k].cols}")
        worst = max(worst, m["rel_O"])
    print(f"{name} {mode}: {len(want)} sampled matrices, worst rel_O {worst:.3e}")
