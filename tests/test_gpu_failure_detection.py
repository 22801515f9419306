"""Failure detection on the GPU without a GPU fault.

Kernel-side waits are bounded: past the limit the waiting thread records
MFSDP_ERR_TIMEOUT in the library's device status word and the kernel returns
normally.  The self-test kernel waits on a barrier that nothing arrives on;
the host reads the status, it is cleared by the read, and the context keeps
working (a normal step still matches the oracle).
"""

import time

import numpy as np
import pytest
import torch

import oracle
from synth.workloads import custom_workload
from tests import _harness as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from matrix_optimizer_step_nesterov_b200 import build
    build.build()


def test_bounded_wait_reports_timeout_and_context_survives():
    from matrix_optimizer_step_nesterov_b200 import _lib as lib
    stream = torch.cuda.current_stream().cuda_stream
    assert lib.mfsdp_get_device_status(stream) == lib.MFSDP_OK
    t0 = time.perf_counter()
    lib.mfsdp_selftest_bounded_wait(20_000_000, stream)          # 20 ms limit
    status = lib.mfsdp_get_device_status(stream)
    elapsed = time.perf_counter() - t0
    assert status == lib.MFSDP_ERR_TIMEOUT
    assert elapsed < 5.0
    assert lib.mfsdp_get_device_status(stream) == lib.MFSDP_OK   # the read cleared it
    # the context is still usable: a normal bf16 step matches the oracle
    wl = custom_workload([(192, 320)], dtype="bf16", seed=41)
    hs = H.host_state(wl, wl.matrices)
    res = H.gpu_step(hs, "bf16")
    H.assert_parity(H.compare_matrix(hs, res, 0, "bf16"), "bf16")
    assert lib.mfsdp_get_device_status(stream) == lib.MFSDP_OK


def test_selftest_rejects_bad_limits():
    from matrix_optimizer_step_nesterov_b200 import _lib as lib
    with pytest.raises(lib.MfsdpError):
        lib.mfsdp_selftest_bounded_wait(10, torch.cuda.current_stream().cuda_stream)
