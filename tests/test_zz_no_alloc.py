"""mfsdp_muon_step_noalloc against mfsdp_muon_step, through the C ABI.

The no-allocation entry point is for callers that cannot allocate device
memory at step time (hosts and plugins that own all device memory through
their own pools, loops that must not enter an allocator): it runs the same
step with the library's fixed 64 MiB device scratch instead of a caller
workspace.  It launches the same kernels over the same layout, so its results
must equal the workspace entry point's bit for bit, call after call, also
when calls alternate between different matrix lists that share the scratch.
One result is also checked against the fp64 oracle.  This file is named to
be collected last, and it also passes alone in a fresh process.
"""

import numpy as np
import pytest
import torch

from synth.workloads import custom_workload
from tests import _harness as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from matrix_optimizer_step_nesterov_b200 import build
    build.build()


def _device_state(hs, dtype):
    dev = torch.device("cuda")
    W = [torch.from_numpy(w).to(dtype).to(dev) for w in hs.W]
    G = [torch.from_numpy(g).to(dtype).to(dev) for g in hs.G]
    B = [torch.from_numpy(b).to(dev) for b in hs.buf]
    O = [torch.empty(w.shape, dtype=torch.float32, device=dev) for w in W]
    return W, G, B, O


def _mats(lib, W, G, B, O):
    code = {torch.float32: lib.MFSDP_DTYPE_F32, torch.bfloat16: lib.MFSDP_DTYPE_BF16}
    return [lib.Matrix(w.data_ptr(), g.data_ptr(), b.data_ptr(), o.data_ptr(), w.shape[0], w.shape[1],
                       code[w.dtype], code[g.dtype]) for w, g, b, o in zip(W, G, B, O)]


class _Pair:
    """One matrix list stepped twice over: through a private workspace and
    through the shared no-allocation scratch, from identical copies of the state."""

    def __init__(self, lib, shapes, mode, seed):
        self.lib = lib
        self.dtype = torch.bfloat16 if mode == "bf16" else torch.float32
        wl = custom_workload(shapes, dtype="bf16" if mode == "bf16" else "f32", seed=seed)
        self.hs = H.host_state(wl, wl.matrices, buf_init="random")
        self.ref = _device_state(self.hs, self.dtype)
        self.new = _device_state(self.hs, self.dtype)
        self.mats_ref = _mats(lib, *self.ref)
        self.mats_new = _mats(lib, *self.new)
        self.hp = lib.muon_hparams(mode=lib.MFSDP_MODE_BF16 if mode == "bf16" else lib.MFSDP_MODE_FP32)
        self.ws_bytes = lib.mfsdp_muon_workspace_size(self.mats_ref, self.hp)
        assert 0 < self.ws_bytes <= lib.NOALLOC_SCRATCH_BYTES
        self.ws = torch.empty(self.ws_bytes + 256, dtype=torch.uint8, device="cuda")
        self.ws_ptr = (self.ws.data_ptr() + 255) // 256 * 256

    def step(self, stream):
        self.lib.mfsdp_muon_step(self.mats_ref, self.hp, self.ws_ptr, self.ws_bytes, stream)
        self.lib.mfsdp_muon_step_noalloc(self.mats_new, self.hp, stream)

    def assert_identical(self, what):
        for k in range(len(self.mats_ref)):
            for name, a, b in zip("WGBO", self.ref, self.new):
                assert torch.equal(a[k], b[k]), f"{what}: matrix {k} {name} differs from the workspace entry point"

    def close(self):
        self.lib.mfsdp_muon_forget_workspace(self.ws_ptr)


@pytest.mark.parametrize("mode", ["fp32", "bf16"])
def test_noalloc_equals_workspace_entry_point_bitwise(mode):
    from matrix_optimizer_step_nesterov_b200 import _lib as lib
    stream = torch.cuda.current_stream().cuda_stream
    a = _Pair(lib, [(256, 512), (384, 128), (100, 300)], mode, seed=77)
    b = _Pair(lib, [(640, 200), (128, 128), (33, 1000), (513, 257)], mode, seed=78)
    try:
        # two calls in a row on list A, then list B, then A again: the shared
        # scratch holds the other list's tables and buffers between them
        for call, pair in enumerate((a, a, b, b, a)):
            pair.step(stream)
            torch.cuda.synchronize()
            pair.assert_identical(f"call {call}")
            if call == 2:
                # list B's first step, right after list A used the scratch, against the oracle
                for k in range(len(b.hs.specs)):
                    _, O_ref, _ = H.oracle_step(b.hs, k)
                    o_new = b.new[3][k].cpu().numpy().astype(np.float64)
                    assert H.rel_frob(o_new, O_ref) <= H.TOL_O[mode], f"matrix {k}: update differs from the oracle"
        assert lib.mfsdp_get_device_status(stream) == 0
    finally:
        a.close()
        b.close()


def test_noalloc_rejects_lists_beyond_its_scratch():
    from matrix_optimizer_step_nesterov_b200 import _lib as lib
    hp = lib.muon_hparams(mode=lib.MFSDP_MODE_BF16)
    # 4096 x 4096 bf16 needs far more than 64 MiB of scratch; rejected before any GPU work
    big = lib.Matrix(1 << 30, 1 << 31, 1 << 32, None, 4096, 4096, lib.MFSDP_DTYPE_BF16, lib.MFSDP_DTYPE_BF16)
    assert lib.mfsdp_muon_workspace_size([big], hp) > lib.NOALLOC_SCRATCH_BYTES
    with pytest.raises(lib.MfsdpError) as e:
        lib.mfsdp_muon_step_noalloc([big], hp, torch.cuda.current_stream().cuda_stream)
    assert e.value.status == lib.MFSDP_ERR_WORKSPACE_TOO_SMALL
