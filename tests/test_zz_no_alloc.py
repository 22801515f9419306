"""mfsdp_muon_step_noalloc against mfsdp_muon_step, through the C ABI.

The no-allocation entry point serves callers that cannot allocate device
memory at step time (stream capture, host-owned memory pools): it runs the
same step with the library's fixed 64 MiB device scratch instead of a caller
workspace.  Two calls in a row must match two calls of the workspace entry
point on the same inputs, within the parity tolerance.  This file is named to
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


@pytest.mark.parametrize("mode", ["fp32", "bf16"])
def test_noalloc_matches_workspace_entry_point_on_two_calls(mode):
    from matrix_optimizer_step_nesterov_b200 import _lib as lib
    dtype = torch.bfloat16 if mode == "bf16" else torch.float32
    shapes = [(256, 512), (384, 128), (100, 300)]
    wl = custom_workload(shapes, dtype="bf16" if mode == "bf16" else "f32", seed=77)
    hs = H.host_state(wl, wl.matrices, buf_init="random")
    hp = lib.muon_hparams(mode=lib.MFSDP_MODE_BF16 if mode == "bf16" else lib.MFSDP_MODE_FP32)
    stream = torch.cuda.current_stream().cuda_stream

    # reference: the workspace entry point, two calls in a row
    Wr, Gr, Br, Or = _device_state(hs, dtype)
    mats_r = _mats(lib, Wr, Gr, Br, Or)
    ws_bytes = lib.mfsdp_muon_workspace_size(mats_r, hp)
    assert ws_bytes <= lib.NOALLOC_SCRATCH_BYTES
    ws = torch.empty(ws_bytes + 256, dtype=torch.uint8, device="cuda")
    ws_ptr = (ws.data_ptr() + 255) // 256 * 256
    # the no-allocation entry point on an identical copy of the state
    Wn, Gn, Bn, On = _device_state(hs, dtype)
    mats_n = _mats(lib, Wn, Gn, Bn, On)

    for call in range(2):
        lib.mfsdp_muon_step(mats_r, hp, ws_ptr, ws_bytes, stream)
        lib.mfsdp_muon_step_noalloc(mats_n, hp, stream)
        torch.cuda.synchronize()
        for k in range(len(shapes)):
            o_ref = Or[k].cpu().numpy().astype(np.float64)
            o_new = On[k].cpu().numpy().astype(np.float64)
            assert H.rel_frob(o_new, o_ref) <= H.TOL_O[mode], f"call {call} matrix {k}: update differs"
            assert H.rel_frob(Bn[k].cpu().numpy(), Br[k].cpu().numpy().astype(np.float64)) <= H.TOL_BUF
            w_ref = Wr[k].cpu().to(torch.float64).numpy()
            w_new = Wn[k].cpu().to(torch.float64).numpy()
            assert H.rel_frob(w_new, w_ref) <= H.TOL_O[mode] * 0.02 + 1e-6
    lib.mfsdp_muon_forget_workspace(ws_ptr)
    assert lib.mfsdp_get_device_status(stream) == 0


def test_noalloc_rejects_lists_beyond_its_scratch():
    from matrix_optimizer_step_nesterov_b200 import _lib as lib
    hp = lib.muon_hparams(mode=lib.MFSDP_MODE_BF16)
    # 4096 x 4096 bf16 needs far more than 64 MiB of scratch; rejected before any GPU work
    big = lib.Matrix(1 << 30, 1 << 31, 1 << 32, None, 4096, 4096, lib.MFSDP_DTYPE_BF16, lib.MFSDP_DTYPE_BF16)
    assert lib.mfsdp_muon_workspace_size([big], hp) > lib.NOALLOC_SCRATCH_BYTES
    with pytest.raises(lib.MfsdpError) as e:
        lib.mfsdp_muon_step_noalloc([big], hp, torch.cuda.current_stream().cuda_stream)
    assert e.value.status == lib.MFSDP_ERR_WORKSPACE_TOO_SMALL
