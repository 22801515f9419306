"""Owner-segment exchange fused into the step (mfsdp_muon_step_p2p).

The gradient of each matrix arrives as R rank contributions that the momentum
kernel sums in rank order; the parameter-write kernel also stores the updated
parameter to D destination buffers.  On one GPU the contributions and copies
are ordinary local buffers standing in for peer memory (the kernels use the
same plain loads and stores either way).

Checks: parity against the oracle on the summed gradient; every copy equals
the parameter bit for bit; and the equivalence invariant (MatrixFSDP: the
owner receives exactly the full gradient, so the owner-local update equals
the full-matrix update): stepping with R parts gives bitwise the same O, W and
momentum as stepping with the same parts pre-summed in the same order.
"""

import numpy as np
import pytest
import torch

import oracle
from synth.workloads import custom_workload
from synth.gen import param_seed
from tests import _harness as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from matrix_optimizer_step_nesterov_b200 import build
    build.build()


def split_grad(G: np.ndarray, R: int, seed: int, dtype: str):
    """R parts (in the grad dtype) of a gradient; their fp32 sum is what the owner sees."""
    rng = param_seed(seed, 0, 0, 99)
    parts = []
    for r in range(R):
        parts.append(H.round_to(G / R + rng.standard_normal(G.shape).astype(np.float32) * np.float32(1e-4), dtype)
                     if r < R - 1 else None)
    acc = np.zeros_like(G, dtype=np.float32)
    for p in parts[:-1]:
        acc = acc + p
    parts[-1] = H.round_to(G - acc, dtype)
    return parts


@pytest.mark.parametrize("mode", ["bf16", "fp32"])
def test_p2p_step_parity_and_copies(mode):
    from matrix_optimizer_step_nesterov_b200 import MuonOwnerStep
    dtype = "bf16" if mode == "bf16" else "f32"
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    shapes = [(256, 512), (600, 300), (128, 128), (77, 1030)]
    wl = custom_workload(shapes, dtype=dtype, seed=21)
    hs = H.host_state(wl, wl.matrices, buf_init="random")
    R, D = 3, 2
    dev = torch.device("cuda")
    parts = [split_grad(hs.G[k], R, 100 + k, dtype) for k in range(len(shapes))]
    W = [torch.from_numpy(w).to(tdt).to(dev) for w in hs.W]
    B = [torch.from_numpy(b).to(dev) for b in hs.buf]
    O = [torch.empty(w.shape, dtype=torch.float32, device=dev) for w in W]
    P = [[torch.from_numpy(p).to(tdt).to(dev) for p in parts[k]] for k in range(len(shapes))]
    C = [[torch.full(w.shape, 7.0, dtype=tdt, device=dev) for _ in range(D)] for w in W]
    st = MuonOwnerStep(W, [None] * len(W), B, O, mode=mode, grad_parts=P, param_copies=C)
    st.step()
    torch.cuda.synchronize()
    st.close()
    hp = H.muon_hparams_as_passed()
    for k in range(len(shapes)):
        # the oracle's owner-segment form: the ranks' contributions summed in rank order
        Wn, On, bn = oracle.muon_step_parts(hs.W[k], parts[k], hs.buf[k], hp)
        assert H.rel_frob(O[k].cpu().numpy(), On) <= H.TOL_O[mode]
        assert H.rel_frob(B[k].cpu().numpy(), bn) <= H.TOL_BUF
        for c in C[k]:
            assert torch.equal(c, W[k]), "a parameter copy differs from the parameter"


@pytest.mark.parametrize("mode", ["bf16", "fp32"])
def test_owner_update_equals_full_gradient_update(mode):
    from matrix_optimizer_step_nesterov_b200 import MuonOwnerStep
    dtype = "bf16" if mode == "bf16" else "f32"
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    shapes = [(384, 256), (256, 640)]
    wl = custom_workload(shapes, dtype=dtype, seed=22)
    hs = H.host_state(wl, wl.matrices, buf_init="random")
    R = 4
    dev = torch.device("cuda")
    parts = [split_grad(hs.G[k], R, 200 + k, dtype) for k in range(len(shapes))]
    # the same parts pre-summed in rank order in fp32 (the owner's full gradient)
    full = []
    for k in range(len(shapes)):
        acc = parts[k][0].astype(np.float32)
        for p in parts[k][1:]:
            acc = acc + p.astype(np.float32)
        full.append(acc)

    def run(use_parts):
        W = [torch.from_numpy(w).to(tdt).to(dev) for w in hs.W]
        B = [torch.from_numpy(b).to(dev) for b in hs.buf]
        O = [torch.empty(w.shape, dtype=torch.float32, device=dev) for w in W]
        if use_parts:
            P = [[torch.from_numpy(p).to(tdt).to(dev) for p in parts[k]] for k in range(len(shapes))]
            st = MuonOwnerStep(W, [None] * len(W), B, O, mode=mode, grad_parts=P)
        else:
            Gf = [torch.from_numpy(g).to(dev) for g in full]          # fp32 gradients
            st = MuonOwnerStep(W, Gf, B, O, mode=mode)
        st.step()
        torch.cuda.synchronize()
        st.close()
        return [w.cpu() for w in W], [o.cpu() for o in O], [b.cpu() for b in B]

    Wa, Oa, Ba = run(True)
    Wb, Ob, Bb = run(False)
    for k in range(len(shapes)):
        assert torch.equal(Oa[k], Ob[k]) and torch.equal(Wa[k], Wb[k]) and torch.equal(Ba[k], Bb[k])


@pytest.mark.parametrize("mode", ["bf16", "fp32"])
@pytest.mark.parametrize("groups", [1, 2, 3])
def test_overlapped_materialisation_equals_the_fused_step(mode, groups):
    """mfsdp_muon_step_p2p_overlap: the list in groups, each group's parameter
    copies on a side stream while later groups compute; results bit for bit
    those of the fused step, every copy equal to its parameter."""
    from matrix_optimizer_step_nesterov_b200 import MuonOwnerStep
    dtype = "bf16" if mode == "bf16" else "f32"
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    shapes = [(256, 512), (600, 300), (128, 128), (77, 1030), (512, 512)]
    wl = custom_workload(shapes, dtype=dtype, seed=23)
    hs = H.host_state(wl, wl.matrices, buf_init="random")
    R, D = 2, 2
    dev = torch.device("cuda")
    parts = [split_grad(hs.G[k], R, 300 + k, dtype) for k in range(len(shapes))]

    def run(overlap):
        W = [torch.from_numpy(w).to(tdt).to(dev) for w in hs.W]
        B = [torch.from_numpy(b).to(dev) for b in hs.buf]
        O = [torch.empty(w.shape, dtype=torch.float32, device=dev) for w in W]
        P = [[torch.from_numpy(p).to(tdt).to(dev) for p in parts[k]] for k in range(len(shapes))]
        C = [[torch.full(w.shape, 3.0, dtype=tdt, device=dev) for _ in range(D)] for w in W]
        st = MuonOwnerStep(W, [None] * len(W), B, O, mode=mode, grad_parts=P, param_copies=C,
                           overlap_groups=overlap)
        st.step()
        st.step()
        torch.cuda.synchronize()
        st.close()
        return W, O, B, C

    Wf, Of, Bf, Cf = run(0)
    Wo, Oo, Bo, Co = run(groups)
    for k in range(len(shapes)):
        assert torch.equal(Wf[k], Wo[k]) and torch.equal(Of[k], Oo[k]) and torch.equal(Bf[k], Bo[k])
        for c in Co[k]:
            assert torch.equal(c, Wo[k]), "a copy differs from its parameter"
