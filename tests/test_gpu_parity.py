"""GPU path (libmfsdp through its C ABI) against the fp64 oracle.

Bars: per-matrix relative Frobenius error of the update O <= 1e-4 (fp32 mode)
or <= 2e-2 (bf16 mode); momentum buffer <= 1e-6; the parameter write within 2
ulp (of the parameter dtype) of the fp64 write of the GPU's own O, plus 2 fp32
ulps of the larger write operand where the two terms cancel; AdamW per element
|d| <= 1e-6 |ref| + 2^-23 max|ref|.  The oracle receives the hyper-parameters
as the ABI passes them (fp32 values).
"""

import numpy as np
import pytest
import torch

import oracle
from synth import workload
from synth.workloads import custom_workload
from synth.gen import tail_inputs
from tests import _harness as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from matrix_optimizer_step_nesterov_b200 import build
    build.build()


MODES = ["fp32", "bf16"]


# ---- config 1: tiny owner step ----------------------------------------------------

@pytest.mark.parametrize("mode", MODES)
def test_tiny_config(mode):
    wl = workload("tiny")
    hs = H.host_state(wl, wl.matrices)
    res = H.gpu_step(hs, mode)
    m = H.compare_matrix(hs, res, 0, mode)
    H.assert_parity(m, mode, "tiny")


@pytest.mark.parametrize("mode", MODES)
def test_tiny_config_three_steps(mode):
    # three consecutive steps with fresh gradients: momentum carries over
    wl = workload("tiny")
    spec = wl.matrices[0]
    hs = H.host_state(wl, [spec])
    from matrix_optimizer_step_nesterov_b200 import MuonOwnerStep
    dev = torch.device("cuda")
    Wt = torch.from_numpy(hs.W[0]).to(dev)
    bt = torch.from_numpy(hs.buf[0]).to(dev)
    O = torch.empty_like(Wt)
    W64, b64 = hs.W[0].astype(np.float64), hs.buf[0].astype(np.float64)
    for step in range(3):
        G = H.host_state(wl, [spec], step=step).G[0]
        Gt = torch.from_numpy(G).to(dev)
        st = MuonOwnerStep([Wt], [Gt], [bt], [O], mode=mode)
        st.step()
        torch.cuda.synchronize()
        st.close()
        W64, O64, b64 = oracle.muon_step(W64, G.astype(np.float64), b64, H.muon_hparams_as_passed())
        assert H.rel_frob(O.cpu().numpy(), O64) <= H.TOL_O[mode]
        assert H.rel_frob(bt.cpu().numpy(), b64) <= 1e-6
    # after three steps the fp32 weights stay close to the fp64 trajectory
    assert H.rel_frob(Wt.cpu().numpy(), W64) <= (1e-6 if mode == "fp32" else 1e-3)


# ---- ragged shapes, edge cases -------------------------------------------------------

RAGGED = [(1, 1), (1, 300), (300, 1), (100, 37), (37, 100), (129, 257), (257, 129), (65, 65),
          (200, 1000), (1000, 200), (128, 128), (255, 513), (600, 1100), (1100, 600), (257, 2049)]


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_ragged_shapes_grouped(mode, dtype):
    wl = custom_workload(RAGGED, dtype=dtype, seed=31)
    hs = H.host_state(wl, wl.matrices, buf_init="random")
    res = H.gpu_step(hs, mode)
    for k, s in enumerate(wl.matrices):
        m = H.compare_matrix(hs, res, k, mode)
        H.assert_parity(m, mode, f"{s.rows}x{s.cols}")


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("ns_steps", [0, 1, 2, 3, 7])
def test_iteration_counts(ns_steps, mode):
    # ns_steps = 1 makes the first iteration also the last (the Frobenius scale
    # enters the final X update); 0 writes the normalised momentum itself
    wl = custom_workload([(96, 160), (160, 96), (300, 520)], dtype="f32" if mode == "fp32" else "bf16", seed=5)
    hs = H.host_state(wl, wl.matrices)
    res = H.gpu_step(hs, mode, ns_steps=ns_steps)
    for k in range(3):
        m = H.compare_matrix(hs, res, k, mode, ns_steps=ns_steps)
        H.assert_parity(m, mode, f"ns_steps={ns_steps} {hs.specs[k].rows}x{hs.specs[k].cols}")
        if mode == "bf16" and ns_steps == 0:
            # no GEMM ran: O is the normalised momentum read back from the bf16
            # hi + lo master, which holds each element within 2^-16 of itself
            assert m["rel_O"] <= 2e-5, f"two-part master error {m['rel_O']:.3e}"


def test_plain_momentum_and_other_hparams():
    wl = custom_workload([(64, 192), (192, 64)], dtype="f32", seed=6)
    hs = H.host_state(wl, wl.matrices, buf_init="random")
    kw = dict(nesterov=False, lr=0.1, beta=0.9, weight_decay=0.1)
    res = H.gpu_step(hs, "fp32", **kw)
    for k in range(2):
        H.assert_parity(H.compare_matrix(hs, res, k, "fp32", **kw), "fp32", "plain momentum")


@pytest.mark.parametrize("mode", MODES)
def test_zero_gradient_is_pure_decay(mode):
    wl = custom_workload([(64, 96)], dtype="bf16", seed=7)
    hs = H.host_state(wl, wl.matrices)
    zeros = [np.zeros_like(hs.G[0])]
    res = H.gpu_step(hs, mode, grads=zeros)
    assert np.all(res.O[0] == 0.0)
    ref = torch.from_numpy(hs.W[0].astype(np.float64) * (1 - 0.02 * 0.01)).to(torch.bfloat16)
    assert H.ulp_distance(res.W[0], ref).max() == 0


def test_empty_and_zero_size_matrices():
    from matrix_optimizer_step_nesterov_b200 import MuonOwnerStep
    dev = torch.device("cuda")
    st = MuonOwnerStep([], [], [], mode="bf16")
    st.step()
    w = torch.randn(0, 8, device=dev)
    st = MuonOwnerStep([w], [w.clone()], [w.clone()], mode="fp32")
    st.step()
    # a zero-size matrix next to a real one leaves the real one's result unchanged
    wl = custom_workload([(48, 80)], dtype="f32", seed=8)
    hs = H.host_state(wl, wl.matrices)
    Wt = torch.from_numpy(hs.W[0]).to(dev)
    Gt = torch.from_numpy(hs.G[0]).to(dev)
    bt = torch.from_numpy(hs.buf[0]).to(dev)
    O = torch.empty_like(Wt)
    e = torch.empty(5, 0, device=dev)
    st = MuonOwnerStep([e, Wt], [e.clone(), Gt], [e.clone(), bt], [None, O], mode="fp32")
    st.step()
    torch.cuda.synchronize()
    _, O64, _ = oracle.muon_step(hs.W[0], hs.G[0], hs.buf[0], H.muon_hparams_as_passed())
    assert H.rel_frob(O.cpu().numpy(), O64) <= 1e-4


@pytest.mark.parametrize("mode", MODES)
def test_deterministic_and_grouping_independent(mode):
    shapes = [(128, 384), (384, 128), (256, 256), (64, 640), (200, 72)]
    wl = custom_workload(shapes, dtype="bf16", seed=9)
    hs = H.host_state(wl, wl.matrices, buf_init="random")
    a = H.gpu_step(hs, mode)
    b = H.gpu_step(hs, mode)
    for k in range(len(shapes)):
        assert np.array_equal(a.O[k], b.O[k])
        assert torch.equal(a.W[k], b.W[k])
    # stepping a subset alone gives bitwise the same result for its matrices
    sub = H.HostState([hs.specs[1], hs.specs[3]], [hs.W[1], hs.W[3]], [hs.G[1], hs.G[3]], [hs.buf[1], hs.buf[3]])
    c = H.gpu_step(sub, mode)
    assert np.array_equal(c.O[0], a.O[1]) and np.array_equal(c.O[1], a.O[3])
    assert torch.equal(c.W[0], a.W[1]) and np.array_equal(c.buf[1], a.buf[3])


def test_device_status_clean():
    from matrix_optimizer_step_nesterov_b200 import device_status
    wl = custom_workload([(32, 64)], dtype="bf16", seed=10)
    hs = H.host_state(wl, wl.matrices)
    H.gpu_step(hs, "bf16")
    assert device_status() == 0


# ---- AdamW tail -----------------------------------------------------------------------

@pytest.mark.parametrize("name", ["tiny", "block", "7b_share", "32b_share"])
def test_adamw_tail_three_steps(name):
    wl = workload(name)
    ti = tail_inputs(wl, state="zeros")
    hp = H.adamw_hparams_as_passed()
    p, m, v = ti.p, ti.m, ti.v
    pr, mr, vr = p.astype(np.float64), m.astype(np.float64), v.astype(np.float64)
    for t in range(1, 4):
        g = tail_inputs(wl, step=t - 1).g
        p, m, v = H.gpu_adamw(p, g, m, v, t)
        pr, mr, vr = oracle.adamw_step(pr, g, mr, vr, t, hp)
        # the next oracle step starts from the same fp32 state as the GPU
        assert H.adamw_tolerance_ok(p, pr) and H.adamw_tolerance_ok(m, mr) and H.adamw_tolerance_ok(v, vr)
        pr, mr, vr = p.astype(np.float64), m.astype(np.float64), v.astype(np.float64)


@pytest.mark.parametrize("n,offset", [(4097, 0), (4096, 1), (1, 0), (3, 2), (1000003, 0)])
def test_adamw_ragged_and_misaligned(n, offset):
    wl = custom_workload([], tail=n, seed=12)
    ti = tail_inputs(wl, state="random")
    p, m, v = H.gpu_adamw(ti.p, ti.g, ti.m, ti.v, 7, offset=offset)
    pr, mr, vr = oracle.adamw_step(ti.p, ti.g, ti.m, ti.v, 7, H.adamw_hparams_as_passed())
    assert H.adamw_tolerance_ok(p, pr) and H.adamw_tolerance_ok(m, mr) and H.adamw_tolerance_ok(v, vr)


def test_adamw_skew_tail_sampled():
    # the 64 Mi-element tail of the skew workload, checked on every element
    wl = workload("skew")
    ti = tail_inputs(wl, state="random")
    p, m, v = H.gpu_adamw(ti.p, ti.g, ti.m, ti.v, 10)
    pr, mr, vr = oracle.adamw_step(ti.p, ti.g, ti.m, ti.v, 10, H.adamw_hparams_as_passed())
    assert H.adamw_tolerance_ok(p, pr) and H.adamw_tolerance_ok(m, mr) and H.adamw_tolerance_ok(v, vr)


@pytest.mark.parametrize("mode", MODES)
def test_cuda_graph_replay_matches_eager_steps(mode):
    # two eager steps against one eager step plus the replay of a captured step:
    # the same launches on the same buffers, so the results are bit-identical
    import torch
    from matrix_optimizer_step_nesterov_b200 import MuonOwnerStep
    wl = custom_workload([(300, 520), (520, 300), (64, 64)], dtype="f32" if mode == "fp32" else "bf16", seed=11)
    hs = H.host_state(wl, wl.matrices, buf_init="random")
    dev = torch.device("cuda")
    dt = torch.float32 if mode == "fp32" else torch.bfloat16

    def make():
        ps = [torch.from_numpy(w).to(dt).to(dev) for w in hs.W]
        gs = [torch.from_numpy(g).to(dt).to(dev) for g in hs.G]
        bs = [torch.from_numpy(b).to(dev) for b in hs.buf]
        return ps, gs, bs, MuonOwnerStep(ps, gs, bs, mode=mode)

    pa, ga, ba, sa = make()
    sa.step()
    sa.step()
    pb, gb, bb, sb = make()
    sb.step()
    g = sb.capture_graph()
    g.replay()
    torch.cuda.synchronize()
    for k in range(len(pa)):
        assert torch.equal(pa[k], pb[k]), f"param {k}"
        assert torch.equal(ba[k], bb[k]), f"momentum {k}"
    del g
    sa.close()
    sb.close()
