"""Host-side checks of libmfsdp: it loads, exports every symbol include/mfsdp.h
declares, validates arguments before touching the GPU, and its planner agrees
exactly with the oracle planner.  No compute call runs here."""

import ctypes
import os
import re

import pytest

import oracle
from synth import workload
from synth.workloads import custom_workload, MATRIX

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from matrix_optimizer_step_nesterov_b200 import build
    build.build()
    from matrix_optimizer_step_nesterov_b200 import _lib
    return _lib


def declared_functions():
    text = open(os.path.join(ROOT, "include", "mfsdp.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mfsdp_\w+)\s*\(", text)))


def test_header_declares_the_binding_names(lib):
    assert declared_functions() == sorted(lib.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    cdll = ctypes.CDLL(lib.LIB_PATH)
    for name in declared_functions():
        assert hasattr(cdll, name), f"libmfsdp.so does not export {name}"


def test_nm_shows_c_linkage(lib):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", lib.LIB_PATH], capture_output=True, text=True).stdout
    syms = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in declared_functions():
        assert name in syms


def test_status_strings_and_version(lib):
    assert lib.status_string(0) == "MFSDP_OK"
    for code in range(-8, 0):
        assert lib.status_string(code).startswith("MFSDP_ERR_")
    assert lib.status_string(12345) == "unknown mfsdp status"
    assert lib.mfsdp_version() == 100


def _descs(wl):
    return [(p.rows, p.cols, p.kind, 1 if p.dtype == "bf16" else 0) for p in wl.params]


@pytest.mark.parametrize("name", ["tiny", "block", "7b_share", "32b_share", "skew"])
def test_planner_matches_oracle_exactly(lib, name):
    wl = workload(name)
    R = wl.world_size or 4
    shards, F, B = lib.mfsdp_plan(_descs(wl), R)
    entries, Fo, Bo = oracle.plan_owners(wl.params, R)
    assert [s.owner for s in shards] == [e.owner for e in entries]
    assert [s.owner_offset for s in shards] == [e.owner_offset for e in entries]
    assert [bool(s.transposed) for s in shards] == [e.transposed for e in entries]
    assert [s.ns_flops for s in shards] == [e.ns_flops for e in entries]
    assert [s.resident_bytes for s in shards] == [e.resident_bytes for e in entries]
    assert [s.shape_scale for s in shards] == [e.shape_scale for e in entries]
    assert F == Fo and B == Bo
    assert lib.mfsdp_heaviest_rank(F, B) == oracle.heaviest_rank(Fo, Bo)


def test_planner_rejects_bad_arguments(lib):
    with pytest.raises(lib.MfsdpError) as e:
        lib.mfsdp_plan([(4, 4, 0, 1)], 0)
    assert e.value.status == lib.MFSDP_ERR_INVALID_ARG
    with pytest.raises(lib.MfsdpError) as e:
        lib.mfsdp_plan([(-1, 4, 0, 1)], 2)
    assert e.value.status == lib.MFSDP_ERR_INVALID_ARG
    with pytest.raises(lib.MfsdpError) as e:
        lib.mfsdp_plan([(4, 4, 0, 7)], 2)
    assert e.value.status == lib.MFSDP_ERR_UNSUPPORTED_DTYPE
    shards, F, B = lib.mfsdp_plan([], 3)
    assert shards == [] and F == [0.0, 0.0, 0.0]


def _mat(lib, rows, cols, base=1 << 20, pdt=1, gdt=1):
    e = 2 if pdt == 1 else 4
    n = rows * cols
    return lib.Matrix(base, base + 4 * n + 4096, base + 8 * n + 8192, None, rows, cols, pdt, gdt)


def test_workspace_size_is_host_only_and_grows_with_shapes(lib):
    hp = lib.muon_hparams(mode=lib.MFSDP_MODE_BF16)
    s1 = lib.mfsdp_muon_workspace_size([_mat(lib, 256, 512)], hp)
    s2 = lib.mfsdp_muon_workspace_size([_mat(lib, 512, 256)], hp)
    s3 = lib.mfsdp_muon_workspace_size([_mat(lib, 256, 1024)], hp)
    assert s1 == s2 > 0 and s3 > s1
    # r x c = 256 x 512: X as bf16 hi and lo parts, each ping-pong; bf16 E_A and E_B
    assert s1 >= 256 * 512 * (2 + 2 + 2 + 2) + 256 * 256 * (2 + 2)
    hp32 = lib.muon_hparams(mode=lib.MFSDP_MODE_FP32)
    assert lib.mfsdp_muon_workspace_size([_mat(lib, 256, 512, pdt=0, gdt=0)], hp32) >= 256 * 512 * 8 + 256 * 256 * 8
    assert lib.mfsdp_muon_workspace_size([], hp) == 0
    assert lib.mfsdp_muon_workspace_size([_mat(lib, 0, 512)], hp) == 0


def test_step_validation_errors_precede_any_device_work(lib):
    hp = lib.muon_hparams()
    m = _mat(lib, 64, 64)
    bad = lib.muon_hparams(ns_steps=17)
    with pytest.raises(lib.MfsdpError) as e:
        lib.mfsdp_muon_step([m], bad, 0, 0, 0)
    assert e.value.status == lib.MFSDP_ERR_INVALID_ARG
    bad = lib.muon_hparams(mode=5)
    with pytest.raises(lib.MfsdpError) as e:
        lib.mfsdp_muon_step([m], bad, 0, 0, 0)
    assert e.value.status == lib.MFSDP_ERR_INVALID_ARG
    bad = lib.muon_hparams(lr=float("nan"))
    with pytest.raises(lib.MfsdpError) as e:
        lib.mfsdp_muon_step([m], bad, 0, 0, 0)
    assert e.value.status == lib.MFSDP_ERR_INVALID_ARG
    # misaligned bf16 param
    mm = lib.Matrix(m.param + 1, m.grad, m.momentum, None, 64, 64, 1, 1)
    with pytest.raises(lib.MfsdpError) as e:
        lib.mfsdp_muon_step([mm], hp, 0, 0, 0)
    assert e.value.status == lib.MFSDP_ERR_MISALIGNED
    # NULL grad
    mm = lib.Matrix(m.param, None, m.momentum, None, 64, 64, 1, 1)
    with pytest.raises(lib.MfsdpError) as e:
        lib.mfsdp_muon_step([mm], hp, 0, 0, 0)
    assert e.value.status == lib.MFSDP_ERR_INVALID_ARG
    # unsupported dtype code
    mm = lib.Matrix(m.param, m.grad, m.momentum, None, 64, 64, 9, 1)
    with pytest.raises(lib.MfsdpError) as e:
        lib.mfsdp_muon_step([mm], hp, 0, 0, 0)
    assert e.value.status == lib.MFSDP_ERR_UNSUPPORTED_DTYPE
    # two matrices writing the same momentum buffer
    m2 = lib.Matrix(m.param + (1 << 24), m.grad + (1 << 24), m.momentum, None, 64, 64, 1, 1)
    with pytest.raises(lib.MfsdpError) as e:
        lib.mfsdp_muon_step([m, m2], hp, 0, 0, 0)
    assert e.value.status == lib.MFSDP_ERR_INVALID_ARG
    # negative shape
    mm = lib.Matrix(m.param, m.grad, m.momentum, None, -1, 64, 1, 1)
    with pytest.raises(lib.MfsdpError) as e:
        lib.mfsdp_muon_step([mm], hp, 0, 0, 0)
    assert e.value.status == lib.MFSDP_ERR_INVALID_ARG


def test_empty_step_is_a_noop_without_a_device(lib):
    hp = lib.muon_hparams()
    lib.mfsdp_muon_step([], hp, 0, 0, 0)
    lib.mfsdp_muon_step([_mat(lib, 0, 64)], hp, 0, 0, 0)


def test_launch_count(lib):
    hp = lib.muon_hparams()
    assert lib.mfsdp_muon_step_launches([_mat(lib, 64, 64)], hp) == 3 + 3 * 5
    assert lib.mfsdp_muon_step_launches([_mat(lib, 64, 64)], lib.muon_hparams(ns_steps=0)) == 3
    assert lib.mfsdp_muon_step_launches([], hp) == 0
    # a tall matrix is tiled, a wide one with 16-byte rows is flat: two streaming launches each
    assert lib.mfsdp_muon_step_launches([_mat(lib, 128, 64), _mat(lib, 64, 128, base=1 << 30)], hp) == 5 + 3 * 5
    assert lib.mfsdp_muon_step_launches([_mat(lib, 128, 64)], hp) == 3 + 3 * 5


def test_adamw_validation(lib):
    hp = lib.adamw_hparams(step=0)
    with pytest.raises(lib.MfsdpError) as e:
        lib.mfsdp_adamw_tail(1 << 20, 2 << 20, 3 << 20, 4 << 20, 16, hp, 0)
    assert e.value.status == lib.MFSDP_ERR_INVALID_ARG
    hp = lib.adamw_hparams(step=1)
    with pytest.raises(lib.MfsdpError) as e:
        lib.mfsdp_adamw_tail((1 << 20) + 2, 2 << 20, 3 << 20, 4 << 20, 16, hp, 0)
    assert e.value.status == lib.MFSDP_ERR_MISALIGNED
    with pytest.raises(lib.MfsdpError) as e:   # p and m overlap
        lib.mfsdp_adamw_tail(1 << 20, 2 << 20, (1 << 20) + 32, 4 << 20, 16, hp, 0)
    assert e.value.status == lib.MFSDP_ERR_INVALID_ARG
    with pytest.raises(lib.MfsdpError) as e:
        lib.mfsdp_adamw_tail(0, 2 << 20, 3 << 20, 4 << 20, 16, hp, 0)
    assert e.value.status == lib.MFSDP_ERR_INVALID_ARG
    lib.mfsdp_adamw_tail(0, 0, 0, 0, 0, hp, 0)   # n == 0 is a no-op


def test_p2p_validation(lib):
    hp = lib.muon_hparams()
    m = lib.Matrix(1 << 20, 0, (1 << 20) + (1 << 24), None, 64, 64, 1, 1)   # grad NULL: parts carry it
    segs, keep = lib.owner_segments([[1 << 26, 2 << 26]], [[3 << 26]])
    assert lib.mfsdp_muon_workspace_size_p2p([m], segs, hp) > lib.mfsdp_muon_workspace_size(
        [lib.Matrix(1 << 20, 1 << 25, (1 << 20) + (1 << 24), None, 64, 64, 1, 1)], hp) - 1
    bad, keep2 = lib.owner_segments([[]], [[]])                      # no parts
    with pytest.raises(lib.MfsdpError) as e:
        lib.mfsdp_muon_step_p2p([m], bad, hp, 0, 0, 0)
    assert e.value.status == lib.MFSDP_ERR_INVALID_ARG
    bad, keep3 = lib.owner_segments([[(1 << 26) + 1]], [[]])         # misaligned bf16 part
    with pytest.raises(lib.MfsdpError) as e:
        lib.mfsdp_muon_step_p2p([m], bad, hp, 0, 0, 0)
    assert e.value.status == lib.MFSDP_ERR_MISALIGNED
    bad, keep4 = lib.owner_segments([[1 << 26]], [[0]])              # NULL copy
    with pytest.raises(lib.MfsdpError) as e:
        lib.mfsdp_muon_step_p2p([m], bad, hp, 0, 0, 0)
    assert e.value.status == lib.MFSDP_ERR_INVALID_ARG
    with pytest.raises(lib.MfsdpError) as e:                           # the plain entry point needs grad
        lib.mfsdp_muon_step([m], hp, 0, 0, 0)
    assert e.value.status == lib.MFSDP_ERR_INVALID_ARG


@pytest.mark.parametrize("name,old_w,new_w", [("7b_share", 8, 16), ("7b_share", 8, 5), ("32b_share", 64, 48),
                                              ("block", 1, 4), ("skew", 4, 7), ("tiny", 1, 2)])
def test_reshard_matches_oracle_exactly(lib, name, old_w, new_w):
    wl = workload(name)
    descs = _descs(wl)
    saved, _, _ = lib.mfsdp_plan(descs, old_w)
    shards, routes, moved = lib.mfsdp_reshard(descs, saved, new_w)
    old_o, _, _ = oracle.plan_owners(wl.params, old_w)
    new_o, routes_o, moved_o = oracle.reshard(wl.params, old_o, new_w)
    assert [s.owner for s in shards] == [e.owner for e in new_o]
    assert [s.owner_offset for s in shards] == [e.owner_offset for e in new_o]
    assert [(r.param_id, r.kind, r.src_rank, r.src_offset, r.dst_rank, r.dst_offset, r.elems, r.state_bytes)
            for r in routes] == [(o.pid, o.kind, o.src_rank, o.src_offset, o.dst_rank, o.dst_offset, o.elems,
                                  o.state_bytes) for o in routes_o]
    assert moved == moved_o
    # the new layout is the planner's own answer for the new world size
    direct, _, _ = lib.mfsdp_plan(descs, new_w)
    assert [(s.owner, s.owner_offset) for s in direct] == [(s.owner, s.owner_offset) for s in shards]


def test_reshard_validation(lib):
    descs = [(64, 64, 0, 1), (32, 64, 0, 1)]
    saved, _, _ = lib.mfsdp_plan(descs, 2)
    with pytest.raises(lib.MfsdpError) as e:
        lib.mfsdp_reshard([(64, 64, 0, 1), (64, 32, 0, 1)], saved, 3)     # shape mismatch
    assert e.value.status == lib.MFSDP_ERR_INVALID_ARG
    with pytest.raises(lib.MfsdpError) as e:
        lib.mfsdp_reshard(descs, saved, 0)
    assert e.value.status == lib.MFSDP_ERR_INVALID_ARG
    bad = list(saved)
    bad[1].owner = -1
    with pytest.raises(lib.MfsdpError) as e:
        lib.mfsdp_reshard(descs, bad, 3)
    assert e.value.status == lib.MFSDP_ERR_INVALID_ARG
    shards, routes, moved = lib.mfsdp_reshard([], [], 3)
    assert shards == [] and routes == [] and moved == 0


def test_planner_and_reshard_match_oracle_on_random_lists(lib):
    # seeded random parameter lists: mixed dtypes, tall and wide matrices, tails,
    # repeated shapes (ties), world sizes 1..9
    import numpy as np
    from synth.workloads import ParamSpec, TAIL
    rng = np.random.default_rng(20261202)
    for trial in range(40):
        n = int(rng.integers(1, 30))
        params = []
        for pid in range(n):
            if rng.random() < 0.15:
                params.append(ParamSpec(pid, f"t{pid}", int(rng.integers(1, 5000)), 1, TAIL, "f32"))
            else:
                r = int(rng.choice([64, 128, 96, 4096, 11008, 5120, 1]) if rng.random() < 0.5 else rng.integers(1, 700))
                c = int(rng.choice([64, 128, 4096, 2048]) if rng.random() < 0.5 else rng.integers(1, 700))
                params.append(ParamSpec(pid, f"m{pid}", r, c, MATRIX, "bf16" if rng.random() < 0.7 else "f32"))
        descs = [(p.rows, p.cols, p.kind, 1 if p.dtype == "bf16" else 0) for p in params]
        R = int(rng.integers(1, 10))
        shards, F, B = lib.mfsdp_plan(descs, R)
        entries, Fo, Bo = oracle.plan_owners(params, R)
        assert [(s.owner, s.owner_offset) for s in shards] == [(e.owner, e.owner_offset) for e in entries], trial
        assert F == Fo and B == Bo, trial
        R2 = int(rng.integers(1, 10))
        new, routes, moved = lib.mfsdp_reshard(descs, shards, R2)
        new_o, routes_o, moved_o = oracle.reshard(params, entries, R2)
        assert [(s.owner, s.owner_offset) for s in new] == [(e.owner, e.owner_offset) for e in new_o], trial
        assert [(r.src_rank, r.src_offset, r.dst_rank, r.dst_offset, r.state_bytes) for r in routes] == \
            [(o.src_rank, o.src_offset, o.dst_rank, o.dst_offset, o.state_bytes) for o in routes_o], trial
        assert moved == moved_o, trial


def test_tile_tables_cover_every_output_tile_once(lib):
    # mfsdp_muon_workspace_size builds the step's tile tables on the host and
    # rejects any table that misses or repeats an output tile; exercise it on
    # seeded random lists (ragged edges, r = 1, tall and wide) in both engines
    import numpy as np
    rng = np.random.default_rng(7)
    for trial in range(60):
        mats = []
        base = 1 << 20
        for i in range(int(rng.integers(1, 12))):
            r = int(rng.choice([1, 63, 64, 255, 256, 257, 600, 1100, 4096]))
            c = int(rng.choice([1, 64, 129, 256, 513, 2049, 11008]))
            mats.append(lib.Matrix(base, base + (1 << 28), base + (2 << 28), None, r, c, 1, 1))
            base += 3 << 28
        for mode in (lib.MFSDP_MODE_BF16, lib.MFSDP_MODE_FP32):
            ms = mats if mode == lib.MFSDP_MODE_BF16 else [
                lib.Matrix(m.param, m.grad, m.momentum, None, m.rows, m.cols, 0, 0) for m in mats]
            assert lib.mfsdp_muon_workspace_size(ms, lib.muon_hparams(mode=mode)) > 0, trial


def test_overlap_entry_points_validate_and_size(lib):
    hp = lib.muon_hparams()
    mats = [_mat(lib, 256, 512), _mat(lib, 300, 100, base=1 << 30), _mat(lib, 128, 128, base=1 << 31)]
    segs, keep = lib.owner_segments([[m.grad] for m in mats], [[(3 << 32) + (k << 24)] for k in range(len(mats))])
    one = lib.mfsdp_muon_workspace_size_p2p(mats, segs, hp)
    # one group: one region, the same size as the fused step's workspace
    assert lib.mfsdp_muon_workspace_size_p2p_overlap(mats, segs, hp, 1) == one
    # more groups: one region per group, each at least its own step's need
    assert lib.mfsdp_muon_workspace_size_p2p_overlap(mats, segs, hp, 3) >= one
    for bad in (0, 65):
        with pytest.raises(lib.MfsdpError) as e:
            lib.mfsdp_muon_workspace_size_p2p_overlap(mats, segs, hp, bad)
        assert e.value.status == lib.MFSDP_ERR_INVALID_ARG
    with pytest.raises(lib.MfsdpError) as e:
        lib.mfsdp_muon_step_p2p_overlap(mats, segs, hp, 0, 0, 0, 0, 0)
    assert e.value.status == lib.MFSDP_ERR_INVALID_ARG
