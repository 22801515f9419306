#!/usr/bin/env python3
"""Benchmark of the owner-local optimizer step (libmfsdp) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 7b_share] [--mode bf16]
    python bench.py --impl reference ...        # the fp64 oracle on host cores

One step = the owner's whole hot path over one batch of synthetic state: the
grouped Muon step over the owner's matrices (momentum, norm, five Newton-Schulz
iterations, scale, decay, write) plus AdamW over the packed tail, all through
the C ABI.  Default workload: the 7B owner share (a 32-layer Llama d=4096
ffn=11008 planned over 8 ranks; the heaviest rank's 28 matrices + the 266,240
element tail).  Under torchrun each rank steps its own planned share (weak
scaling, no collective on the data path); rank 0 prints one JSON line.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import tempfile
import sys
import time
from typing import Dict, List, Optional

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "owner-step latency (ms) & NS5 TFLOP/s at 7B owner share; tail AdamW GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SPEC_HBM_GBS = 8000.0      # B200 HBM3e, the nominal figure (for a second fraction beside the measured one)


# ---- host-side logic shared with the CPU tests --------------------------------------

def planned_share(params, world_size: int, rank: int, plan_fn, heaviest_fn):
    """Matrices (ParamSpec) and tail ownership of bench rank ``rank``: planned rank
    (heaviest + rank) mod world_size of an owner plan over ``world_size`` ranks."""
    shards, F, B = plan_fn(params, world_size)
    h = heaviest_fn(F, B)
    planned = (h + rank) % world_size
    mats = [p for p, s in zip(params, shards) if s.kind == 0 and s.owner == planned]
    owns_tail = any(s.kind != 0 and s.owner == planned for s in shards)
    return planned, mats, owns_tail, F[planned]


def product_plan(params, world_size):
    from matrix_optimizer_step_nesterov_b200 import mfsdp_plan
    descs = [(p.rows, p.cols, p.kind, 1 if p.dtype == "bf16" else 0) for p in params]
    return mfsdp_plan(descs, world_size)


def product_heaviest(F, B):
    from matrix_optimizer_step_nesterov_b200 import mfsdp_heaviest_rank
    return mfsdp_heaviest_rank(F, B)


def plan_balance(params, world_size: int) -> dict:
    """Balance of the owner plan over ``world_size`` ranks (host only): the
    heaviest rank's Newton-Schulz FLOPs and resident bytes over the per-rank
    means.  A multi-GPU step's makespan is the heaviest rank's step."""
    shards, F, B = product_plan(params, world_size)
    h = product_heaviest(F, B)
    mf, mb = sum(F) / len(F), sum(B) / len(B)
    return {"world_size": world_size, "heaviest_rank": h,
            "imbalance_flops": round(max(F) / mf, 6) if mf > 0 else None,
            "imbalance_bytes": round(max(B) / mb, 6) if mb > 0 else None,
            "ranks_with_matrices": sum(1 for f in F if f > 0)}


def ns_flops_algorithmic(specs, steps: int = 5) -> float:
    """Symmetric-exploiting work: per iteration r^2 c (A = X X^T, one triangle),
    r^3 (A A, one triangle) and 2 r^2 c (B X)."""
    tot = 0.0
    for s in specs:
        r, c = min(s.rows, s.cols), max(s.rows, s.cols)
        tot += steps * (3.0 * r * r * c + 1.0 * r ** 3)
    return tot


def ns_flops_dense(specs, steps: int = 5) -> float:
    tot = 0.0
    for s in specs:
        r, c = min(s.rows, s.cols), max(s.rows, s.cols)
        tot += steps * (4.0 * r * r * c + 2.0 * r ** 3)
    return tot


# Per-launch DRAM bytes of the GEMM phases at the 7B share, from ncu
# (dram__bytes_read.sum + dram__bytes_write.sum) on the 4-matrix case
# 2 x 4096^2 + 4096x11008 + 11008x4096: GRAM 0.4968 GB x 6.544, POLY 0.1116 GB x 7.0,
# APPLY 1.2954 GB x 6.544 (X's and A's element counts), averaged over 5 GRAM + 5 POLY
# + 5 APPLY/FINAL launches.
GEMM_TRAFFIC_7B = round((5 * 0.4968e9 * 6.544 + 5 * 0.1116e9 * 7.0 + 5 * 1.2954e9 * 6.544) / 15)


def split_groups(specs, n_groups: int) -> List[List[int]]:
    """Matrix-index groups for the pipelined e2e measurement.  With three or
    more groups the first and the last hold a single small matrix, so that the
    copies nothing overlaps (the first group's upload, the last group's
    download) stay short; the matrices between are split into groups of about
    equal dense NS FLOPs."""
    costs = [ns_flops_dense([s]) for s in specs]
    order = list(range(len(specs)))
    if n_groups >= 3 and len(specs) >= n_groups:
        by_size = sorted(order, key=lambda i: (costs[i], i))
        first, last = by_size[0], by_size[1]
        middle = [i for i in order if i not in (first, last)]
        return [[first]] + _balanced(middle, costs, n_groups - 2) + [[last]]
    return _balanced(order, costs, n_groups)


def _balanced(idx: List[int], costs: List[float], n_groups: int) -> List[List[int]]:
    total = sum(costs[i] for i in idx)
    groups: List[List[int]] = [[] for _ in range(max(1, n_groups))]
    acc, g = 0.0, 0
    for i in idx:
        if g < len(groups) - 1 and groups[g] and acc + costs[i] / 2 > total * (g + 1) / len(groups):
            g += 1
        groups[g].append(i)
        acc += costs[i]
    return [grp for grp in groups if grp]


def bench_workload(args):
    """The named workload, or a single-owner list of explicit shapes (--shapes RxC,RxC)."""
    from synth import workload
    from synth.workloads import custom_workload
    if args.shapes:
        shapes = [tuple(int(v) for v in sh.lower().split("x")) for sh in args.shapes.split(",")]
        dtype = "bf16" if args.mode == "bf16" else "f32"
        return custom_workload(shapes, dtype=dtype, tail=args.tail, seed=4242, spike_rule="rank:4:rel:10",
                               name="shapes " + args.shapes)
    wl = workload(args.workload)
    if args.seed is not None:                # a second draw of the same workload
        import dataclasses
        wl = dataclasses.replace(wl, seed=args.seed)
    return wl


def max_over_ranks(x: float) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    dev = torch.device("cuda") if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def load_peaks() -> Dict[str, float]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return dict(FALLBACK_PEAKS, source="fallback")


# ---- clocks ---------------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: Optional[str]):
        self.proc = None
        # raw samples: $MFSDP_CLOCKS_DIR (default: the temporary directory)
        out_dir = os.environ.get("MFSDP_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"clocks_{os.getpid()}.csv")
        self.gpu_index = gpu_index

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
            if self.gpu_index is not None:
                cmd += ["-i", self.gpu_index]
            self._f = open(self.path, "w")
            self.proc = subprocess.Popen(cmd, stdout=self._f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> Optional[dict]:
        if self.proc is None:
            return None
        try:
            self.proc.terminate()
            self.proc.wait(timeout=5)
        except Exception:
            try:
                self.proc.kill()
            except Exception:
                pass
        self._f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
                except ValueError:
                    continue
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3]) if v.lower() == "active"})
        loaded = [r for r in rows if r[2] > 200.0] or rows
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(loaded),
                "power_w_max": max(r[2] for r in rows)}


def gpu_index_of(dev: int) -> Optional[str]:
    try:
        import torch
        p = torch.cuda.get_device_properties(dev)
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except Exception:
        return None


# ---- oracle timing (cpu baseline / reference arm) ---------------------------------------------

def oracle_threads() -> int:
    import oracle
    return oracle.native.threads()


def oracle_share_estimate(wl, specs, tail_n: int, budget_s: float = 20.0):
    """Host time of the fp64 C++ oracle on the owner's whole step, from a bounded sample.

    The oracle's step on one matrix is momentum + norm + write (the same work
    whatever ns_steps is) plus ns_steps identical Newton-Schulz iterations, so
    its time is T(ns) = T(0) + ns (T(1) - T(0)).  For each distinct shape, in
    ascending size until ``budget_s`` is spent, one matrix is timed at ns = 0
    and ns = 1 and its full-step time taken from that line; shapes past the
    budget are extrapolated at the measured rate of dense Newton-Schulz FLOPs
    per second.  The per-shape times are scaled by the shape counts, and AdamW
    over the whole tail is added (timed whole).  Both benchmark arms use this
    one estimator.  Returns a dict: ms, sample text, seconds of oracle work
    measured, extrapolation factor (estimated / measured oracle seconds)."""
    import dataclasses
    import oracle
    from synth.gen import matrix_inputs, tail_inputs
    by_shape: Dict[tuple, list] = {}
    for s in specs:
        by_shape.setdefault((s.rows, s.cols), []).append(s)
    shapes = sorted(by_shape, key=lambda sh: ns_flops_dense([by_shape[sh][0]]))
    hp5 = oracle.MuonHParams()
    per_shape = {}
    spent = 0.0
    for sh in shapes:
        if per_shape and spent > budget_s:
            break
        mi = matrix_inputs(wl, by_shape[sh][0])
        t = []
        for ns in (0, 1):
            t0 = time.perf_counter()
            oracle.muon_step(mi.W, mi.G, mi.buf, dataclasses.replace(hp5, ns_steps=ns))
            t.append(time.perf_counter() - t0)
        spent += t[0] + t[1]
        per_shape[sh] = (t[0], t[1], t[0] + hp5.ns_steps * max(t[1] - t[0], 0.0))
    measured_flops = sum(ns_flops_dense([by_shape[sh][0]], steps=1) for sh in per_shape)
    rate = measured_flops / max(sum(v[1] - v[0] for v in per_shape.values()), 1e-9)
    total = 0.0
    for sh in shapes:
        full = per_shape[sh][2] if sh in per_shape else ns_flops_dense([by_shape[sh][0]]) / rate
        total += full * len(by_shape[sh])
    tail_s = 0.0
    if tail_n:
        ti = tail_inputs(wl)
        t0 = time.perf_counter()
        oracle.adamw_step(ti.p, ti.g, ti.m, ti.v, 1, oracle.AdamWHParams())
        tail_s = time.perf_counter() - t0
        spent += tail_s
    est_s = total + tail_s
    sample = (f"fp64 C++ oracle on {oracle_threads()} host threads: one matrix of each of {len(per_shape)}/"
              f"{len(shapes)} distinct shapes ({', '.join(f'{r}x{c}' for r, c in per_shape)}) timed at "
              f"ns_steps = 0 and 1, full step = T(0) + {hp5.ns_steps} (T(1) - T(0))"
              + (f", other shapes at the measured {rate / 1e9:.1f} GFLOP/s" if len(per_shape) < len(shapes) else "")
              + f", scaled by shape counts over {len(specs)} matrices; AdamW timed over the whole "
              f"{tail_n}-element tail; value extrapolated x{est_s / max(spent, 1e-9):.1f} from {spent:.1f} s "
              "of measured oracle work")
    return {"ms": est_s * 1e3, "sample": sample, "spent_s": spent,
            "extrapolation": est_s / max(spent, 1e-9), "gflops": rate / 1e9}


# ---- the GPU arm --------------------------------------------------------------------------------------

def run_ours(args) -> int:
    import torch
    import torch.distributed as dist
    from synth import workload
    from synth.gen import matrix_inputs_many, tail_inputs
    from matrix_optimizer_step_nesterov_b200 import MuonOwnerStep, adamw_tail, _lib

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: WORLD_SIZE={world} but --gpus {args.gpus}", file=sys.stderr)
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)

    wl = bench_workload(args)
    R = wl.world_size or 1
    if wl.world_size is None:
        specs, owns_tail, planned = wl.matrices, True, 0
    else:
        planned, specs, owns_tail, _ = planned_share(wl.params, R, rank, product_plan, product_heaviest)
    tail_n = wl.tail_numel if owns_tail else 0
    plan_info = plan_balance(wl.params, R) if wl.world_size else None

    t_gen = time.perf_counter()
    ins = matrix_inputs_many(wl, specs)
    dt = {"f32": torch.float32, "bf16": torch.bfloat16}
    Ws = [torch.from_numpy(i.W).to(dt[s.dtype]).to(dev) for i, s in zip(ins, specs)]
    Gs = [torch.from_numpy(i.G).to(dt[s.dtype]).to(dev) for i, s in zip(ins, specs)]
    Bs = [torch.from_numpy(i.buf).to(dev) for i in ins]
    if tail_n:
        ti = tail_inputs(wl)
        tp, tg, tm, tv = (torch.from_numpy(x).to(dev) for x in (ti.p, ti.g, ti.m, ti.v))
    gen_s = time.perf_counter() - t_gen

    step = MuonOwnerStep(Ws, Gs, Bs, mode=args.mode)
    stream = torch.cuda.current_stream()
    t_counter = [0]

    def one_step():
        step.step(stream)
        if tail_n:
            t_counter[0] += 1
            adamw_tail(tp, tg, tm, tv, t_counter[0], stream=stream)

    launches_per_step = step.launches + (1 if tail_n else 0)
    state_bytes = sum(s.numel * (2 * (2 if s.dtype == "bf16" else 4) + 4) for s in specs) + 16 * tail_n
    ws_bytes = step.workspace_bytes

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()

    def timed_steps(profile: bool):
        """K steps between a barrier and a synchronise on both sides; returns
        (ms per step over the region, per-step times, per-kernel-class profile).
        With profile, the library brackets each of its launches with two CUDA
        events on its launch stream (which also keeps consecutive phases from
        overlapping through programmatic dependent launch)."""
        if profile:
            _lib.mfsdp_profile_begin(args.steps * launches_per_step + 8)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev_steps = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ev0.record(stream)
        for k in range(args.steps):
            one_step()
            ev_steps[k].record(stream)       # per-step boundaries, for the median and minimum
        ev1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        prof_ = _lib.mfsdp_profile_end() if profile else {}
        per = [ev0.elapsed_time(ev_steps[0])] + [ev_steps[k - 1].elapsed_time(ev_steps[k])
                                                 for k in range(1, args.steps)]
        return ev0.elapsed_time(ev1) / args.steps, per, prof_

    # the timed region of `value`: the steps alone; then the same number of steps
    # again with per-kernel events, for the phase split and the rooflines
    sampler = ClockSampler(gpu_index_of(local)) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    ms_local, per_step, _ = timed_steps(profile=False)
    clocks = sampler.stop() if sampler else None
    ms = max_over_ranks(ms_local)
    step_stats = {"median_ms": round(max_over_ranks(statistics.median(per_step)), 4),
                  "min_ms": round(max_over_ranks(min(per_step)), 4),
                  "max_ms": round(max_over_ranks(max(per_step)), 4)}
    ms_prof_local, _, prof = timed_steps(profile=True)
    ms_prof = max_over_ranks(ms_prof_local)

    # e2e through host buffers: every gradient in (pinned H2D) and every updated
    # parameter out (D2H) each step.  The owner's matrices are split into
    # --e2e-groups groups stepped one after another through the same C ABI, so
    # that the copies of one group overlap the step of another.
    e2e = None
    if not args.no_e2e:
        hG = [g.cpu().pin_memory() for g in Gs]
        hW = [torch.empty(w.shape, dtype=w.dtype, pin_memory=True) for w in Ws]
        if tail_n:
            htg = tg.cpu().pin_memory()
            htp = torch.empty(tp.shape, dtype=tp.dtype, pin_memory=True)
        h2d = sum(g.numel() * g.element_size() for g in hG) + (htg.numel() * 4 if tail_n else 0)
        d2h = sum(w.numel() * w.element_size() for w in hW) + (htp.numel() * 4 if tail_n else 0)
        groups = split_groups(specs, max(1, min(args.e2e_groups, len(specs))))
        gsteps = [MuonOwnerStep([Ws[i] for i in grp], [Gs[i] for i in grp], [Bs[i] for i in grp], mode=args.mode)
                  for grp in groups]
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        # per group: its step of the previous call is done (its grads may be
        # overwritten), and its parameters of the previous call are on the host
        # (they may be updated again).  Consecutive steps overlap: a group's
        # upload for step k + 1 runs while later groups of step k compute.
        done_step = [None] * len(groups)
        done_d2h = [None] * len(groups)

        def e2e_step():
            ev_in = []
            with torch.cuda.stream(s_in):
                for g, grp in enumerate(groups):
                    if done_step[g] is not None:
                        s_in.wait_event(done_step[g])
                    for i in grp:
                        Gs[i].copy_(hG[i], non_blocking=True)
                    if g == 0 and tail_n:
                        tg.copy_(htg, non_blocking=True)
                    ev = torch.cuda.Event()
                    ev.record(s_in)
                    ev_in.append(ev)
            for g, grp in enumerate(groups):
                stream.wait_event(ev_in[g])
                if done_d2h[g] is not None:
                    stream.wait_event(done_d2h[g])
                gsteps[g].step(stream)
                if g == 0 and tail_n:
                    t_counter[0] += 1
                    adamw_tail(tp, tg, tm, tv, t_counter[0], stream=stream)
                ev = torch.cuda.Event()
                ev.record(stream)
                done_step[g] = ev
                s_out.wait_event(ev)
                with torch.cuda.stream(s_out):
                    for i in grp:
                        hW[i].copy_(Ws[i], non_blocking=True)
                    if g == 0 and tail_n:
                        htp.copy_(tp, non_blocking=True)
                    ev2 = torch.cuda.Event()
                    ev2.record(s_out)
                    done_d2h[g] = ev2

        for _ in range(max(1, min(args.warmup, 3))):
            e2e_step()
        stream.wait_stream(s_out)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        k_e2e = max(1, min(args.steps, 10))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        s_in.wait_stream(stream)                     # no upload starts before the timed region
        for _ in range(k_e2e):
            e2e_step()
        stream.wait_stream(s_out)                    # the region ends when the last parameter is on the host
        e1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / k_e2e)
        e2e = {"value": round(e2e_ms, 4), "unit": "ms", "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "steps": k_e2e, "groups": len(groups),
               "what": "per step: pinned H2D of every gradient (and the tail grad), the step through the C ABI "
                       f"in {len(groups)} groups whose copies overlap other groups' compute (also across "
                       "consecutive steps), D2H of every updated parameter (and the tail param); optimizer "
                       "state resident; value = (first upload to last download over the timed steps) / steps"}
        for st_ in gsteps:
            st_.close()
        del gsteps

    # 64 Mi-element tail (the skew workload's tail size): AdamW GB/s alone
    tail_bench = None
    if not args.no_tail_bench and rank == 0:
        n = 1 << 26
        P = torch.randn(n, device=dev) * 0.02
        Gt = torch.randn(n, device=dev) * 1e-3
        M = torch.zeros(n, device=dev)
        V = torch.zeros(n, device=dev)
        for t in range(1, 4):
            adamw_tail(P, Gt, M, V, t, stream=stream)
        k_t = max(5, args.steps)
        torch.cuda.synchronize()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for t in range(4, 4 + k_t):
            adamw_tail(P, Gt, M, V, t, stream=stream)
        a1.record(stream)
        torch.cuda.synchronize()
        t_ms = a0.elapsed_time(a1) / k_t
        tail_bench = {"elements": n, "ms": round(t_ms, 5), "gbs": round(28.0 * n / (t_ms * 1e-3) / 1e9, 1),
                      "bytes_per_elem": 28, "launches": k_t}
        del P, Gt, M, V

    if world > 1:
        dist.barrier()
    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return 0

    peaks = load_peaks()
    flops_alg = ns_flops_algorithmic(specs)
    flops_dense = ns_flops_dense(specs)
    gemm_ms = sum(prof.get(k, (0, 0.0))[1] for k in ("gram", "poly", "apply", "final"))
    gemm_launches = sum(prof.get(k, (0, 0))[0] for k in ("gram", "poly", "apply", "final"))
    steps_timed = args.steps
    ns_tflops_kernel = flops_alg * steps_timed / (gemm_ms * 1e-3) / 1e12 if gemm_ms > 0 else None
    ns_tflops_step = flops_alg / (ms * 1e-3) / 1e12
    if args.mode == "bf16":
        peak = peaks["bf16_tflops_sustained"]
        roof = {"bound": "tensor", "achieved": round(ns_tflops_kernel, 1) if ns_tflops_kernel else None,
                "peak": peak, "unit": "TFLOP/s",
                "frac": round(ns_tflops_kernel / peak, 4) if ns_tflops_kernel else None,
                # ncu dram__bytes_read.sum + dram__bytes_write.sum of one GRAM, POLY and APPLY launch on
                # 2 x 4096^2 + 4096x11008 + 11008x4096, scaled to the 7B share (GRAM and APPLY by X's
                # elements, POLY by A's) and averaged over a step's 15 GEMM launches
                "traffic": GEMM_TRAFFIC_7B if wl.name == "7b_share" else None,
                "traffic_note": "ncu DRAM bytes of one GRAM, POLY and APPLY launch on four 7B-share matrices, "
                                "scaled to the share and averaged over a step's GEMM launches"
                                if wl.name == "7b_share" else None,
                "kernel": "Newton-Schulz GEMM phases (gram + poly + apply + final launches)",
                "flops_per_launch": flops_alg * steps_timed / max(gemm_launches, 1),
                "avg_launch_ms": gemm_ms / max(gemm_launches, 1),
                "count": "algorithmic: per matrix per iteration r^2 c + r^3 + 2 r^2 c (symmetric halves)",
                "peak_kind": f"{peaks['source']} sustained cuBLAS bf16 (kernel timed inside a long step)"}
    else:
        # fp32 FFMA: 148 SMs x 128 lanes x 2 FLOP x clock
        mhz = (clocks or {}).get("sm_mhz") or 1965.0
        peak = 148 * 128 * 2 * mhz * 1e6 / 1e12
        roof = {"bound": "alu", "achieved": round(ns_tflops_kernel, 2) if ns_tflops_kernel else None,
                "peak": round(peak, 1), "unit": "TFLOP/s",
                "frac": round(ns_tflops_kernel / peak, 4) if ns_tflops_kernel else None, "traffic": None,
                "kernel": "Newton-Schulz GEMM phases on FFMA (fp32 mode)",
                "peak_kind": f"148 SMs x 128 FP32 lanes x 2 x {mhz:.0f} MHz (median SM clock under load)"}
    phases = {k: {"launches": v[0], "ms_total": round(v[1], 4), "ms_per_step": round(v[1] / steps_timed, 4)}
              for k, v in prof.items()}
    tail_roof = None
    if tail_bench:
        tail_roof = {"bound": "hbm", "achieved": tail_bench["gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(tail_bench["gbs"] / peaks["hbm_gbs"], 4),
                     "frac_of_spec": round(tail_bench["gbs"] / SPEC_HBM_GBS, 4),
                     # ncu dram__bytes_read.sum + dram__bytes_write.sum of one 64 Mi launch
                     "traffic": 1.8233e9 if tail_bench["elements"] == 64 << 20 else None,
                     "kernel": "AdamW tail, 64 Mi fp32 elements, 28 B/elem"}
    # the streaming kernels of the matrix step, from the same timed region
    n_elems = sum(s.numel for s in specs)
    wbytes = 2 if all(s.dtype == "bf16" for s in specs) else 4
    hbm_kernels = {
        # bf16 mode: G 2 + buf 4 in, buf 4 + X hi 2 + X lo 2 out; fp32 mode: G 4 + buf 4 in, buf 4 + X 4 out
        "momentum": n_elems * (14 if args.mode == "bf16" else 16),
        # bf16 mode: X hi 2 + X lo 2 + W in, W out; fp32 mode: X 4 + W in, W out
        "write": n_elems * (4 + 2 * wbytes),
    }
    roof_hbm = {}
    for k, nbytes in hbm_kernels.items():
        v = prof.get(k)
        if v and v[1] > 0:
            gbs = nbytes * v[0] / (v[1] * 1e-3) / 1e9
            roof_hbm[k] = {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                           "frac": round(gbs / peaks["hbm_gbs"], 4), "frac_of_spec": round(gbs / SPEC_HBM_GBS, 4),
                           "bytes_per_launch": nbytes, "avg_launch_ms": round(v[1] / v[0], 5)}
    mom_gbs = roof_hbm.get("momentum", {}).get("achieved")

    cpu_baseline = None
    if world == 1 and not args.no_cpu_baseline:
        est = oracle_share_estimate(wl, specs, tail_n, budget_s=args.cpu_budget)
        cpu_baseline = {"value": round(est["ms"], 1), "unit": "ms", "cores": oracle_threads(), "kind": "oracle",
                        "sample": est["sample"], "cpu_seconds_spent": round(est["spent_s"], 1),
                        "extrapolation": round(est["extrapolation"], 2)}

    line = {
        "metric": METRIC,
        "value": round(ms, 4),
        "unit": "ms",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 4),
        "step_ms": step_stats,
        "ms_per_step_profiled": round(ms_prof, 4),
        "timing": "value: CUDA events around K steps on the launch stream, barrier and synchronise on both "
                  "sides; phases and rooflines: the same K steps again with two CUDA events around each library "
                  "launch (ms_per_step_profiled)",
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if args.mode == "bf16" else "f32",
        "data": "synthetic",
        "config": {
            "workload": f"{wl.name}: {wl.description}; planned rank {planned} of {R}",
            "matrices": len(specs), "tail_elements": tail_n, "mode": args.mode,
            "state_bytes_resident": state_bytes, "workspace_bytes": ws_bytes,
            "l2": "inputs larger than L2 (126 MB); no flush between steps",
            "parallelism": f"owner shards: each of {world} rank(s) steps its own planned share, no collective",
        },
        "ns_tflops": {"algorithmic_per_gemm_time": round(ns_tflops_kernel, 1) if ns_tflops_kernel else None,
                      "algorithmic_per_step_time": round(ns_tflops_step, 1),
                      "dense_equivalent_per_gemm_time": round(flops_dense * steps_timed / (gemm_ms * 1e-3) / 1e12, 1)
                      if gemm_ms > 0 else None,
                      "flops_algorithmic_per_step": flops_alg, "flops_dense_per_step": flops_dense},
        "tail_gbs": tail_bench["gbs"] if tail_bench else None,
        "tail_64Mi": tail_bench,
        "momentum_gbs": mom_gbs,
        "roofline": roof,
        "roofline_tail": tail_roof,
        "roofline_hbm": roof_hbm or None,
        "plan": plan_info,
        "phases": phases,
        "cpu_baseline": cpu_baseline,
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "peaks": peaks,
        "setup_seconds": round(gen_s, 1),
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


# ---- the reference arm: the oracle on host cores -------------------------------------------------------

def run_reference(args) -> int:
    """The reference arm: the fp64 C++ oracle on the host cores, as it stands.
    Each step runs the same bounded-sample estimator as the GPU arm's
    cpu_baseline leg; warm-up steps run it on the smallest shape only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    wl = bench_workload(args)
    R = wl.world_size or 1
    if wl.world_size is None:
        specs, owns_tail = wl.matrices, True
    else:
        _, specs, owns_tail, _ = planned_share(wl.params, R, 0, oracle.plan_owners, oracle.heaviest_rank)
    tail_n = wl.tail_numel if owns_tail else 0
    smallest = [min(specs, key=lambda s: ns_flops_dense([s]))]
    for _ in range(args.warmup):
        oracle_share_estimate(wl, smallest, 0, budget_s=0.0)
    ests = [oracle_share_estimate(wl, specs, tail_n, budget_s=args.cpu_budget) for _ in range(args.steps)]
    v = statistics.median(e["ms"] for e in ests)
    spent = sum(e["spent_s"] for e in ests)
    line = {
        "impl": "reference",
        "metric": METRIC, "value": round(v, 1), "unit": "ms", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(v, 1), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{wl.name}: {wl.description}", "matrices": len(specs), "tail_elements": tail_n},
        "cpu_baseline": {"value": round(v, 1), "unit": "ms", "cores": oracle_threads(), "kind": "oracle",
                         "sample": "each step (median of the steps): " + ests[-1]["sample"],
                         "cpu_seconds_spent": round(spent, 1),
                         "extrapolation": round(statistics.median(e["extrapolation"] for e in ests), 2)},
        "e2e": {"value": round(v, 1), "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="7b_share")
    ap.add_argument("--mode", default="bf16", choices=["bf16", "fp32"])
    ap.add_argument("--shapes", default="", help="explicit matrix list RxC,RxC (profiling cases) instead of --workload")
    ap.add_argument("--tail", type=int, default=0, help="tail length with --shapes")
    ap.add_argument("--seed", type=int, default=None, help="input seed instead of the workload's own")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-groups", type=int, default=6, help="matrix groups pipelined in the e2e measurement")
    ap.add_argument("--no-tail-bench", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=10.0,
                    help="seconds of oracle work after which unmeasured shapes are extrapolated")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        print("note: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
