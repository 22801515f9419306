"""Seeded draws of a workload's state: weights, gradients, momentum, tail.

Every draw comes from its own counter-free PCG64 stream keyed by
``(workload seed, parameter id, step, purpose)``, so any single matrix can be
regenerated without drawing the others, and the GPU path and the oracle see
bit-identical inputs.

Values are returned as float32 numpy arrays whose entries are exactly
representable in the parameter's storage dtype (bf16 values are rounded to
nearest-even once, here).
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

from .workloads import ParamSpec, Workload

# purposes of the random streams
_W, _G_SIGMA, _G_NOISE, _G_SPIKE, _BUF, _TAIL_P, _TAIL_G, _TAIL_M, _TAIL_V = range(9)


def param_seed(workload_seed: int, pid: int, step: int, purpose: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([workload_seed, pid, step, purpose])))


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """float32 array -> float32 array holding values of ``dtype`` (RNE)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "f32":
        return x
    if dtype == "bf16":
        return torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    raise ValueError(dtype)


@dataclasses.dataclass
class MatrixInputs:
    spec: ParamSpec
    W: np.ndarray      # rows x cols, float32 holding values of spec.dtype
    G: np.ndarray      # rows x cols, float32 holding values of spec.dtype
    buf: np.ndarray    # rows x cols, float32 momentum buffer
    sigma: float
    spike_rank: int


def _sigma(rule: str, rng: np.random.Generator) -> float:
    kind, *args = rule.split(":")
    if kind == "fixed":
        return float(args[0])
    if kind == "loguniform":
        lo, hi = math.log(float(args[0])), math.log(float(args[1]))
        return float(math.exp(rng.uniform(lo, hi)))
    raise ValueError(rule)


def _spike(rule: str, sigma: float, rng: np.random.Generator):
    parts = rule.split(":")
    if parts[0] == "rank":
        rank = int(parts[1])
        rest = parts[2:]
    elif parts[0] == "uniform":
        rank = int(rng.integers(int(parts[1]), int(parts[2]) + 1))
        rest = parts[3:]
    else:
        raise ValueError(rule)
    amp = float(rest[1]) if rest[0] == "amp" else float(rest[1]) * sigma
    return rank, amp


def draw_grad(wl: Workload, spec: ParamSpec, step: int = 0):
    """G = sigma * N(0,1) + amp * sum_k u_k v_k^T, u_k, v_k with N(0,1) entries."""
    rng_s = param_seed(wl.seed, spec.pid, step, _G_SIGMA)
    sigma = _sigma(wl.sigma_rule, rng_s)
    rank, amp = _spike(wl.spike_rule, sigma, rng_s)
    rng_n = param_seed(wl.seed, spec.pid, step, _G_NOISE)
    G = rng_n.standard_normal((spec.rows, spec.cols), dtype=np.float32)
    G *= np.float32(sigma)
    if rank > 0 and amp != 0.0:
        rng_k = param_seed(wl.seed, spec.pid, step, _G_SPIKE)
        U = rng_k.standard_normal((spec.rows, rank), dtype=np.float32)
        V = rng_k.standard_normal((spec.cols, rank), dtype=np.float32)
        G += np.float32(amp) * (U @ V.T)
    return round_to(G, spec.dtype), sigma, rank


def draw_weight(wl: Workload, spec: ParamSpec) -> np.ndarray:
    rng = param_seed(wl.seed, spec.pid, 0, _W)
    W = rng.standard_normal((spec.rows, spec.cols), dtype=np.float32)
    W *= np.float32(0.02)
    return round_to(W, spec.dtype)


def matrix_inputs(wl: Workload, spec: ParamSpec, step: int = 0,
                  buf_init: str = "zeros") -> MatrixInputs:
    """State of one matrix before optimizer step ``step`` (grads differ per step).

    ``buf_init`` is "zeros" (first step) or "random" (a non-trivial momentum
    buffer with N(0, (1e-3)^2) entries, for multi-step parity cases).
    """
    W = draw_weight(wl, spec)
    G, sigma, rank = draw_grad(wl, spec, step)
    if buf_init == "zeros":
        buf = np.zeros((spec.rows, spec.cols), np.float32)
    elif buf_init == "random":
        rng = param_seed(wl.seed, spec.pid, step, _BUF)
        buf = rng.standard_normal((spec.rows, spec.cols), dtype=np.float32) * np.float32(1e-3)
    else:
        raise ValueError(buf_init)
    return MatrixInputs(spec, W, G, buf, sigma, rank)


def matrix_inputs_many(wl: Workload, specs, step: int = 0, buf_init: str = "zeros",
                       threads: Optional[int] = None):
    """matrix_inputs for many matrices, drawn in parallel threads (same values
    as drawing them one by one: every matrix has its own streams)."""
    import concurrent.futures as cf
    import os
    n = threads or min(32, os.cpu_count() or 1)
    with cf.ThreadPoolExecutor(max_workers=n) as ex:
        return list(ex.map(lambda s: matrix_inputs(wl, s, step=step, buf_init=buf_init), specs))


@dataclasses.dataclass
class TailInputs:
    p: np.ndarray
    g: np.ndarray
    m: np.ndarray
    v: np.ndarray


def tail_inputs(wl: Workload, step: int = 0, state: str = "zeros",
                numel: Optional[int] = None) -> TailInputs:
    """The packed fp32 tail: every TAIL parameter of the workload, concatenated
    in parameter-list order.  ``state`` "zeros" gives m = v = 0 (first step);
    "random" gives m ~ N(0,(1e-3)^2), v ~ U(0, 2e-6) (a warmed-up state).
    ``numel`` truncates the tail (bounded samples)."""
    parts_p, parts_g = [], []
    for spec in wl.tail:
        rng = param_seed(wl.seed, spec.pid, 0, _TAIL_P)
        x = rng.standard_normal(spec.numel, dtype=np.float32)
        if spec.init == "norm":
            x = np.float32(1.0) + np.float32(0.01) * x
        else:
            x *= np.float32(0.02)
        parts_p.append(x)
        rng_g = param_seed(wl.seed, spec.pid, step, _TAIL_G)
        parts_g.append(rng_g.standard_normal(spec.numel, dtype=np.float32) * np.float32(1e-3))
    p = np.concatenate(parts_p) if parts_p else np.zeros(0, np.float32)
    g = np.concatenate(parts_g) if parts_g else np.zeros(0, np.float32)
    if numel is not None:
        p, g = p[:numel].copy(), g[:numel].copy()
    n = p.size
    if state == "zeros":
        m = np.zeros(n, np.float32)
        v = np.zeros(n, np.float32)
    elif state == "random":
        rng = param_seed(wl.seed, 1 << 30, step, _TAIL_M)
        m = rng.standard_normal(n, dtype=np.float32) * np.float32(1e-3)
        rng = param_seed(wl.seed, 1 << 30, step, _TAIL_V)
        v = rng.uniform(0.0, 2e-6, n).astype(np.float32)
    else:
        raise ValueError(state)
    return TailInputs(p, g, m, v)
