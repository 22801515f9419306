"""The five owner-step workloads: parameter lists, dtypes and draw recipes.

Shapes follow torch's Linear layout: rows = out features, cols = in features.
A workload lists the whole model's parameters.  Where a workload is an owner
share, the caller plans the list over ``world_size`` simulated data-parallel
ranks with an owner planner and steps the heaviest rank's matrices plus the
whole packed tail; this module does no planning itself.
"""

from __future__ import annotations

import dataclasses
from typing import Callable, Dict, List, Optional

import numpy as np

MATRIX = 0
TAIL = 1


@dataclasses.dataclass(frozen=True)
class ParamSpec:
    pid: int          # position in the model's parameter list
    name: str
    rows: int
    cols: int
    kind: int         # MATRIX or TAIL
    dtype: str        # "f32" or "bf16" (tail entries are always "f32")
    init: str = "weight"   # "weight" N(0, 0.02^2) | "norm" 1 + 0.01 N(0,1) | "generic" N(0, 0.02^2)

    @property
    def numel(self) -> int:
        return self.rows * self.cols


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    params: List[ParamSpec]
    world_size: Optional[int]      # None: one owner holds every matrix
    param_dtype: str               # dtype of matrices and their grads
    # grad draw: sigma per matrix and spike rank per matrix, both seeded
    sigma_rule: str                # "fixed:<v>" or "loguniform:<lo>:<hi>"
    spike_rule: str                # "rank:<r>:amp:<a>" (amp absolute) or "rank:<r>:rel:<k>" (k*sigma)
                                   # or "uniform:<lo>:<hi>:rel:<k>"
    description: str
    # optimizer hyper-parameters used for every workload
    lr: float = 0.02
    beta: float = 0.95
    weight_decay: float = 0.01
    adam_beta1: float = 0.9
    adam_beta2: float = 0.95
    adam_eps: float = 1e-8

    @property
    def matrices(self) -> List[ParamSpec]:
        return [p for p in self.params if p.kind == MATRIX]

    @property
    def tail(self) -> List[ParamSpec]:
        return [p for p in self.params if p.kind == TAIL]

    @property
    def tail_numel(self) -> int:
        return sum(p.numel for p in self.tail)


def _tiny() -> Workload:
    params = [
        ParamSpec(0, "w", 256, 512, MATRIX, "f32"),
        ParamSpec(1, "tail", 4096, 1, TAIL, "f32", "generic"),
    ]
    return Workload(
        name="tiny", seed=1001, params=params, world_size=None, param_dtype="f32",
        sigma_rule="fixed:1e-3", spike_rule="rank:1:amp:1e-2",
        description="one 256x512 fp32 weight, G = N(0,1e-3^2) + 1e-2 u v^T, 4096-element fp32 tail",
    )


def _llama_layer(pid0: int, layer: int, d: int, ffn: int, kv: int, dtype: str) -> List[ParamSpec]:
    names = [
        ("wq", d, d), ("wk", kv, d), ("wv", kv, d), ("wo", d, d),
        ("wgate", ffn, d), ("wup", ffn, d), ("wdown", d, ffn),
    ]
    return [ParamSpec(pid0 + i, f"layers.{layer}.{n}", r, c, MATRIX, dtype)
            for i, (n, r, c) in enumerate(names)]


def _block() -> Workload:
    params = _llama_layer(0, 0, 2048, 5504, 2048, "bf16")
    params += [ParamSpec(7, "layers.0.attn_norm", 2048, 1, TAIL, "f32", "norm"),
               ParamSpec(8, "layers.0.mlp_norm", 2048, 1, TAIL, "f32", "norm")]
    return Workload(
        name="block", seed=1002, params=params, world_size=None, param_dtype="bf16",
        sigma_rule="loguniform:1e-4:1e-2", spike_rule="rank:4:rel:10",
        description="one Llama block d=2048 ffn=5504 on one owner; bf16 params, fp32 momentum",
    )


def _seven_b() -> Workload:
    params: List[ParamSpec] = []
    d, ffn = 4096, 11008
    for layer in range(32):
        params += _llama_layer(len(params), layer, d, ffn, d, "bf16")
    for layer in range(32):
        params.append(ParamSpec(len(params), f"layers.{layer}.attn_norm", d, 1, TAIL, "f32", "norm"))
        params.append(ParamSpec(len(params), f"layers.{layer}.mlp_norm", d, 1, TAIL, "f32", "norm"))
    params.append(ParamSpec(len(params), "final_norm", d, 1, TAIL, "f32", "norm"))
    return Workload(
        name="7b_share", seed=1003, params=params, world_size=8, param_dtype="bf16",
        sigma_rule="loguniform:1e-4:1e-2", spike_rule="rank:4:rel:10",
        description="32-layer Llama d=4096 ffn=11008 planned over 8 ranks; heaviest share stepped",
    )


def _thirty_two_b() -> Workload:
    params: List[ParamSpec] = []
    d, ffn, kv = 5120, 27648, 1024
    for layer in range(64):
        params += _llama_layer(len(params), layer, d, ffn, kv, "bf16")
    params.append(ParamSpec(len(params), "tail", 1 << 20, 1, TAIL, "f32", "generic"))
    return Workload(
        name="32b_share", seed=1004, params=params, world_size=64, param_dtype="bf16",
        sigma_rule="loguniform:1e-4:1e-2", spike_rule="rank:8:rel:10",
        description="64-layer d=5120 ffn=27648 GQA (kv 1024) planned over 64 ranks; heaviest share stepped",
    )


def _skew() -> Workload:
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([1005, 7])))
    params: List[ParamSpec] = []
    rows = 128 * rng.integers(1, 33, size=512)
    cols = 128 * rng.integers(1, 33, size=512)
    for i in range(512):
        params.append(ParamSpec(len(params), f"skew.{i}", int(rows[i]), int(cols[i]), MATRIX, "bf16"))
    for i in range(8):
        params.append(ParamSpec(len(params), f"wide.{i}", 64, 16384, MATRIX, "bf16"))
    for i in range(8):
        params.append(ParamSpec(len(params), f"tall.{i}", 16384, 64, MATRIX, "bf16"))
    params.append(ParamSpec(len(params), "tail", 1 << 26, 1, TAIL, "f32", "generic"))
    return Workload(
        name="skew", seed=1005, params=params, world_size=None, param_dtype="bf16",
        sigma_rule="fixed:1e-3", spike_rule="uniform:1:16:rel:10",
        description="512 shapes (128*U{1..32})^2 + 8x 64x16384 + 8x 16384x64, 64 Mi-element tail",
    )


WORKLOADS: Dict[str, Callable[[], Workload]] = {
    "tiny": _tiny,
    "block": _block,
    "7b_share": _seven_b,
    "32b_share": _thirty_two_b,
    "skew": _skew,
}


def workload(name: str) -> Workload:
    try:
        return WORKLOADS[name]()
    except KeyError:
        raise KeyError(f"unknown workload {name!r}; known: {sorted(WORKLOADS)}") from None


def custom_workload(shapes, dtype: str = "bf16", tail: int = 0, seed: int = 4242,
                    sigma_rule: str = "fixed:1e-3", spike_rule: str = "rank:2:rel:10",
                    name: str = "custom") -> Workload:
    """A single-owner workload over explicit (rows, cols) shapes (test cases)."""
    params = [ParamSpec(i, f"m{i}", int(r), int(c), MATRIX, dtype) for i, (r, c) in enumerate(shapes)]
    if tail:
        params.append(ParamSpec(len(params), "tail", int(tail), 1, TAIL, "f32", "generic"))
    return Workload(name=name, seed=seed, params=params, world_size=None, param_dtype=dtype,
                    sigma_rule=sigma_rule, spike_rule=spike_rule, description=name)
