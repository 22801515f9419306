"""Test harness: seeded inputs -> (GPU path through the C ABI, fp64 oracle) -> metrics.

The two sides share only the seeded inputs from ``synth``.  The GPU side goes
through ``matrix_optimizer_step_nesterov_b200`` (libmfsdp); the oracle side
through ``oracle`` (its fp64 C++ library).  No expected value is ever taken from the GPU path except
where a check is explicitly "given the GPU's own O" (the parameter-write
check, which tests the write alone).
"""

from __future__ import annotations

import dataclasses
import os
from typing import Dict, List, Optional, Sequence

import numpy as np
import torch

import oracle
from synth import workloads as W
from synth.gen import matrix_inputs_many, tail_inputs, round_to  # noqa: F401

TOL_O = {"fp32": 1e-4, "bf16": 2e-2}
TOL_BUF = 1e-6
TOL_ADAMW = 1e-6

_TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def rel_frob(x: np.ndarray, ref: np.ndarray) -> float:
    den = float(np.linalg.norm(ref))
    num = float(np.linalg.norm(np.asarray(x, np.float64) - ref))
    return num / den if den > 0 else num


def ordered_bits(x: torch.Tensor) -> np.ndarray:
    """Map float32 / bfloat16 values to integers whose difference counts ulps."""
    if x.dtype == torch.bfloat16:
        i = x.view(torch.int16).to(torch.int64).numpy()
        return np.where(i < 0, -(i & 0x7FFF), i)
    i = x.to(torch.float32).view(torch.int32).to(torch.int64).numpy()
    return np.where(i < 0, -(i & 0x7FFFFFFF), i)


def ulp_distance(a: torch.Tensor, b: torch.Tensor) -> np.ndarray:
    return np.abs(ordered_bits(a) - ordered_bits(b))


def owner_share(wl: W.Workload):
    """The matrices a workload steps: all of them, or the heaviest planned rank's
    (planned with the oracle's planner; the product planner is tested equal)."""
    if wl.world_size is None:
        return wl.matrices
    entries, F, B = oracle.plan_owners(wl.params, wl.world_size)
    h = oracle.heaviest_rank(F, B)
    by_pid = {p.pid: p for p in wl.params}
    return [by_pid[e.pid] for e in entries if e.owner == h and e.kind == W.MATRIX]


@dataclasses.dataclass
class HostState:
    specs: List[W.ParamSpec]
    W: List[np.ndarray]
    G: List[np.ndarray]
    buf: List[np.ndarray]


def host_state(wl: W.Workload, specs: Sequence[W.ParamSpec], step: int = 0, buf_init: str = "zeros") -> HostState:
    ins = matrix_inputs_many(wl, specs, step=step, buf_init=buf_init)
    return HostState(list(specs), [i.W for i in ins], [i.G for i in ins], [i.buf for i in ins])


@dataclasses.dataclass
class GpuResult:
    W: List[torch.Tensor]      # cpu tensors in the param dtype
    O: List[Optional[np.ndarray]]
    buf: List[np.ndarray]


def gpu_step(hs: HostState, mode: str, want_o: Optional[Sequence[int]] = None, ns_steps: int = 5,
             nesterov: bool = True, lr: float = 0.02, beta: float = 0.95, weight_decay: float = 0.01,
             grads: Optional[List[np.ndarray]] = None, repeat: int = 1, keep: Optional[Sequence[int]] = None
             ) -> GpuResult:
    """Run the product step over every matrix of ``hs`` in ONE grouped call
    (``repeat`` calls in a row with the same gradients).  ``keep`` limits the
    matrices whose W and momentum are copied back (default: all)."""
    from matrix_optimizer_step_nesterov_b200 import MuonOwnerStep
    dev = torch.device("cuda")
    want = set(range(len(hs.specs))) if want_o is None else set(want_o)
    kept = set(range(len(hs.specs))) if keep is None else set(keep)
    params, gs, bufs, outs = [], [], [], []
    for k, s in enumerate(hs.specs):
        dt = _TORCH_DT[s.dtype]
        params.append(torch.from_numpy(hs.W[k]).to(dt).to(dev))
        g = hs.G[k] if grads is None else grads[k]
        gs.append(torch.from_numpy(g).to(dt).to(dev))
        bufs.append(torch.from_numpy(hs.buf[k]).to(dev))
        outs.append(torch.empty(s.rows, s.cols, dtype=torch.float32, device=dev) if k in want else None)
    step = MuonOwnerStep(params, gs, bufs, outs, lr=lr, beta=beta, weight_decay=weight_decay,
                         ns_steps=ns_steps, nesterov=nesterov, mode=mode)
    for _ in range(repeat):
        step.step()
    torch.cuda.synchronize()
    res = GpuResult([p.cpu() if k in kept else None for k, p in enumerate(params)],
                    [o.cpu().numpy().astype(np.float64) if o is not None else None for o in outs],
                    [b.cpu().numpy() if k in kept else None for k, b in enumerate(bufs)])
    step.close()
    del params, gs, bufs, outs
    return res


def f32(x: float) -> float:
    """A hyper-parameter as the library receives it (the ABI takes fp32)."""
    return float(np.float32(x))


def muon_hparams_as_passed(ns_steps: int = 5, nesterov: bool = True, lr: float = 0.02, beta: float = 0.95,
                           weight_decay: float = 0.01) -> "oracle.MuonHParams":
    d = oracle.MuonHParams()
    return oracle.MuonHParams(lr=f32(lr), beta=f32(beta), weight_decay=f32(weight_decay), eps=f32(d.eps),
                              a=f32(d.a), b=f32(d.b), c=f32(d.c), ns_steps=ns_steps, nesterov=nesterov)


def adamw_hparams_as_passed(lr=0.02, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.01) -> "oracle.AdamWHParams":
    return oracle.AdamWHParams(lr=f32(lr), beta1=f32(beta1), beta2=f32(beta2), eps=f32(eps),
                               weight_decay=f32(weight_decay))


def oracle_step(hs: HostState, k: int, ns_steps: int = 5, nesterov: bool = True, lr: float = 0.02,
                beta: float = 0.95, weight_decay: float = 0.01):
    """The oracle on the same inputs as the GPU, hyper-parameters included (fp32 values)."""
    hp = muon_hparams_as_passed(ns_steps, nesterov, lr, beta, weight_decay)
    return oracle.muon_step(hs.W[k].astype(np.float64), hs.G[k].astype(np.float64),
                            hs.buf[k].astype(np.float64), hp)


def dtype_spacing(x: np.ndarray, dtype: torch.dtype) -> np.ndarray:
    """One ulp of the storage dtype at |x| (normal range; bf16 keeps 8 of fp32's 24 bits)."""
    sp = np.spacing(np.abs(x).astype(np.float32)).astype(np.float64)
    return sp * 65536.0 if dtype == torch.bfloat16 else sp


def check_write(W0: np.ndarray, O_gpu: np.ndarray, W_gpu: torch.Tensor, lr: float = 0.02,
                wd: float = 0.01) -> Dict[str, float]:
    """The parameter write given the GPU's own O: W_ref = W0 (1 - lr wd) - lr O_gpu
    in fp64, rounded once to the parameter dtype.  The bound per element is
    2 ulp of the stored dtype at |W_ref| plus 2 fp32 ulps at the larger
    operand max(|W0|, lr |O|): the write is computed in fp32, whose rounding
    of the operands cannot be smaller than that when the two terms cancel.
    Returns the max ulp distance (informational) and the max error / bound."""
    if W0.size == 0:
        return {"write_ulp": 0, "write_excess": 0.0}
    ref = W0.astype(np.float64) * (1.0 - lr * wd) - lr * O_gpu
    ref_t = torch.from_numpy(ref).to(W_gpu.dtype)
    ulp = int(ulp_distance(W_gpu, ref_t).max())
    got = W_gpu.to(torch.float64).numpy()
    scale = np.maximum(np.abs(W0.astype(np.float64)), lr * np.abs(O_gpu))
    bound = 2.0 * dtype_spacing(ref, W_gpu.dtype) + 2.0 * dtype_spacing(scale, torch.float32)
    excess = float(np.max(np.abs(got - ref) / bound))
    return {"write_ulp": ulp, "write_excess": excess}


def compare_matrix(hs: HostState, res: GpuResult, k: int, mode: str, ref=None, **kw) -> Dict[str, float]:
    """Errors of matrix k of a GPU result against the oracle on the same inputs
    (``ref`` = a precomputed oracle_step(hs, k, **kw), else computed here)."""
    Wn, O, bn = ref if ref is not None else oracle_step(hs, k, **kw)
    out = {"rel_O": rel_frob(res.O[k], O) if res.O[k] is not None else float("nan"),
           "rel_buf": rel_frob(res.buf[k], bn)}
    if res.O[k] is not None:
        out.update(check_write(hs.W[k], res.O[k], res.W[k],
                               lr=kw.get("lr", 0.02), wd=kw.get("weight_decay", 0.01)))
    return out


def _report(metrics: Dict[str, float], mode: str, label: str) -> None:
    """Append the measured errors to the JSON-lines file named by
    MFSDP_PARITY_REPORT, when set (error margins for the design notes)."""
    path = os.environ.get("MFSDP_PARITY_REPORT")
    if not path:
        return
    import json
    rec = {"label": label, "mode": mode}
    rec.update({k: (float(v) if isinstance(v, (int, float, np.floating, np.integer)) else v)
                for k, v in metrics.items()})
    with open(path, "a") as f:
        f.write(json.dumps(rec) + "\n")


def assert_parity(metrics: Dict[str, float], mode: str, label: str = "") -> None:
    _report(metrics, mode, label)
    assert metrics["rel_O"] <= TOL_O[mode], f"{label} rel Frobenius error of O {metrics['rel_O']:.3e} > {TOL_O[mode]}"
    assert metrics["rel_buf"] <= TOL_BUF, f"{label} momentum rel error {metrics['rel_buf']:.3e}"
    if "write_excess" in metrics:
        assert metrics["write_excess"] <= 1.0, (
            f"{label} parameter write error {metrics['write_excess']:.2f}x its bound "
            f"(max {metrics['write_ulp']} ulp)")


# ---- AdamW ----------------------------------------------------------------------

def adamw_tolerance_ok(x: np.ndarray, ref: np.ndarray) -> bool:
    """|d| <= 1e-6 |ref| + 2^-23 max|ref| per element (the floor covers cancellation)."""
    if ref.size == 0:
        return True
    d = np.abs(np.asarray(x, np.float64) - ref)
    bound = TOL_ADAMW * np.abs(ref) + 2.0 ** -23 * float(np.max(np.abs(ref)))
    return bool(np.all(d <= bound))


def gpu_adamw(p, g, m, v, t, offset: int = 0, **hp):
    from matrix_optimizer_step_nesterov_b200 import adamw_tail
    dev = torch.device("cuda")
    n = p.size

    def up(x):
        buf = torch.zeros(n + offset, dtype=torch.float32, device=dev)
        buf[offset:] = torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(dev)
        return buf, buf[offset:]

    (_, P), (_, G), (_, M), (_, V) = up(p), up(g), up(m), up(v)
    adamw_tail(P, G, M, V, t, **hp)
    torch.cuda.synchronize()
    return P.cpu().numpy(), M.cpu().numpy(), V.cpu().numpy()


def gpu_available() -> bool:
    return torch.cuda.is_available()


def lib_built() -> bool:
    from matrix_optimizer_step_nesterov_b200 import _lib
    return os.path.exists(_lib.LIB_PATH)
