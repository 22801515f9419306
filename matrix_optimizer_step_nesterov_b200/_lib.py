"""ctypes binding of libmfsdp (include/mfsdp.h): same names, marshalling only.

Every step of the owner update runs in the library's CUDA kernels; this module
only converts Python values and torch tensors into the C structs and raw
pointers the ABI takes.  It raises if the shared library is missing: there is
no fallback path.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmfsdp.so")

MFSDP_OK = 0
MFSDP_ERR_INVALID_ARG = -1
MFSDP_ERR_UNSUPPORTED_DTYPE = -2
MFSDP_ERR_MISALIGNED = -3
MFSDP_ERR_WORKSPACE_TOO_SMALL = -4
MFSDP_ERR_CUDA = -5
MFSDP_ERR_TIMEOUT = -6
MFSDP_ERR_DEVICE_FAULT = -7
MFSDP_ERR_UNSUPPORTED_DEVICE = -8

MFSDP_DTYPE_F32 = 0
MFSDP_DTYPE_BF16 = 1
MFSDP_KIND_MATRIX = 0
MFSDP_KIND_TAIL = 1
MFSDP_MODE_FP32 = 0
MFSDP_MODE_BF16 = 1

# every symbol include/mfsdp.h declares
EXPORTED = (
    "mfsdp_plan", "mfsdp_heaviest_rank", "mfsdp_muon_workspace_size", "mfsdp_muon_step",
    "mfsdp_muon_step_launches", "mfsdp_muon_forget_workspace", "mfsdp_adamw_tail",
    "mfsdp_get_device_status", "mfsdp_status_string", "mfsdp_version",
    "mfsdp_profile_begin", "mfsdp_profile_end", "mfsdp_muon_step_noalloc",
    "mfsdp_muon_workspace_size_p2p", "mfsdp_muon_step_p2p", "mfsdp_selftest_bounded_wait",
    "mfsdp_reshard", "mfsdp_muon_workspace_size_p2p_overlap", "mfsdp_muon_step_p2p_overlap",
    "mfsdp_muon_forget_workspace_range",
)

MFSDP_MAX_PARTS = 64
MFSDP_MAX_COPIES = 64

KCLASS_NAMES = ("momentum", "norm", "gram", "poly", "apply", "write", "adamw", "final")


class MfsdpError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


class ParamDesc(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("kind", ctypes.c_int32), ("dtype", ctypes.c_int32)]


class MatrixShard(ctypes.Structure):
    _fields_ = [("param_id", ctypes.c_int64), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("owner", ctypes.c_int32), ("kind", ctypes.c_int32), ("transposed", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("ns_flops", ctypes.c_double),
                ("resident_bytes", ctypes.c_int64), ("owner_offset", ctypes.c_int64),
                ("shape_scale", ctypes.c_double)]


class ReshardRoute(ctypes.Structure):
    _fields_ = [("param_id", ctypes.c_int64), ("kind", ctypes.c_int32), ("src_rank", ctypes.c_int32),
                ("dst_rank", ctypes.c_int32), ("reserved", ctypes.c_int32), ("src_offset", ctypes.c_int64),
                ("dst_offset", ctypes.c_int64), ("elems", ctypes.c_int64), ("state_bytes", ctypes.c_int64)]


class Matrix(ctypes.Structure):
    _fields_ = [("param", ctypes.c_void_p), ("grad", ctypes.c_void_p), ("momentum", ctypes.c_void_p),
                ("update_out", ctypes.c_void_p), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("param_dtype", ctypes.c_int32), ("grad_dtype", ctypes.c_int32)]


class MuonHParams(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta", ctypes.c_float), ("weight_decay", ctypes.c_float),
                ("eps", ctypes.c_float), ("a", ctypes.c_float), ("b", ctypes.c_float), ("c", ctypes.c_float),
                ("ns_steps", ctypes.c_int32), ("nesterov", ctypes.c_int32), ("mode", ctypes.c_int32)]


class AdamWHParams(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("eps", ctypes.c_float), ("weight_decay", ctypes.c_float), ("reserved", ctypes.c_int32),
                ("step", ctypes.c_int64)]


class OwnerSegments(ctypes.Structure):
    _fields_ = [("grad_parts", ctypes.POINTER(ctypes.c_void_p)), ("param_copies", ctypes.POINTER(ctypes.c_void_p)),
                ("nparts", ctypes.c_int32), ("ncopies", ctypes.c_int32)]


class Profile(ctypes.Structure):
    _fields_ = [("launches", ctypes.c_int32 * 8), ("ms", ctypes.c_double * 8)]


_lib: Optional[ctypes.CDLL] = None


def load() -> ctypes.CDLL:
    """Load libmfsdp.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libmfsdp.so not built at {LIB_PATH}; run "
                          "`python -m matrix_optimizer_step_nesterov_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    i32, i64, p = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p
    lib.mfsdp_plan.argtypes = [ctypes.POINTER(ParamDesc), i64, i32, i32, ctypes.POINTER(MatrixShard),
                               ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)]
    lib.mfsdp_plan.restype = ctypes.c_int
    lib.mfsdp_heaviest_rank.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64), i32,
                                        ctypes.POINTER(ctypes.c_int32)]
    lib.mfsdp_heaviest_rank.restype = ctypes.c_int
    lib.mfsdp_reshard.argtypes = [ctypes.POINTER(ParamDesc), ctypes.POINTER(MatrixShard), i64, i32, i32,
                                  ctypes.POINTER(MatrixShard), ctypes.POINTER(ReshardRoute),
                                  ctypes.POINTER(ctypes.c_int64)]
    lib.mfsdp_reshard.restype = ctypes.c_int
    lib.mfsdp_muon_workspace_size.argtypes = [ctypes.POINTER(Matrix), i32, ctypes.POINTER(MuonHParams),
                                              ctypes.POINTER(ctypes.c_size_t)]
    lib.mfsdp_muon_workspace_size.restype = ctypes.c_int
    lib.mfsdp_muon_step.argtypes = [ctypes.POINTER(Matrix), i32, ctypes.POINTER(MuonHParams), p,
                                    ctypes.c_size_t, p]
    lib.mfsdp_muon_step.restype = ctypes.c_int
    lib.mfsdp_muon_step_launches.argtypes = [ctypes.POINTER(Matrix), i32, ctypes.POINTER(MuonHParams),
                                             ctypes.POINTER(ctypes.c_int32)]
    lib.mfsdp_muon_step_launches.restype = ctypes.c_int
    lib.mfsdp_muon_forget_workspace.argtypes = [p]
    lib.mfsdp_muon_forget_workspace.restype = ctypes.c_int
    lib.mfsdp_muon_forget_workspace_range.argtypes = [p, ctypes.c_size_t]
    lib.mfsdp_muon_forget_workspace_range.restype = ctypes.c_int
    lib.mfsdp_adamw_tail.argtypes = [p, p, p, p, i64, ctypes.POINTER(AdamWHParams), p]
    lib.mfsdp_adamw_tail.restype = ctypes.c_int
    lib.mfsdp_get_device_status.argtypes = [p, ctypes.POINTER(ctypes.c_int32)]
    lib.mfsdp_get_device_status.restype = ctypes.c_int
    lib.mfsdp_status_string.argtypes = [i32]
    lib.mfsdp_status_string.restype = ctypes.c_char_p
    lib.mfsdp_profile_begin.argtypes = [i32]
    lib.mfsdp_profile_begin.restype = ctypes.c_int
    lib.mfsdp_profile_end.argtypes = [ctypes.POINTER(Profile)]
    lib.mfsdp_profile_end.restype = ctypes.c_int
    lib.mfsdp_muon_workspace_size_p2p.argtypes = [ctypes.POINTER(Matrix), ctypes.POINTER(OwnerSegments), i32,
                                                  ctypes.POINTER(MuonHParams), ctypes.POINTER(ctypes.c_size_t)]
    lib.mfsdp_muon_workspace_size_p2p.restype = ctypes.c_int
    lib.mfsdp_muon_step_p2p.argtypes = [ctypes.POINTER(Matrix), ctypes.POINTER(OwnerSegments), i32,
                                        ctypes.POINTER(MuonHParams), p, ctypes.c_size_t, p]
    lib.mfsdp_muon_step_p2p.restype = ctypes.c_int
    lib.mfsdp_muon_workspace_size_p2p_overlap.argtypes = [ctypes.POINTER(Matrix), ctypes.POINTER(OwnerSegments),
                                                          i32, ctypes.POINTER(MuonHParams), i32,
                                                          ctypes.POINTER(ctypes.c_size_t)]
    lib.mfsdp_muon_workspace_size_p2p_overlap.restype = ctypes.c_int
    lib.mfsdp_muon_step_p2p_overlap.argtypes = [ctypes.POINTER(Matrix), ctypes.POINTER(OwnerSegments), i32,
                                                ctypes.POINTER(MuonHParams), i32, p, ctypes.c_size_t, p, p]
    lib.mfsdp_muon_step_p2p_overlap.restype = ctypes.c_int
    lib.mfsdp_muon_step_noalloc.argtypes = [ctypes.POINTER(Matrix), i32, ctypes.POINTER(MuonHParams), p]
    lib.mfsdp_muon_step_noalloc.restype = ctypes.c_int
    lib.mfsdp_selftest_bounded_wait.argtypes = [i64, p]
    lib.mfsdp_selftest_bounded_wait.restype = ctypes.c_int
    lib.mfsdp_version.argtypes = []
    lib.mfsdp_version.restype = ctypes.c_int32
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().mfsdp_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != MFSDP_OK:
        raise MfsdpError(status, where)


# ---- planner -----------------------------------------------------------------

def mfsdp_plan(params: Sequence[tuple], world_size: int, ns_steps: int = 5):
    """params: sequence of (rows, cols, kind, dtype) -> (shards, rank_flops, rank_bytes)."""
    lib = load()
    n = len(params)
    arr = (ParamDesc * max(n, 1))()
    for i, (r, c, k, d) in enumerate(params):
        arr[i] = ParamDesc(int(r), int(c), int(k), int(d))
    out = (MatrixShard * max(n, 1))()
    flops = (ctypes.c_double * world_size)()
    byts = (ctypes.c_int64 * world_size)()
    _check(lib.mfsdp_plan(arr, n, world_size, ns_steps, out, flops, byts), "mfsdp_plan")
    return list(out)[:n], list(flops), list(byts)


def mfsdp_heaviest_rank(rank_flops: Sequence[float], rank_bytes: Sequence[int]) -> int:
    lib = load()
    R = len(rank_flops)
    f = (ctypes.c_double * R)(*rank_flops)
    b = (ctypes.c_int64 * R)(*rank_bytes)
    out = ctypes.c_int32()
    _check(lib.mfsdp_heaviest_rank(f, b, R, ctypes.byref(out)), "mfsdp_heaviest_rank")
    return out.value


def mfsdp_reshard(params: Sequence[tuple], saved: Sequence[MatrixShard], new_world_size: int, ns_steps: int = 5):
    """params: (rows, cols, kind, dtype) per parameter; saved: its MatrixShard
    records of the saved layout -> (new shards, routes, moved state bytes)."""
    lib = load()
    n = len(params)
    arr = (ParamDesc * max(n, 1))()
    for i, (r, c, k, d) in enumerate(params):
        arr[i] = ParamDesc(int(r), int(c), int(k), int(d))
    sv = (MatrixShard * max(n, 1))()
    for i, rec in enumerate(saved):
        sv[i] = rec
    out = (MatrixShard * max(n, 1))()
    routes = (ReshardRoute * max(n, 1))()
    moved = ctypes.c_int64()
    _check(lib.mfsdp_reshard(arr, sv, n, new_world_size, ns_steps, out, routes, ctypes.byref(moved)),
           "mfsdp_reshard")
    return list(out)[:n], list(routes)[:n], moved.value


# ---- Muon step -----------------------------------------------------------------

def muon_hparams(lr=0.02, beta=0.95, weight_decay=0.01, eps=1e-7, a=3.4445, b=-4.7750, c=2.0315,
                 ns_steps=5, nesterov=True, mode=MFSDP_MODE_BF16) -> MuonHParams:
    return MuonHParams(lr, beta, weight_decay, eps, a, b, c, ns_steps, int(bool(nesterov)), mode)


def matrix_array(mats: Sequence[Matrix]):
    arr = (Matrix * max(len(mats), 1))()
    for i, m in enumerate(mats):
        arr[i] = m
    return arr


def mfsdp_muon_workspace_size(mats: Sequence[Matrix], hp: MuonHParams) -> int:
    out = ctypes.c_size_t()
    _check(load().mfsdp_muon_workspace_size(matrix_array(mats), len(mats), ctypes.byref(hp),
                                            ctypes.byref(out)), "mfsdp_muon_workspace_size")
    return out.value


def mfsdp_muon_step(mats: Sequence[Matrix], hp: MuonHParams, workspace_ptr: int, workspace_bytes: int,
                    stream: int, arr=None) -> None:
    if arr is None:
        arr = matrix_array(mats)
    _check(load().mfsdp_muon_step(arr, len(mats), ctypes.byref(hp), workspace_ptr, workspace_bytes, stream),
           "mfsdp_muon_step")


def mfsdp_muon_step_launches(mats: Sequence[Matrix], hp: MuonHParams) -> int:
    out = ctypes.c_int32()
    _check(load().mfsdp_muon_step_launches(matrix_array(mats), len(mats), ctypes.byref(hp), ctypes.byref(out)),
           "mfsdp_muon_step_launches")
    return out.value


def mfsdp_muon_forget_workspace(workspace_ptr: int) -> None:
    _check(load().mfsdp_muon_forget_workspace(workspace_ptr), "mfsdp_muon_forget_workspace")


def mfsdp_muon_forget_workspace_range(workspace_ptr: int, nbytes: int) -> None:
    _check(load().mfsdp_muon_forget_workspace_range(workspace_ptr, nbytes), "mfsdp_muon_forget_workspace_range")


# ---- AdamW tail ------------------------------------------------------------------

def adamw_hparams(lr=0.02, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.01, step=1) -> AdamWHParams:
    return AdamWHParams(lr, beta1, beta2, eps, weight_decay, 0, int(step))


def mfsdp_adamw_tail(p: int, g: int, m: int, v: int, n: int, hp: AdamWHParams, stream: int) -> None:
    _check(load().mfsdp_adamw_tail(p, g, m, v, n, ctypes.byref(hp), stream), "mfsdp_adamw_tail")


# ---- status --------------------------------------------------------------------------

def mfsdp_get_device_status(stream: int) -> int:
    out = ctypes.c_int32()
    _check(load().mfsdp_get_device_status(stream, ctypes.byref(out)), "mfsdp_get_device_status")
    return out.value


def mfsdp_selftest_bounded_wait(limit_ns: int, stream: int) -> None:
    _check(load().mfsdp_selftest_bounded_wait(int(limit_ns), stream), "mfsdp_selftest_bounded_wait")


def mfsdp_version() -> int:
    return int(load().mfsdp_version())


# ---- profiling ------------------------------------------------------------------------

def mfsdp_profile_begin(max_launches: int) -> None:
    _check(load().mfsdp_profile_begin(int(max_launches)), "mfsdp_profile_begin")


def mfsdp_profile_end() -> dict:
    """{class name: (timed launches, summed ms)} for the classes that ran."""
    out = Profile()
    _check(load().mfsdp_profile_end(ctypes.byref(out)), "mfsdp_profile_end")
    return {KCLASS_NAMES[k]: (int(out.launches[k]), float(out.ms[k]))
            for k in range(8) if out.launches[k] > 0}


# ---- step without a caller workspace ----------------------------------------------------

NOALLOC_SCRATCH_BYTES = 64 << 20


def mfsdp_muon_step_noalloc(mats: Sequence[Matrix], hp: MuonHParams, stream: int) -> None:
    """mfsdp_muon_step with the library's fixed 64 MiB device scratch: for callers
    that cannot allocate device memory (stream capture, host-managed memory pools).
    Calls that overlap on the GPU share the scratch and race."""
    _check(load().mfsdp_muon_step_noalloc(matrix_array(mats), len(mats), ctypes.byref(hp), stream),
           "mfsdp_muon_step_noalloc")


# ---- owner-segment exchange fused into the step -----------------------------------------

def owner_segments(parts_per_matrix: Sequence[Sequence[int]], copies_per_matrix: Sequence[Sequence[int]]):
    """OwnerSegments array from per-matrix lists of device pointers.  Returns
    (array, keepalive): the pointer arrays must outlive every call using them."""
    n = len(parts_per_matrix)
    arr = (OwnerSegments * max(n, 1))()
    keep = []
    for i, (parts, copies) in enumerate(zip(parts_per_matrix, copies_per_matrix)):
        pa = (ctypes.c_void_p * max(len(parts), 1))(*parts)
        ca = (ctypes.c_void_p * max(len(copies), 1))(*copies)
        keep += [pa, ca]
        arr[i] = OwnerSegments(ctypes.cast(pa, ctypes.POINTER(ctypes.c_void_p)),
                               ctypes.cast(ca, ctypes.POINTER(ctypes.c_void_p)) if copies else None,
                               len(parts), len(copies))
    return arr, keep


def mfsdp_muon_workspace_size_p2p(mats: Sequence[Matrix], segs, hp: MuonHParams) -> int:
    out = ctypes.c_size_t()
    _check(load().mfsdp_muon_workspace_size_p2p(matrix_array(mats), segs, len(mats), ctypes.byref(hp),
                                                ctypes.byref(out)), "mfsdp_muon_workspace_size_p2p")
    return out.value


def mfsdp_muon_step_p2p(mats: Sequence[Matrix], segs, hp: MuonHParams, workspace_ptr: int, workspace_bytes: int,
                        stream: int, arr=None) -> None:
    if arr is None:
        arr = matrix_array(mats)
    _check(load().mfsdp_muon_step_p2p(arr, segs, len(mats), ctypes.byref(hp), workspace_ptr, workspace_bytes,
                                      stream), "mfsdp_muon_step_p2p")


def mfsdp_muon_workspace_size_p2p_overlap(mats: Sequence[Matrix], segs, hp: MuonHParams, groups: int) -> int:
    out = ctypes.c_size_t()
    _check(load().mfsdp_muon_workspace_size_p2p_overlap(matrix_array(mats), segs, len(mats), ctypes.byref(hp),
                                                        int(groups), ctypes.byref(out)),
           "mfsdp_muon_workspace_size_p2p_overlap")
    return out.value


def mfsdp_muon_step_p2p_overlap(mats: Sequence[Matrix], segs, hp: MuonHParams, groups: int, workspace_ptr: int,
                                workspace_bytes: int, stream: int, copy_stream: int, arr=None) -> None:
    if arr is None:
        arr = matrix_array(mats)
    _check(load().mfsdp_muon_step_p2p_overlap(arr, segs, len(mats), ctypes.byref(hp), int(groups), workspace_ptr,
                                              workspace_bytes, stream, copy_stream),
           "mfsdp_muon_step_p2p_overlap")
