"""ctypes binding of the fp64 C++ oracle (test infrastructure only).

The oracle of record for the owner step: a plain fp64 C++ implementation of
"MatrixFSDP: communication-free matrix optimizers under ZeRO-3 parameter
sharding" (arxivlens summary page, Abstract; gist.science French summary,
Methodologie sections 1-2): Nesterov momentum, Frobenius normalisation,
quintic Newton-Schulz with the short side first, the shape scale, decoupled
weight decay and the write, plus AdamW over the packed tail.  The arithmetic
lives in ``oracle/csrc/muon.cpp``; this module only marshals numpy float64
arrays in and out, and builds the library with g++ on first use.

Only ``tests/``, ``__graft_entry__.smoke()`` and the host-baseline legs of
``bench.py`` may use it.  The functions mirror the numpy oracle's names and
signatures (``oracle.muon``, ``oracle.adamw``), so the same pins run against
both.

Pins (tests/test_oracle_native.py, tests/test_oracle_muon.py,
tests/test_oracle_adamw.py, tests/test_oracle_equivalence.py): the matrix
product bit for bit against an exact-rational replay of its definition; the
singular-value closed form of Newton-Schulz through an SVD; rank-1 and
orthonormal-row closed forms; transpose and orthogonal equivariance; the
momentum and AdamW closed forms; the owner-equivalence invariants.
"""

from __future__ import annotations

import ctypes
import math
import threading
from typing import List, Sequence, Tuple

import numpy as np

from . import build as _build
from .adamw import AdamWHParams
from .muon import MuonHParams

_lib = None
_lock = threading.Lock()

_dp = ctypes.POINTER(ctypes.c_double)
_dpp = ctypes.POINTER(_dp)


class _MuonHp(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_double), ("beta", ctypes.c_double), ("weight_decay", ctypes.c_double),
                ("eps", ctypes.c_double), ("a", ctypes.c_double), ("b", ctypes.c_double), ("c", ctypes.c_double),
                ("ns_steps", ctypes.c_int32), ("nesterov", ctypes.c_int32)]


class _AdamWHp(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_double), ("beta1", ctypes.c_double), ("beta2", ctypes.c_double),
                ("eps", ctypes.c_double), ("weight_decay", ctypes.c_double)]


def lib():
    """The loaded oracle library (built with g++ when missing or stale)."""
    global _lib
    with _lock:
        if _lib is None:
            path = _build.build()
            L = ctypes.CDLL(path)
            i64, i32, dbl = ctypes.c_int64, ctypes.c_int32, ctypes.c_double
            L.oracle_matmul.argtypes = [i64, i64, i64, _dp, i64, i32, _dp, i64, i32, _dp, i64]
            L.oracle_momentum.argtypes = [i64, _dp, _dp, dbl, i32, _dp, _dp]
            L.oracle_newton_schulz.argtypes = [i64, i64, _dp, dbl, dbl, dbl, i32, dbl, _dp]
            L.oracle_muon_step.argtypes = [i64, i64, _dp, _dp, _dp, ctypes.POINTER(_MuonHp), _dp, _dp, _dp]
            L.oracle_muon_step_parts.argtypes = [i64, i64, _dp, _dpp, i32, _dp, ctypes.POINTER(_MuonHp),
                                                 _dp, _dp, _dp]
            L.oracle_muon_step_list.argtypes = [i32, ctypes.POINTER(i64), ctypes.POINTER(i64), _dpp, _dpp, _dpp,
                                                ctypes.POINTER(_MuonHp), _dpp, _dpp, _dpp]
            L.oracle_adamw_step.argtypes = [i64, _dp, _dp, _dp, _dp, i64, ctypes.POINTER(_AdamWHp), _dp, _dp, _dp]
            L.oracle_set_threads.argtypes = [i32]
            L.oracle_get_threads.restype = i32
            for f in ("oracle_matmul", "oracle_momentum", "oracle_newton_schulz", "oracle_muon_step",
                      "oracle_muon_step_parts", "oracle_muon_step_list", "oracle_adamw_step"):
                getattr(L, f).restype = ctypes.c_int
            _lib = L
    return _lib


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float64)


def _p(a: np.ndarray):
    return a.ctypes.data_as(_dp)


def _check(st: int, what: str) -> None:
    if st != 0:
        raise ValueError(f"oracle {what}: invalid arguments (status {st})")


def set_threads(n: int) -> None:
    """Host threads the oracle uses (n <= 0: every CPU this process may run on)."""
    lib().oracle_set_threads(int(n))


def threads() -> int:
    return int(lib().oracle_get_threads())


def _hp(hp: MuonHParams) -> _MuonHp:
    return _MuonHp(hp.lr, hp.beta, hp.weight_decay, hp.eps, hp.a, hp.b, hp.c, int(hp.ns_steps),
                   1 if hp.nesterov else 0)


# ---- the matrix product primitive ----------------------------------------------------------

def matmul(A: np.ndarray, B: np.ndarray, trans_a: bool = False, trans_b: bool = False) -> np.ndarray:
    """op(A) op(B) with ascending-k fused-multiply-add sums (matmul.cpp)."""
    A, B = _f64(A), _f64(B)
    M, K = (A.shape[1], A.shape[0]) if trans_a else A.shape
    K2, N = (B.shape[1], B.shape[0]) if trans_b else B.shape
    if K != K2:
        raise ValueError("inner dimensions differ")
    C = np.empty((M, N), np.float64)
    lda, ldb = max(A.shape[1], 1), max(B.shape[1], 1)      # row-major, contiguous
    _check(lib().oracle_matmul(M, N, K, _p(A), lda, int(trans_a), _p(B), ldb, int(trans_b), _p(C), max(N, 1)),
           "matmul")
    return C


# ---- the Muon step (names and signatures of oracle.muon) -------------------------------------

def nesterov_momentum(G: np.ndarray, buf: np.ndarray, beta: float, nesterov: bool = True
                      ) -> Tuple[np.ndarray, np.ndarray]:
    """Step 1.  Returns (M, buf_new)."""
    G, buf = _f64(G), _f64(buf)
    M, bn = np.empty_like(G), np.empty_like(G)
    _check(lib().oracle_momentum(G.size, _p(G), _p(buf), float(beta), 1 if nesterov else 0, _p(M), _p(bn)),
           "momentum")
    return M, bn


def frobenius_normalise(T: np.ndarray, eps: float) -> np.ndarray:
    """Step 3 alone: Newton-Schulz with zero iterations on a wide-or-square T."""
    return newton_schulz(T, 0.0, 0.0, 0.0, 0, eps)


def newton_schulz(M: np.ndarray, a: float, b: float, c: float, steps: int = 5, eps: float = 1e-7) -> np.ndarray:
    """Steps 2-4 and the transpose back (no shape scale)."""
    M = _f64(M)
    O = np.zeros_like(M)
    _check(lib().oracle_newton_schulz(M.shape[0], M.shape[1], _p(M), float(a), float(b), float(c), int(steps),
                                      float(eps), _p(O)), "newton_schulz")
    return O


def shape_scale(rows: int, cols: int) -> float:
    return math.sqrt(max(1.0, rows / cols))


def muon_step(W: np.ndarray, G: np.ndarray, buf: np.ndarray, hp: MuonHParams
              ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """The owner's whole step for one matrix.  Returns (W_new, O, buf_new), float64."""
    W, G, buf = _f64(W), _f64(G), _f64(buf)
    Wn, O, bn = np.empty_like(W), np.zeros_like(W), np.empty_like(W)
    h = _hp(hp)
    _check(lib().oracle_muon_step(W.shape[0], W.shape[1], _p(W), _p(G), _p(buf), ctypes.byref(h), _p(Wn), _p(O),
                                  _p(bn)), "muon_step")
    return Wn, O, bn


def muon_update(G: np.ndarray, buf: np.ndarray, hp: MuonHParams) -> Tuple[np.ndarray, np.ndarray]:
    """Steps 1-5.  Returns (O, buf_new)."""
    G = _f64(G)
    _, O, bn = muon_step(np.zeros_like(G), G, buf, hp)
    return O, bn


def muon_step_parts(W: np.ndarray, parts: Sequence[np.ndarray], buf: np.ndarray, hp: MuonHParams
                    ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """The owner's step on a gradient given as ranks' contributions, summed in order."""
    W, buf = _f64(W), _f64(buf)
    ps = [_f64(p) for p in parts]
    arr = (_dp * len(ps))(*[_p(p) for p in ps])
    Wn, O, bn = np.empty_like(W), np.zeros_like(W), np.empty_like(W)
    h = _hp(hp)
    _check(lib().oracle_muon_step_parts(W.shape[0], W.shape[1], _p(W), arr, len(ps), _p(buf), ctypes.byref(h),
                                        _p(Wn), _p(O), _p(bn)), "muon_step_parts")
    return Wn, O, bn


def muon_step_list(Ws: Sequence[np.ndarray], Gs: Sequence[np.ndarray], bufs: Sequence[np.ndarray],
                   hp: MuonHParams) -> Tuple[List[np.ndarray], List[np.ndarray], List[np.ndarray]]:
    """The owner's list of matrices in one call.  Returns (W_new list, O list, buf_new list)."""
    Ws, Gs, bufs = [_f64(w) for w in Ws], [_f64(g) for g in Gs], [_f64(b) for b in bufs]
    n = len(Ws)
    Wn = [np.empty_like(w) for w in Ws]
    O = [np.zeros_like(w) for w in Ws]
    bn = [np.empty_like(w) for w in Ws]
    rows = (ctypes.c_int64 * n)(*[w.shape[0] for w in Ws])
    cols = (ctypes.c_int64 * n)(*[w.shape[1] for w in Ws])
    arr = lambda xs: (_dp * n)(*[_p(x) for x in xs])  # noqa: E731
    h = _hp(hp)
    _check(lib().oracle_muon_step_list(n, rows, cols, arr(Ws), arr(Gs), arr(bufs), ctypes.byref(h), arr(Wn),
                                       arr(O), arr(bn)), "muon_step_list")
    return Wn, O, bn


# ---- AdamW (names and signature of oracle.adamw) ---------------------------------------------

def adamw_step(p: np.ndarray, g: np.ndarray, m: np.ndarray, v: np.ndarray, t: int, hp: AdamWHParams
               ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """One AdamW step at step count t >= 1.  Returns (p_new, m_new, v_new), float64."""
    if t < 1:
        raise ValueError("AdamW step count starts at 1")
    p, g, m, v = _f64(p), _f64(g), _f64(m), _f64(v)
    pn, mn, vn = np.empty_like(p), np.empty_like(p), np.empty_like(p)
    h = _AdamWHp(hp.lr, hp.beta1, hp.beta2, hp.eps, hp.weight_decay)
    _check(lib().oracle_adamw_step(p.size, _p(p), _p(g), _p(m), _p(v), int(t), ctypes.byref(h), _p(pn), _p(mn),
                                   _p(vn)), "adamw_step")
    return pn, mn, vn
