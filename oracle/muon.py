"""fp64 oracle of the owner-local Muon update (test infrastructure only).

Source of the method: "MatrixFSDP: communication-free matrix optimizers under
ZeRO-3 parameter sharding", arxivlens summary page, Abstract -- Muon smooths
the matrix gradient with momentum and orthogonalises the result with
Newton-Schulz; the step needs the complete 2D matrix, which under owner-shaped
placement lives on one data-parallel owner (gist.science French summary,
Methodologie section 1; Portuguese summary, Metodologia section 1), so the
owner runs the update locally with no collective.

The pages name the steps but print no formula.  The arithmetic below is the
standard Muon definition this library implements:

  1. Nesterov momentum in EMA form:
       buf <- beta * buf + (1 - beta) * G
       M   <- (1 - beta) * G + beta * buf            (plain momentum: M <- buf)
  2. short side first: T = M^T if rows > cols else M     (X is r x c, r <= c)
  3. Frobenius normalisation: X_0 = T / (||T||_F + eps)
  4. five quintic Newton-Schulz iterations, (a, b, c) = (3.4445, -4.7750, 2.0315):
       A = X X^T ;  B = b A + c A A ;  X <- a X + B X
  5. O = (transpose back) X_5 * sqrt(max(1, rows / cols))
  6. decoupled weight decay and write: W <- W (1 - lr wd) - lr O

Readings taken where the pages are silent: EMA-form Nesterov momentum,
eps = 1e-7 added to the norm, strict rows > cols for the transpose, the shape
scale on the original rows/cols, weight decay multiplied by lr and applied to
the pre-update W.

Pins (tests/test_oracle_muon.py): the singular-value closed form
NS5(X_0) = U p^5(S) V^T with p(s) = a s + b s^3 + c s^5 checked through an SVD;
rank-1 and orthonormal-row closed forms; transpose and orthogonal
equivariance; scale invariance; the constant-gradient momentum closed form;
the zero-gradient case; the linearity of the write in O.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Tuple

import numpy as np


@dataclasses.dataclass(frozen=True)
class MuonHParams:
    lr: float = 0.02
    beta: float = 0.95
    weight_decay: float = 0.01
    eps: float = 1e-7
    a: float = 3.4445
    b: float = -4.7750
    c: float = 2.0315
    ns_steps: int = 5
    nesterov: bool = True


def nesterov_momentum(G: np.ndarray, buf: np.ndarray, beta: float,
                      nesterov: bool = True) -> Tuple[np.ndarray, np.ndarray]:
    """Step 1.  Returns (M, buf_new), both float64."""
    G = np.asarray(G, np.float64)
    buf = np.asarray(buf, np.float64)
    buf_new = beta * buf + (1.0 - beta) * G
    if nesterov:
        M = (1.0 - beta) * G + beta * buf_new
    else:
        M = buf_new
    return M, buf_new


def frobenius_normalise(T: np.ndarray, eps: float) -> np.ndarray:
    """Step 3.  X_0 = T / (sqrt(sum of squares of T) + eps)."""
    T = np.asarray(T, np.float64)
    norm = math.sqrt(float(np.sum(T * T)))
    return T / (norm + eps)


def newton_schulz(M: np.ndarray, a: float, b: float, c: float, steps: int = 5,
                  eps: float = 1e-7) -> np.ndarray:
    """Steps 2-4 and the transpose back: the orthogonalised M (no shape scale)."""
    M = np.asarray(M, np.float64)
    transposed = M.shape[0] > M.shape[1]
    X = M.T if transposed else M
    X = frobenius_normalise(X, eps)
    for _ in range(steps):
        A = X @ X.T
        B = b * A + c * (A @ A)
        X = a * X + B @ X
    return X.T.copy() if transposed else X


def shape_scale(rows: int, cols: int) -> float:
    """Step 5's scale on the parameter's own (out, in) shape."""
    return math.sqrt(max(1.0, rows / cols))


def muon_update(G: np.ndarray, buf: np.ndarray, hp: MuonHParams) -> Tuple[np.ndarray, np.ndarray]:
    """Steps 1-5.  Returns (O, buf_new)."""
    M, buf_new = nesterov_momentum(G, buf, hp.beta, hp.nesterov)
    rows, cols = M.shape
    if rows == 0 or cols == 0:
        return np.zeros((rows, cols)), buf_new
    O = newton_schulz(M, hp.a, hp.b, hp.c, hp.ns_steps, hp.eps) * shape_scale(rows, cols)
    return O, buf_new


def apply_update(W: np.ndarray, O: np.ndarray, lr: float, weight_decay: float) -> np.ndarray:
    """Step 6: W (1 - lr wd) - lr O, float64."""
    W = np.asarray(W, np.float64)
    return W * (1.0 - lr * weight_decay) - lr * np.asarray(O, np.float64)


def muon_step(W: np.ndarray, G: np.ndarray, buf: np.ndarray,
              hp: MuonHParams) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """The owner's whole step for one matrix.  Returns (W_new, O, buf_new), float64."""
    O, buf_new = muon_update(G, buf, hp)
    return apply_update(W, O, hp.lr, hp.weight_decay), O, buf_new
