"""fp64 oracle of AdamW over the packed non-matrix tail (test infrastructure only).

Source: "MatrixFSDP: communication-free matrix optimizers under ZeRO-3
parameter sharding", arxivlens summary page, Abstract -- non-matrix tensors are
packed into tail owners and stay on AdamW; gist.science French summary,
Methodologie section 1, "Tenseurs Non-Matrices" (1D vectors go to a separate
owner and keep the standard AdamW optimizer).

The pages print no AdamW formula; this is the standard decoupled form (PyTorch
convention), with step count t starting at 1:

  m <- beta1 m + (1 - beta1) g
  v <- beta2 v + (1 - beta2) g^2
  p <- p (1 - lr wd) - lr (m / (1 - beta1^t)) / (sqrt(v / (1 - beta2^t)) + eps)

Pins (tests/test_oracle_adamw.py): t = 1 from zero state gives
p (1 - lr wd) - lr g / (|g| + eps); a constant gradient gives a bias-corrected
first moment equal to g at every t; g = 0 from zero state is pure decay; a
scalar recurrence unrolled by hand for three steps.
"""

from __future__ import annotations

import dataclasses
from typing import Tuple

import numpy as np


@dataclasses.dataclass(frozen=True)
class AdamWHParams:
    lr: float = 0.02
    beta1: float = 0.9
    beta2: float = 0.95
    eps: float = 1e-8
    weight_decay: float = 0.01


def adamw_step(p: np.ndarray, g: np.ndarray, m: np.ndarray, v: np.ndarray, t: int,
               hp: AdamWHParams) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """One AdamW step at step count t >= 1.  Returns (p_new, m_new, v_new), float64."""
    if t < 1:
        raise ValueError("AdamW step count starts at 1")
    p = np.asarray(p, np.float64)
    g = np.asarray(g, np.float64)
    m = np.asarray(m, np.float64)
    v = np.asarray(v, np.float64)
    m_new = hp.beta1 * m + (1.0 - hp.beta1) * g
    v_new = hp.beta2 * v + (1.0 - hp.beta2) * g * g
    bc1 = 1.0 - hp.beta1 ** t
    bc2 = 1.0 - hp.beta2 ** t
    m_hat = m_new / bc1
    v_hat = v_new / bc2
    p_new = p * (1.0 - hp.lr * hp.weight_decay) - hp.lr * m_hat / (np.sqrt(v_hat) + hp.eps)
    return p_new, m_new, v_new

