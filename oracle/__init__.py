"""fp64 oracle of the MatrixFSDP owner-local optimizer step.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It
shares no code with the CUDA library under
``matrix_optimizer_step_nesterov_b200/`` and never imports it.

What it computes, in plain numpy float64 (a matrix product is the only library
primitive it leans on):

* ``muon``  - the owner's full-matrix Muon update: Nesterov momentum,
  Frobenius normalisation, five quintic Newton-Schulz iterations with the
  short side first, the sqrt(max(1, rows/cols)) shape scale, decoupled weight
  decay and the parameter write.  Source: "MatrixFSDP: communication-free
  matrix optimizers under ZeRO-3 parameter sharding" (arxivlens summary page),
  Abstract: Muon orthogonalises momentum-smoothed matrix updates with
  Newton-Schulz and needs the whole 2D matrix, which the owner holds.
* ``adamw`` - AdamW over the packed non-matrix tail (same page, Abstract:
  non-matrix tensors are packed into tail owners and stay on AdamW).
* ``plan``  - the balance-aware owner planner (same page, Abstract; the
  gist.science French summary, Methodologie section 2, "Metadonnees
  MatrixShard & Planificateur Global": owners are chosen to balance resident
  bytes and optimizer work).

Every function is pinned by ``tests/test_oracle_*.py`` against closed forms,
invariants, special cases and brute force (see each function's docstring for
its pins).
"""

from .muon import (  # noqa: F401
    MuonHParams,
    nesterov_momentum,
    frobenius_normalise,
    newton_schulz,
    shape_scale,
    muon_update,
    muon_step,
)
from .adamw import AdamWHParams, adamw_step  # noqa: F401
from .plan import plan_owners, PlanEntry, heaviest_rank, reshard, ReshardRoute, state_bytes  # noqa: F401
