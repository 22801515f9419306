"""fp64 oracle of the MatrixFSDP owner-local optimizer step.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It
shares no code with the CUDA library under
``matrix_optimizer_step_nesterov_b200/`` and never imports it.

Two independent writings of the same definitions:

* the oracle of record, a plain fp64 C++ library (``oracle/csrc``, bound by
  ``oracle/native.py``, built with g++ by ``oracle/build.py``): the owner's
  full-matrix Muon update (Nesterov momentum, Frobenius normalisation, five
  quintic Newton-Schulz iterations with the short side first, the
  sqrt(max(1, rows/cols)) shape scale, decoupled weight decay and the
  parameter write), its owner-segment form (the gradient arriving as ranks'
  contributions), and AdamW over the packed non-matrix tail.  Its only
  primitive is an fp64 matrix product defined as ascending-k fused sums;
* the first writing in numpy (``oracle.muon``, ``oracle.adamw``), kept as an
  independent cross-check of the C++ one.

Source: "MatrixFSDP: communication-free matrix optimizers under ZeRO-3
parameter sharding" (arxivlens summary page, Abstract: Muon orthogonalises
momentum-smoothed matrix updates with Newton-Schulz and needs the whole 2D
matrix, which the owner holds; non-matrix tensors are packed into tail owners
and stay on AdamW), and the gist.science French summary, Methodologie
sections 1-2 (the owner receives exactly the full gradient; owners are chosen
to balance resident bytes and optimizer work).

``plan`` is the balance-aware owner planner and the checkpoint resharding
routes (host logic, in Python).

Every function is pinned by ``tests/test_oracle_*.py`` against closed forms,
invariants, special cases, brute force and exact-rational replays.
"""

from .muon import MuonHParams  # noqa: F401
from .adamw import AdamWHParams  # noqa: F401
from . import muon, adamw  # noqa: F401  (the numpy writing, cross-check)
from .native import (  # noqa: F401  (the oracle of record: fp64 C++)
    nesterov_momentum,
    frobenius_normalise,
    newton_schulz,
    shape_scale,
    muon_update,
    muon_step,
    muon_step_parts,
    muon_step_list,
    adamw_step,
)
from . import native  # noqa: F401
from .plan import plan_owners, PlanEntry, heaviest_rank, reshard, ReshardRoute, state_bytes  # noqa: F401
