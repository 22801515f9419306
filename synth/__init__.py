"""Seeded synthetic workloads for the owner-local optimizer step.

This package is shared harness code: both the fp64 oracle tests and the GPU
path read the inputs it produces.  It holds no arithmetic of the optimizer
itself (no momentum, normalisation, Newton-Schulz, decay or AdamW): only the
parameter lists of the workloads and seeded random draws of their initial
state.
"""

from .workloads import (  # noqa: F401
    ParamSpec,
    Workload,
    WORKLOADS,
    workload,
)
from .gen import (  # noqa: F401
    MatrixInputs,
    TailInputs,
    matrix_inputs,
    tail_inputs,
    param_seed,
)
