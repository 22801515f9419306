"""B200-native owner-local optimizer step of MatrixFSDP (libmfsdp).

The C ABI (include/mfsdp.h) is the product; ``_lib`` binds it with ctypes and
``owner_step`` marshals torch tensors into it.  The first call into the
library loads libmfsdp.so and raises ImportError if it has not been built:
there is no CPU or PyTorch fallback for any step of the update.
"""

from . import _lib  # noqa: F401
from ._lib import (  # noqa: F401
    MfsdpError,
    mfsdp_plan,
    mfsdp_heaviest_rank,
    mfsdp_version,
    load,
)
from .owner_step import MuonOwnerStep, adamw_tail, device_status  # noqa: F401

