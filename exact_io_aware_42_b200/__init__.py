"""B200-native (sm_100a) exact IO-aware attention: forward, backward, FP8.

The compute lives in ``libfa_b200.so`` (CUDA kernels behind a C ABI, see
include/fa.h); ``api`` marshals torch tensors into it.  Importing this package
does not load the library; the first call does, and raises if it is missing.
"""
from .api import (  # noqa: F401
    bwd,
    bwd_noalloc,
    bwd_workspace_size,
    clear_status,
    fwd,
    fwd_fp8,
    get_status,
    n_blocks,
    quant_fp8,
    set_tuning,
    get_tuning,
)
from ._lib import FaError, library_path  # noqa: F401
