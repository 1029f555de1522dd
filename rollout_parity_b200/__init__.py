"""Batch-invariant zero-centred and gated RMSNorm (forward + backward) for B200.

The computation lives in librn.so (CUDA kernels for sm_100a behind a C ABI,
declared in include/rn.h).  This package is its thin binding: ``ops`` has one
function per C entry point with the same name; ``autograd`` wraps them as
torch.autograd Functions; ``workloads`` draws seeded synthetic inputs.
"""
from ._lib import LIB_PATH, Act, DType, RNError, Status, load  # noqa: F401
from .ops import (  # noqa: F401
    act_code,
    gated_norm_bwd,
    gated_norm_fwd,
    norm_bwd,
    norm_bwd_workspace_bytes,
    norm_fwd,
    rn_describe,
    rn_fold_rows,
    rn_test_set_geometry,
    rn_test_set_validate_only,
    rmsnorm_add_bwd,
    rmsnorm_add_fwd,
    rmsnorm_bwd,
    rmsnorm_bwd_chunks,
    rn_fold_tree,
    rmsnorm_fwd,
    workspace,
)
from . import autograd  # noqa: E402,F401
