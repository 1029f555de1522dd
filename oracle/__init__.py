"""fp64 CPU oracle for the norm operators -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference legs may import this package.  The library never does.
"""
from .rmsnorm import (  # noqa: F401
    ACTS,
    FORMATS,
    residual_add,
    rmsnorm_add_bwd,
    rmsnorm_add_fwd,
    round_to_format,
    dx_cancellation_scale,
    dz_cancellation_scale,
    gated_norm_bwd,
    gated_norm_fwd,
    norm_bwd,
    norm_fwd,
    rmsnorm_bwd,
    rmsnorm_dx_scale,
    rmsnorm_dz_scale,
    rmsnorm_fwd,
    rstd,
    sigmoid,
    silu,
)
