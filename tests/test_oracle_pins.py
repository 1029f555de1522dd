"""The fp64 oracle against closed forms, worked examples, derivatives and
brute force (CPU only)."""
import numpy as np
import pytest

import oracle
import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    with np.errstate(over="ignore"):
        pin(oracle)


def test_oracle_rejects_non_2d():
    with pytest.raises(ValueError):
        oracle.rstd(np.zeros(4), 1e-6)


def test_oracle_large_magnitude_gate_is_finite():
    # outlier channels scaled x50 push |z| to ~200; the fp64 oracle must stay finite
    rng = np.random.default_rng(0)
    x = rng.normal(size=(4, 16)) * 50
    z = rng.normal(size=(4, 16)) * 200
    w = rng.normal(size=16)
    dy = rng.normal(size=(4, 16)) * 50
    y, _ = oracle.gated_norm_fwd(x, z, w, 1e-6)
    dx, dz, dw = oracle.gated_norm_bwd(x, z, w, dy, 1e-6)
    for a in (y, dx, dz, dw):
        assert np.all(np.isfinite(a))
