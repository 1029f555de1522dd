"""CPU: the bitwise rstd-identity checks can see a one-kernel perturbation.

The GPU tests compare the gated (and every general) forward's rstd with the
plain forward's bit for bit (the rstd identity of PR #468, Summary, "rstd"
bullet).  Mistakes are planted only in the oracle and only on the CPU, so the
kernels are not mutated to show that those checks are sensitive.  This test
shows it on the same inputs instead: an fp32 statistic in which one kernel
added 1e-4 to each square, as a mistake in one of two copies of the code would,
differs in its bits from the unperturbed one in every row the GPU checks use.
"""
import numpy as np
import pytest

from rollout_parity_b200 import workloads


def rstd32(x: np.ndarray, eps: float, bump: float = 0.0) -> np.ndarray:
    x = x.astype(np.float32)
    sq = x * x + np.float32(bump)
    ss = np.sum(sq, axis=1, dtype=np.float32)
    ms = ss / np.float32(x.shape[1])
    return (np.float32(1.0) / np.sqrt(ms + np.float32(eps))).astype(np.float32)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("width", [8, 128, 136, 2048, 5120, 8192, 16384])
@pytest.mark.parametrize("eps", [1e-6, 0.0, 0.5])
def test_perturbed_squares_change_every_rows_rstd_bits(dtype, width, eps):
    wl = workloads.make("gated", 97, width, dtype, seed=width)   # the GPU check's inputs
    x = workloads.as_f64(wl.x)
    plain = rstd32(x, eps)
    bumped = rstd32(x, eps, bump=1e-4)
    assert np.isfinite(plain).all()
    assert (plain.view(np.int32) != bumped.view(np.int32)).all()
