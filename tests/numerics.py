"""Comparison helpers for the parity tests: exact fp64 -> bf16 / fp16 rounding,
their ulps, and the tolerance rules.  No norm arithmetic lives here.

Tolerances (the operators' contract asks for fp32 accumulation and bf16 outputs;
the bar is 2 bf16 ulp per bf16 element and relative L2 <= 1e-4 for fp32 tensors):
  * bf16 y:        |gpu - ref| <= 2 ulp_bf16(|ref|)   (fp16: the same in fp16 ulps)
  * bf16 dx, dz:   |gpu - ref| <= 2 ulp_bf16(|ref|) + 2**-16 * T
    where T is the size of the largest term that cancels in that element
    (the oracle's cancellation scale; for dx's mean term it is built from the
    magnitudes of the row sum's terms, which bound that sum's rounding error);
    fp32 rounding of those terms is amplified by the cancellation, and no bf16
    rounding can hide it.
  * fp32 tensors:  ||gpu - ref||_2 / ||ref||_2 <= 1e-4
"""
from __future__ import annotations

import numpy as np
import torch

# 16-bit formats: (significant bits, exponent of the subnormal spacing, largest finite)
BF16 = (8, -133, float.fromhex("0x1.fep127"))
F16 = (11, -24, 65504.0)
BF16_MIN_EXP = BF16[1]       # bf16 subnormal spacing is 2**-133
BF16_MAX = BF16[2]


def round16(a, fmt) -> np.ndarray:
    """Round fp64 values to the nearest value of the 16-bit format ``fmt``
    (BF16 or F16), ties to even, in one step (no intermediate fp32 rounding);
    past the largest finite value, to infinity.  Returns fp64."""
    p, min_exp, vmax = fmt
    a = np.asarray(a, dtype=np.float64)
    out = np.zeros_like(a)
    nz = (a != 0) & np.isfinite(a)
    _, e = np.frexp(a[nz])                       # a = m * 2**e, 0.5 <= |m| < 1
    step = np.ldexp(1.0, np.maximum(e - p, min_exp))
    q = np.rint(a[nz] / step) * step             # exact scaling; rint is ties-to-even
    q = np.where(np.abs(q) > vmax, np.copysign(np.inf, q), q)
    out[nz] = q
    out[~np.isfinite(a)] = a[~np.isfinite(a)]
    out[a == 0] = a[a == 0]
    return out


def ulp16(a, fmt) -> np.ndarray:
    """Spacing of the 16-bit format's values at |a| (the subnormal spacing at
    the bottom)."""
    p, min_exp, _ = fmt
    a = np.abs(np.asarray(a, dtype=np.float64))
    _, e = np.frexp(np.where(a == 0, 1e-300, a))
    return np.ldexp(1.0, np.maximum(e - p, min_exp))


def bf16_round(a) -> np.ndarray:
    return round16(a, BF16)


def bf16_ulp(a) -> np.ndarray:
    return ulp16(a, BF16)


FMT_OF = {torch.bfloat16: BF16, torch.float16: F16}


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


def counts_16(g: np.ndarray, ref: np.ndarray, fmt, scale=None, ulps=2.0,
              floor=2.0 ** -16) -> dict:
    """Counts behind the 16-bit tolerance for values ``g`` of format ``fmt``
    (exact in fp64) against the fp64 reference: elements equal to the
    reference rounded once to the format (correctly rounded), within the plain
    ``ulps`` bound, passing only through the cancellation floor
    (floor * scale), and out of tolerance; the largest error in ulps."""
    ulp = ulp16(ref, fmt)
    err = np.abs(g - ref)
    lim_plain = ulps * ulp
    lim = lim_plain if scale is None else lim_plain + floor * np.asarray(scale)
    bad = ~(err <= lim)          # NaN counts as out of tolerance
    return {
        "n": int(g.size),
        "correctly_rounded": int(np.sum(g == round16(ref, fmt))),
        "plain_pass": int(np.sum(err <= lim_plain)),
        "floor_hits": int(np.sum((err > lim_plain) & ~bad)),
        "out_of_tolerance": int(np.sum(bad)),
        "max_err_ulps": float(np.max(err / ulp)) if g.size else 0.0,
    }


def check_16(got: torch.Tensor, ref: np.ndarray, scale=None, what="", ulps=2.0,
             floor=2.0 ** -16) -> dict:
    """Assert the 16-bit (bf16 or fp16) tolerance; return pass statistics."""
    fmt = FMT_OF[got.dtype]
    g = to64(got)
    ref = np.asarray(ref, dtype=np.float64)
    assert g.shape == ref.shape, (what, g.shape, ref.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    c = counts_16(g, ref, fmt, scale, ulps, floor)
    n = max(1, c["n"])
    stats = {
        "n": c["n"],
        "max_err_ulps": c["max_err_ulps"],
        "plain_2ulp_pass_frac": c["plain_pass"] / n if c["n"] else 1.0,
        "floor_hits": c["floor_hits"],
        "correctly_rounded_frac": c["correctly_rounded"] / n if c["n"] else 1.0,
    }
    if c["out_of_tolerance"]:
        err = np.abs(g - ref)
        lim = ulps * ulp16(ref, fmt) + (0.0 if scale is None else floor * np.asarray(scale))
        bad = err > lim
        i = np.unravel_index(np.argmax(err - lim), err.shape)
        raise AssertionError(
            f"{what}: {int(bad.sum())}/{g.size} elements out of tolerance; worst at {i}: "
            f"got {g[i]!r} want {ref[i]!r} lim {lim[i]!r}")
    return stats


def check_f32(got: torch.Tensor, ref: np.ndarray, what="", rel_l2=1e-4) -> dict:
    g = to64(got)
    ref = np.asarray(ref, dtype=np.float64)
    assert g.shape == ref.shape, (what, g.shape, ref.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((g - ref).ravel())
    r = num / den if den > 0 else num
    denom = np.maximum(np.abs(ref), 1e-30)
    stats = {"rel_l2": float(r), "max_rel": float(np.max(np.abs(g - ref) / denom)) if g.size else 0.0}
    assert r <= rel_l2, f"{what}: relative L2 {r:.3e} > {rel_l2:.1e}"
    return stats


def check_out(got: torch.Tensor, ref: np.ndarray, scale=None, what="") -> dict:
    if got.dtype in FMT_OF:
        return check_16(got, ref, scale=scale, what=what)
    return check_f32(got, ref, what=what)
