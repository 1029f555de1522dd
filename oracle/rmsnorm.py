"""fp64 CPU oracle for zero-centred and gated RMSNorm, forward and backward.

TEST INFRASTRUCTURE ONLY.  The parity tests under ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference leg are
the only callers.  The library (``rollout_parity_b200``) never imports, links or
runs anything here, and nothing here imports the library: the two share no
code.  The only module both sides use is the seeded input generator
(``rollout_parity_b200.workloads``), which holds none of this arithmetic.

What is computed, and where it is defined
-----------------------------------------
[PR468] RL-Kernel PR #468, "[WS1][CUDA][Qwen3-Next] Gated RMSNorm CUDA kernel for
        the GDN block", section "Summary" (the displayed formula for y, and the
        kernel, activation, rstd and backward bullets).
[RFC415] RL-Kernel RFC #415 (Gemma-4-31B consistency roadmap), section 4
        "Numerical contract" (declared accumulator, casts only at epilogues).

For one row x of width H (all values are the stored inputs widened exactly to
fp64; nothing here rounds to a narrower type):

    ms   = (1/H) * sum_j x_j^2                    mean square over the width
    rho  = 1 / sqrt(ms + eps)                     the row's rstd
    xh_j = x_j * rho
    zero-centred:  y_j = xh_j * (1 + w_j)         weight offset 1
    gated:         y_j = xh_j * w_j * silu(z_j)   weight offset 0, act = silu
                   silu(z) = z * s(z),  s(z) = 1 / (1 + exp(-z))

The backward is the exact gradient of L = sum_rj y_rj * dy_rj (plain calculus of
the forward; [PR468] Summary, "Backward" bullet, states that the gated dx is the
ungated dx with the gain (w + offset) replaced by (w + offset) * act(z)):

    g_j  = 1 + w_j            (zero-centred)   or   w_j * silu(z_j)   (gated)
    m    = (1/H) * sum_j g_j * dy_j * xh_j
    dx_j = rho * (g_j * dy_j - xh_j * m)
    dz_j = dy_j * xh_j * w_j * s_j * (1 + z_j * (1 - s_j))            (gated)
    dw_j = sum_r dy_rj * xh_rj                     (zero-centred)
         = sum_r dy_rj * xh_rj * silu(z_rj)        (gated)

The general form ([PR468] Summary, the displayed formula and the
"Activation" bullet: a weight offset and a gate activation, silu or sigmoid;
[PR468] "Changes to existing code, in detail", "Signed zero" bullet: the offset
is added only when it is nonzero, so a -0.0 weight keeps its sign):

    u_j  = w_j + offset   (offset != 0)   or   w_j   (offset == 0)
    y_j  = xh_j * u_j * a(z_j),  a = 1 (no gate), silu(z), or s(z)
    g_j  = u_j * a(z_j);  dx as above;  dz_j = dy_j * xh_j * u_j * a'(z_j)
    dw_j = sum_r dy_rj * xh_rj * a(z_rj)
    a'(z) = s(z) * (1 + z * (1 - s(z)))  (silu)   or   s(z) * (1 - s(z))  (sigmoid)

The zero-centred and gated operators above are (offset 1, no gate) and
(offset 0, silu).

Row mask for dw ([PR468] "Changes to existing code, in detail": the dw entry
point takes a mask; read as one flag per row, rows with the flag clear left out
of dw's sum, e.g. padding):  dw_j = sum over rows r with mask_r of
dy_rj * xh_rj * a(z_rj); dx and dz are unchanged.  A sum over no row (no rows
at all, or a mask that selects none) is -0.0, the identity of IEEE addition
(see _sum_over_rows).

Parity pins (``tests/oracle_pins.py``, run by ``tests/test_oracle_pins.py``,
with planted mistakes in ``tests/test_oracle_mutations.py``):
  rstd/forward : constant-row closed form, RMS(xh) == 1 at eps = 0, scale
                 invariance at eps = 0, w = 0 reduces y to xh, exact rational
                 worked examples (in tests/oracle_pins.py), sigmoid at ln(k)
                 points.
  backward     : central finite differences of L (dx, dz, dw), the scale
                 identity sum_j x_j dx_j = rho * S * eps / (ms + eps), and a
                 brute-force double loop for dw.
  general form : a rational worked example (sigmoid gate, offset 1), finite
                 differences for every activation x offset {0, 1, 1/2}, the
                 signed-zero rule, and reduction to the two operators above.
  residual add : fp32 -> bf16 / fp16 rounding against torch's conversions and
                 hand-checked ties, an exact example where the rounded sum is
                 the worked example's row, r = 0 reduces to the plain forward,
                 finite differences of sum(y*dy) + sum(h*dh) in x and in r.
  row mask     : all-ones equals no mask, a brute-force loop over the selected
                 rows, masked rows holding NaN/Inf leave dw finite and dx of the
                 other rows unchanged, dw(mask) + dw(not mask) = dw.
Every public function below is pinned; none is "parity unpinned".
"""
from __future__ import annotations

import numpy as np


def _rows(a) -> np.ndarray:
    a = np.asarray(a, dtype=np.float64)
    if a.ndim != 2:
        raise ValueError("expected a [rows, width] array")
    return a


def sigmoid(z):
    """s(z) = 1 / (1 + exp(-z)) in fp64 ([PR468] Summary, activation bullet)."""
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-z))


def silu(z):
    """silu(z) = z * s(z); "swish" is the same function ([PR468] Summary)."""
    z = np.asarray(z, dtype=np.float64)
    return z * sigmoid(z)


def rstd(x, eps: float) -> np.ndarray:
    """rho_r = 1 / sqrt(mean_j x_rj^2 + eps), one value per row ([PR468]
    Summary, rstd bullet: a sum of squares over the row, then the reciprocal
    square root of its mean plus eps)."""
    x = _rows(x)
    width = x.shape[1]
    ms = np.sum(x * x, axis=1) / width
    return 1.0 / np.sqrt(ms + eps)


def norm_fwd(x, w, eps: float):
    """Zero-centred RMSNorm forward: y = x * rho * (1 + w).  Returns (y, rho)."""
    x = _rows(x)
    w = np.asarray(w, dtype=np.float64)
    rho = rstd(x, eps)
    xh = x * rho[:, None]
    return xh * (1.0 + w)[None, :], rho


def gated_norm_fwd(x, z, w, eps: float):
    """Gated RMSNorm forward: y = x * rho * w * silu(z), the norm applied before
    the gate and one group per row.  Returns (y, rho)."""
    x, z = _rows(x), _rows(z)
    w = np.asarray(w, dtype=np.float64)
    rho = rstd(x, eps)
    xh = x * rho[:, None]
    return xh * w[None, :] * silu(z), rho


def _sum_over_rows(c) -> np.ndarray:
    """dw's sum over rows, per column, started from -0.0.

    -0.0 is the identity of IEEE addition (-0.0 + v == v for every v, +0.0
    included), so starting there changes no sum that has a term; it fixes the
    value of the empty sum -- a batch of no rows, or a row mask that selects
    none -- at -0.0 in every column.  The pages fix no value for that case
    ([PR468] Notes only say the T == 0 call returns early); this is the
    reading taken."""
    return np.sum(np.asarray(c, dtype=np.float64), axis=0, initial=-0.0)


def _dx(x, g, dy, rho):
    width = x.shape[1]
    xh = x * rho[:, None]
    m = np.sum(g * dy * xh, axis=1) / width
    return rho[:, None] * (g * dy - xh * m[:, None])


def norm_bwd(x, w, dy, eps: float):
    """Zero-centred RMSNorm backward.  Returns (dx [rows, width], dw [width])."""
    x, dy = _rows(x), _rows(dy)
    w = np.asarray(w, dtype=np.float64)
    rho = rstd(x, eps)
    g = np.broadcast_to((1.0 + w)[None, :], x.shape)
    dx = _dx(x, g, dy, rho)
    dw = _sum_over_rows(dy * (x * rho[:, None]))
    return dx, dw


def gated_norm_bwd(x, z, w, dy, eps: float):
    """Gated RMSNorm backward.  Returns (dx, dz, dw)."""
    x, z, dy = _rows(x), _rows(z), _rows(dy)
    w = np.asarray(w, dtype=np.float64)
    rho = rstd(x, eps)
    xh = x * rho[:, None]
    s = sigmoid(z)
    g = w[None, :] * (z * s)
    dx = _dx(x, g, dy, rho)
    dz = dy * xh * w[None, :] * s * (1.0 + z * (1.0 - s))
    dw = _sum_over_rows(dy * xh * (z * s))
    return dx, dz, dw


# ---------------------------------------------------------------------------
# Cancellation scales used by the parity tolerance.  They are not outputs of
# the method: they give, per element, the size of the largest term that
# cancels in an fp32 evaluation of dx or dz, so a test can allow for the
# rounding that cancellation amplifies.
# ---------------------------------------------------------------------------
def dx_cancellation_scale(x, w, dy, eps: float, z=None) -> np.ndarray:
    """max(|rho * g * dy|, |rho * xh| * mean_k |g_k * dy_k * xh_k|) per element.

    The two terms of dx are rho*g*dy and rho*xh*m.  m is a sum over the row, so
    its rounding error scales with the sum of the magnitudes of its terms, not
    with |m| (the dot-product error bound, Higham, "Accuracy and Stability of
    Numerical Algorithms", 2nd ed., section 3.1); the second term therefore uses
    mean_k |g_k dy_k xh_k| in place of |m|."""
    x, dy = _rows(x), _rows(dy)
    w = np.asarray(w, dtype=np.float64)
    rho = rstd(x, eps)
    xh = x * rho[:, None]
    if z is None:
        g = np.broadcast_to((1.0 + w)[None, :], x.shape)
    else:
        g = w[None, :] * silu(_rows(z))
    m_abs = np.sum(np.abs(g * dy * xh), axis=1) / x.shape[1]
    a = np.abs(rho[:, None] * g * dy)
    b = np.abs(rho[:, None] * xh * m_abs[:, None])
    return np.maximum(a, b)


def dz_cancellation_scale(x, z, w, dy, eps: float) -> np.ndarray:
    """|dy * xh * w * s| * max(1, |z * (1 - s)|) per element."""
    x, z, dy = _rows(x), _rows(z), _rows(dy)
    w = np.asarray(w, dtype=np.float64)
    rho = rstd(x, eps)
    s = sigmoid(z)
    lead = np.abs(dy * x * rho[:, None] * w[None, :] * s)
    return lead * np.maximum(1.0, np.abs(z * (1.0 - s)))


# ---------------------------------------------------------------------------
# The general operator: weight offset and gate activation as parameters.
# ---------------------------------------------------------------------------
ACTS = ("none", "silu", "sigmoid")


def _gain(w, weight_offset):
    w = np.asarray(w, dtype=np.float64)
    return w + weight_offset if weight_offset != 0 else w


def _act(z, act):
    """(a(z), a'(z)) for the gate; (1, 0) when there is none."""
    if act == "none":
        return 1.0, 0.0
    s = sigmoid(z)
    if act == "silu":
        return z * s, s * (1.0 + z * (1.0 - s))
    if act == "sigmoid":
        return s, s * (1.0 - s)
    raise ValueError(f"unknown activation {act!r}")


def rmsnorm_fwd(x, w, eps: float, weight_offset: float = 1.0, z=None, act: str = "none"):
    """y = x * rho * u * a(z) with u = w + offset (offset added only when
    nonzero).  Returns (y, rho)."""
    x = _rows(x)
    rho = rstd(x, eps)
    u = _gain(w, weight_offset)
    a, _ = _act(None if z is None else _rows(z), act)
    return x * rho[:, None] * u[None, :] * a, rho


def rmsnorm_bwd(x, w, dy, eps: float, weight_offset: float = 1.0, z=None, act: str = "none",
                row_mask=None):
    """Returns (dx, dz, dw); dz is None without a gate.  row_mask (one value per
    row, nonzero = the row counts) limits dw's sum to those rows; dx and dz are
    every row's.  A row outside the mask adds nothing, whatever its values."""
    x, dy = _rows(x), _rows(dy)
    rho = rstd(x, eps)
    xh = x * rho[:, None]
    u = _gain(w, weight_offset)[None, :]
    a, da = _act(None if z is None else _rows(z), act)
    g = u * a
    dx = _dx(x, np.broadcast_to(g, x.shape), dy, rho)
    dz = None if act == "none" else dy * xh * u * da
    contrib = dy * xh * a * np.ones_like(x)
    if row_mask is not None:
        contrib = contrib[np.asarray(row_mask).astype(bool)]
    dw = _sum_over_rows(contrib)
    return dx, dz, dw


def rmsnorm_dx_scale(x, w, dy, eps: float, weight_offset: float = 1.0, z=None,
                     act: str = "none") -> np.ndarray:
    """dx_cancellation_scale for the general operator (g = u * a(z))."""
    x, dy = _rows(x), _rows(dy)
    rho = rstd(x, eps)
    xh = x * rho[:, None]
    a, _ = _act(None if z is None else _rows(z), act)
    g = np.broadcast_to(_gain(w, weight_offset)[None, :] * a, x.shape)
    m_abs = np.sum(np.abs(g * dy * xh), axis=1) / x.shape[1]
    return np.maximum(np.abs(rho[:, None] * g * dy), np.abs(rho[:, None] * xh * m_abs[:, None]))


def rmsnorm_dz_scale(x, w, dy, eps: float, weight_offset: float, z, act: str) -> np.ndarray:
    """Largest term inside dz = dy*xh*u*s*c(z), c = 1 + z(1-s) (silu) or 1 - s
    (sigmoid): |dy*xh*u*s| times max(1, |z(1-s)|) for silu and 1 for the
    sigmoid, whose 1 - s is a difference of terms no larger than 1."""
    x, z, dy = _rows(x), _rows(z), _rows(dy)
    rho = rstd(x, eps)
    s = sigmoid(z)
    lead = np.abs(dy * x * rho[:, None] * _gain(w, weight_offset)[None, :] * s)
    if act == "silu":
        return lead * np.maximum(1.0, np.abs(z * (1.0 - s)))
    if act == "sigmoid":
        return lead
    raise ValueError(f"no dz without a gate (act {act!r})")


# ---------------------------------------------------------------------------
# Residual add.  [PR468] mentions an RMSNorm variant that also adds a residual
# ("Notes", on the strict profile's norm choice) and defines nothing more; read as the
# usual fused form: the residual stream h = x + r is stored in the tensors'
# format and normalised:
#     h = fmt(x + r),   y = h * rho(h) * u * a(z)
# The sum is formed in fp32 and rounded once to the format, the kernel's
# precision for that rounding decision (RFC #415 and PR #468 fix none).  Backward: the
# gradient reaching h is the norm's plus dh, the gradient of the residual
# output, and both x and r receive it:  dx = dr = dnorm(h; dy) + dh.
# ---------------------------------------------------------------------------
FORMATS = ("f32", "bf16", "f16", "f64")


def round_to_format(a, fmt: str) -> np.ndarray:
    """fp32 values rounded to nearest even in the 16-bit formats (f32 keeps
    them; f64 means no rounding at all).  Returns fp64."""
    if fmt == "f64":
        return np.asarray(a, dtype=np.float64)
    a32 = np.asarray(a, dtype=np.float32)
    if fmt == "f32":
        return a32.astype(np.float64)
    if fmt == "f16":
        return a32.astype(np.float16).astype(np.float64)   # IEEE round to nearest even
    if fmt == "bf16":
        # keep the top 16 bits of the fp32 encoding, rounding the dropped 16 to
        # nearest with ties to the even kept value (finite inputs)
        b = a32.view(np.uint32).astype(np.uint64)
        b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
        return b.astype(np.uint32).view(np.float32).astype(np.float64)
    raise ValueError(f"unknown format {fmt!r}")


def residual_add(x, r, fmt: str) -> np.ndarray:
    """h = fmt(fp32(x) + fp32(r)); x and r hold values of the format."""
    if fmt == "f64":
        return _rows(x) + _rows(r)
    s = np.asarray(x, dtype=np.float32) + np.asarray(r, dtype=np.float32)
    return round_to_format(s, fmt).reshape(_rows(x).shape)


def rmsnorm_add_fwd(x, r, w, eps: float, weight_offset: float = 1.0, z=None, act: str = "none",
                    fmt: str = "bf16"):
    """Returns (h, y, rho)."""
    h = residual_add(x, r, fmt)
    y, rho = rmsnorm_fwd(h, w, eps, weight_offset, z, act)
    return h, y, rho


def rmsnorm_add_bwd(h, w, dy, dh, eps: float, weight_offset: float = 1.0, z=None,
                    act: str = "none", row_mask=None):
    """Returns (dx, dz, dw); dx is the gradient of both x and r."""
    dx, dz, dw = rmsnorm_bwd(h, w, dy, eps, weight_offset, z, act, row_mask)
    if dh is not None:
        dx = dx + _rows(dh)
    return dx, dz, dw
