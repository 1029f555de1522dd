"""Planted mistakes in copies of the oracle (CPU only).

Each mutant replaces one function of a freshly loaded copy of
``oracle/rmsnorm.py`` with a version carrying one plausible mistake -- a dropped
term, a wrong sign, a wrong divisor, the offset added where it does not belong --
and the test asserts that at least one pin in ``oracle_pins`` fails for it.
The real oracle is never modified.
"""
import importlib.util
import os

import numpy as np
import pytest

import oracle_pins

ORACLE_SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                          "oracle", "rmsnorm.py")


def fresh():
    spec = importlib.util.spec_from_file_location("oracle_mutant", ORACLE_SRC)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def m_eps_outside_sqrt(o):
    def rstd(x, eps):
        x = np.asarray(x, dtype=np.float64)
        return 1.0 / (np.sqrt(np.sum(x * x, axis=1) / x.shape[1]) + eps)
    o.rstd = rstd


def m_mean_over_h_minus_1(o):
    def rstd(x, eps):
        x = np.asarray(x, dtype=np.float64)
        return 1.0 / np.sqrt(np.sum(x * x, axis=1) / (x.shape[1] - 1) + eps)
    o.rstd = rstd


def m_eps_dropped(o):
    def rstd(x, eps):
        x = np.asarray(x, dtype=np.float64)
        return 1.0 / np.sqrt(np.sum(x * x, axis=1) / x.shape[1])
    o.rstd = rstd


def m_no_offset(o):
    def norm_fwd(x, w, eps):
        x = np.asarray(x, dtype=np.float64); w = np.asarray(w, dtype=np.float64)
        rho = o.rstd(x, eps)
        return x * rho[:, None] * w[None, :], rho
    o.norm_fwd = norm_fwd


def m_gate_sigmoid_not_silu(o):
    def gated_norm_fwd(x, z, w, eps):
        x = np.asarray(x, dtype=np.float64); z = np.asarray(z, dtype=np.float64)
        w = np.asarray(w, dtype=np.float64)
        rho = o.rstd(x, eps)
        return x * rho[:, None] * w[None, :] * o.sigmoid(z), rho
    o.gated_norm_fwd = gated_norm_fwd


def m_sigmoid_sign(o):
    o.sigmoid = lambda z: 1.0 / (1.0 + np.exp(np.asarray(z, dtype=np.float64)))


def m_dx_drops_mean_term(o):
    def _dx(x, g, dy, rho):
        return rho[:, None] * (g * dy)
    o._dx = _dx


def m_dx_mean_not_divided(o):
    def _dx(x, g, dy, rho):
        xh = x * rho[:, None]
        m = np.sum(g * dy * xh, axis=1)
        return rho[:, None] * (g * dy - xh * m[:, None])
    o._dx = _dx


def m_dx_drops_rho(o):
    def _dx(x, g, dy, rho):
        xh = x * rho[:, None]
        m = np.sum(g * dy * xh, axis=1) / x.shape[1]
        return g * dy - xh * m[:, None]
    o._dx = _dx


def m_dx_sign(o):
    def _dx(x, g, dy, rho):
        xh = x * rho[:, None]
        m = np.sum(g * dy * xh, axis=1) / x.shape[1]
        return rho[:, None] * (g * dy + xh * m[:, None])
    o._dx = _dx


def m_dz_drops_one_minus_s(o):
    def gated_norm_bwd(x, z, w, dy, eps):
        x = np.asarray(x, dtype=np.float64); z = np.asarray(z, dtype=np.float64)
        w = np.asarray(w, dtype=np.float64); dy = np.asarray(dy, dtype=np.float64)
        rho = o.rstd(x, eps); xh = x * rho[:, None]; s = o.sigmoid(z)
        dx = o._dx(x, w[None, :] * z * s, dy, rho)
        dz = dy * xh * w[None, :] * s * (1.0 + z)
        return dx, dz, np.sum(dy * xh * z * s, axis=0)
    o.gated_norm_bwd = gated_norm_bwd


def m_dz_sigmoid_derivative_only(o):
    def gated_norm_bwd(x, z, w, dy, eps):
        x = np.asarray(x, dtype=np.float64); z = np.asarray(z, dtype=np.float64)
        w = np.asarray(w, dtype=np.float64); dy = np.asarray(dy, dtype=np.float64)
        rho = o.rstd(x, eps); xh = x * rho[:, None]; s = o.sigmoid(z)
        dx = o._dx(x, w[None, :] * z * s, dy, rho)
        dz = dy * xh * w[None, :] * s * (1.0 - s)
        return dx, dz, np.sum(dy * xh * z * s, axis=0)
    o.gated_norm_bwd = gated_norm_bwd


def m_gated_dw_drops_gate(o):
    def gated_norm_bwd(x, z, w, dy, eps):
        x = np.asarray(x, dtype=np.float64); z = np.asarray(z, dtype=np.float64)
        w = np.asarray(w, dtype=np.float64); dy = np.asarray(dy, dtype=np.float64)
        rho = o.rstd(x, eps); xh = x * rho[:, None]; s = o.sigmoid(z)
        dx = o._dx(x, w[None, :] * z * s, dy, rho)
        dz = dy * xh * w[None, :] * s * (1.0 + z * (1.0 - s))
        return dx, dz, np.sum(dy * xh, axis=0)
    o.gated_norm_bwd = gated_norm_bwd


def m_gated_gain_adds_offset(o):
    def gated_norm_bwd(x, z, w, dy, eps):
        x = np.asarray(x, dtype=np.float64); z = np.asarray(z, dtype=np.float64)
        w = np.asarray(w, dtype=np.float64); dy = np.asarray(dy, dtype=np.float64)
        rho = o.rstd(x, eps); xh = x * rho[:, None]; s = o.sigmoid(z)
        dx = o._dx(x, (1.0 + w[None, :]) * z * s, dy, rho)
        dz = dy * xh * w[None, :] * s * (1.0 + z * (1.0 - s))
        return dx, dz, np.sum(dy * xh * z * s, axis=0)
    o.gated_norm_bwd = gated_norm_bwd


def m_norm_dw_uses_x(o):
    def norm_bwd(x, w, dy, eps):
        x = np.asarray(x, dtype=np.float64); w = np.asarray(w, dtype=np.float64)
        dy = np.asarray(dy, dtype=np.float64)
        rho = o.rstd(x, eps)
        dx = o._dx(x, np.broadcast_to((1.0 + w)[None, :], x.shape), dy, rho)
        return dx, np.sum(dy * x, axis=0)
    o.norm_bwd = norm_bwd


def m_norm_dw_wrong_axis(o):
    def norm_bwd(x, w, dy, eps):
        x = np.asarray(x, dtype=np.float64); w = np.asarray(w, dtype=np.float64)
        dy = np.asarray(dy, dtype=np.float64)
        rho = o.rstd(x, eps)
        dx = o._dx(x, np.broadcast_to((1.0 + w)[None, :], x.shape), dy, rho)
        c = dy * x * rho[:, None]
        return dx, c[-1]          # last row only instead of the sum over rows
    o.norm_bwd = norm_bwd


def m_general_offset_always_added(o):
    o._gain = lambda w, off: np.asarray(w, dtype=np.float64) + off


def m_general_offset_never_added(o):
    o._gain = lambda w, off: np.asarray(w, dtype=np.float64)


def m_general_sigmoid_takes_silu_derivative(o):
    real = o._act

    def _act(z, act):
        a, da = real(z, act)
        if act == "sigmoid":
            s = o.sigmoid(z)
            da = s * (1.0 + z * (1.0 - s))
        return a, da
    o._act = _act


def m_general_sigmoid_gate_is_silu(o):
    real = o._act
    o._act = lambda z, act: real(z, "silu" if act == "sigmoid" else act)


def m_general_dz_without_offset(o):
    real = o.rmsnorm_bwd

    def rmsnorm_bwd(x, w, dy, eps, weight_offset=1.0, z=None, act="none"):
        dx, dz, dw = real(x, w, dy, eps, weight_offset, z, act)
        if dz is not None and weight_offset != 0:
            u = o._gain(w, weight_offset)
            dz = dz / u[None, :] * np.asarray(w, dtype=np.float64)[None, :]
        return dx, dz, dw
    o.rmsnorm_bwd = rmsnorm_bwd


def m_general_dw_drops_gate(o):
    real = o.rmsnorm_bwd

    def rmsnorm_bwd(x, w, dy, eps, weight_offset=1.0, z=None, act="none"):
        dx, dz, _ = real(x, w, dy, eps, weight_offset, z, act)
        x = np.asarray(x, dtype=np.float64)
        xh = x * o.rstd(x, eps)[:, None]
        return dx, dz, np.sum(np.asarray(dy, dtype=np.float64) * xh, axis=0)
    o.rmsnorm_bwd = rmsnorm_bwd


def m_mask_ignored(o):
    real = o.rmsnorm_bwd
    o.rmsnorm_bwd = lambda x, w, dy, eps, weight_offset=1.0, z=None, act="none", row_mask=None: \
        real(x, w, dy, eps, weight_offset, z, act)


def m_mask_inverted(o):
    real = o.rmsnorm_bwd

    def rmsnorm_bwd(x, w, dy, eps, weight_offset=1.0, z=None, act="none", row_mask=None):
        m = None if row_mask is None else 1 - np.asarray(row_mask)
        if m is not None and not m.any():
            m = None
        return real(x, w, dy, eps, weight_offset, z, act, m)
    o.rmsnorm_bwd = rmsnorm_bwd


def m_mask_zeroes_dx(o):
    real = o.rmsnorm_bwd

    def rmsnorm_bwd(x, w, dy, eps, weight_offset=1.0, z=None, act="none", row_mask=None):
        dx, dz, dw = real(x, w, dy, eps, weight_offset, z, act, row_mask)
        if row_mask is not None:
            dx = dx * np.asarray(row_mask, dtype=np.float64)[:, None]
        return dx, dz, dw
    o.rmsnorm_bwd = rmsnorm_bwd


def m_mask_multiplies_contributions(o):
    # a multiply by the mask instead of leaving rows out: NaN * 0 is NaN
    real = o.rmsnorm_bwd

    def rmsnorm_bwd(x, w, dy, eps, weight_offset=1.0, z=None, act="none", row_mask=None):
        dx, dz, dw = real(x, w, dy, eps, weight_offset, z, act)
        if row_mask is not None:
            xr = np.asarray(x, dtype=np.float64)
            rho = o.rstd(xr, eps)
            a, _ = o._act(None if z is None else np.asarray(z, dtype=np.float64), act)
            c = np.asarray(dy, dtype=np.float64) * xr * rho[:, None] * a
            dw = np.sum(c * np.asarray(row_mask, dtype=np.float64)[:, None], axis=0)
        return dx, dz, dw
    o.rmsnorm_bwd = rmsnorm_bwd


def m_residual_not_rounded(o):
    real = o.residual_add
    o.residual_add = lambda x, r, fmt: real(x, r, "f64")


def m_residual_dh_dropped(o):
    real = o.rmsnorm_add_bwd
    o.rmsnorm_add_bwd = lambda h, w, dy, dh, eps, weight_offset=1.0, z=None, act="none", \
        row_mask=None: real(h, w, dy, None, eps, weight_offset, z, act, row_mask)


def m_residual_norm_of_unrounded_sum(o):
    def rmsnorm_add_fwd(x, r, w, eps, weight_offset=1.0, z=None, act="none", fmt="bf16"):
        h = o.residual_add(x, r, fmt)
        y, rho = o.rmsnorm_fwd(o.residual_add(x, r, "f64"), w, eps, weight_offset, z, act)
        return h, y, rho
    o.rmsnorm_add_fwd = rmsnorm_add_fwd


def m_bf16_round_truncates(o):
    real = o.round_to_format

    def round_to_format(a, fmt):
        if fmt != "bf16":
            return real(a, fmt)
        b = np.asarray(a, dtype=np.float32).view(np.uint32) & np.uint32(0xFFFF0000)
        return b.view(np.float32).astype(np.float64)
    o.round_to_format = round_to_format


def m_bf16_round_ties_up(o):
    real = o.round_to_format

    def round_to_format(a, fmt):
        if fmt != "bf16":
            return real(a, fmt)
        b = np.asarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
        b = (b + 0x8000) & 0xFFFF0000
        return b.astype(np.uint32).view(np.float32).astype(np.float64)
    o.round_to_format = round_to_format


def m_rstd_sqrt_not_rsqrt(o):
    def rstd(x, eps):
        x = np.asarray(x, dtype=np.float64)
        return np.sqrt(np.sum(x * x, axis=1) / x.shape[1] + eps)
    o.rstd = rstd


def m_rstd_mean_over_rows(o):
    # the mean square taken down a column (over the batch) instead of along the row
    def rstd(x, eps):
        x = np.asarray(x, dtype=np.float64)
        col = np.sum(x * x, axis=0) / x.shape[0]
        return 1.0 / np.sqrt(np.resize(col, x.shape[0]) + eps)
    o.rstd = rstd


def m_dx_mean_drops_xh(o):
    def _dx(x, g, dy, rho):
        m = np.sum(g * dy, axis=1) / x.shape[1]
        return rho[:, None] * (g * dy - x * rho[:, None] * m[:, None])
    o._dx = _dx


def m_dw_rows_shifted(o):
    # each row's contribution pairs its xh with the next row's dy (an index slip)
    real = o.rmsnorm_bwd

    def rmsnorm_bwd(x, w, dy, eps, weight_offset=1.0, z=None, act="none", row_mask=None):
        dx, dz, _ = real(x, w, dy, eps, weight_offset, z, act, row_mask)
        _, _, dw = real(x, w, np.roll(np.asarray(dy, dtype=np.float64), 1, axis=0), eps,
                        weight_offset, z, act, row_mask)
        return dx, dz, dw
    o.rmsnorm_bwd = rmsnorm_bwd


def m_sigmoid_derivative_sign(o):
    real = o._act

    def _act(z, act):
        a, da = real(z, act)
        if act == "sigmoid":
            s = o.sigmoid(z)
            da = s * (1.0 + s)
        return a, da
    o._act = _act


def m_general_dz_drops_weight(o):
    real = o.rmsnorm_bwd

    def rmsnorm_bwd(x, w, dy, eps, weight_offset=1.0, z=None, act="none", row_mask=None):
        dx, dz, dw = real(x, w, dy, eps, weight_offset, z, act, row_mask)
        if dz is not None:
            u = o._gain(w, weight_offset)[None, :]
            with np.errstate(all="ignore"):
                dz = np.where(u != 0, dz / u, dz)
        return dx, dz, dw
    o.rmsnorm_bwd = rmsnorm_bwd


def m_residual_subtracts(o):
    def residual_add(x, r, fmt):
        if fmt == "f64":
            return o._rows(x) - o._rows(r)
        s = np.asarray(x, dtype=np.float32) - np.asarray(r, dtype=np.float32)
        return o.round_to_format(s, fmt).reshape(o._rows(x).shape)
    o.residual_add = residual_add


def m_f16_round_as_bf16(o):
    real = o.round_to_format
    o.round_to_format = lambda a, fmt: real(a, "bf16" if fmt == "f16" else fmt)


# --- the cancellation scales of the dx / dz tolerance ----------------------
def m_dx_scale_times_1024(o):
    real = o.dx_cancellation_scale
    o.dx_cancellation_scale = lambda *a, **k: 1024.0 * real(*a, **k)


def m_dx_scale_over_1024(o):
    real = o.dx_cancellation_scale
    o.dx_cancellation_scale = lambda *a, **k: real(*a, **k) / 1024.0


def m_dx_scale_uses_abs_m(o):
    def dx_cancellation_scale(x, w, dy, eps, z=None):
        x, dy = o._rows(x), o._rows(dy)
        w = np.asarray(w, dtype=np.float64)
        rho = o.rstd(x, eps)
        xh = x * rho[:, None]
        g = np.broadcast_to((1.0 + w)[None, :], x.shape) if z is None else \
            w[None, :] * o.silu(o._rows(z))
        m = np.abs(np.sum(g * dy * xh, axis=1)) / x.shape[1]
        return np.maximum(np.abs(rho[:, None] * g * dy), np.abs(rho[:, None] * xh * m[:, None]))
    o.dx_cancellation_scale = dx_cancellation_scale


def m_dz_scale_drops_silu_factor(o):
    def dz_cancellation_scale(x, z, w, dy, eps):
        x, z, dy = o._rows(x), o._rows(z), o._rows(dy)
        rho = o.rstd(x, eps)
        return np.abs(dy * x * rho[:, None] * np.asarray(w)[None, :] * o.sigmoid(z))
    o.dz_cancellation_scale = dz_cancellation_scale


def m_dz_scale_times_1024(o):
    real = o.dz_cancellation_scale
    o.dz_cancellation_scale = lambda *a, **k: 1024.0 * real(*a, **k)


def m_general_dx_scale_over_1024(o):
    real = o.rmsnorm_dx_scale
    o.rmsnorm_dx_scale = lambda *a, **k: real(*a, **k) / 1024.0


def m_general_dx_scale_times_1024(o):
    real = o.rmsnorm_dx_scale
    o.rmsnorm_dx_scale = lambda *a, **k: 1024.0 * real(*a, **k)


def m_general_dx_scale_drops_mean_term(o):
    def rmsnorm_dx_scale(x, w, dy, eps, weight_offset=1.0, z=None, act="none"):
        x, dy = o._rows(x), o._rows(dy)
        rho = o.rstd(x, eps)
        a, _ = o._act(None if z is None else o._rows(z), act)
        g = np.broadcast_to(o._gain(w, weight_offset)[None, :] * a, x.shape)
        return np.abs(rho[:, None] * g * dy)
    o.rmsnorm_dx_scale = rmsnorm_dx_scale


def m_general_dz_scale_over_1024(o):
    real = o.rmsnorm_dz_scale
    o.rmsnorm_dz_scale = lambda *a, **k: real(*a, **k) / 1024.0


def m_general_dz_scale_drops_silu_factor(o):
    def rmsnorm_dz_scale(x, w, dy, eps, weight_offset, z, act):
        x, z, dy = o._rows(x), o._rows(z), o._rows(dy)
        rho = o.rstd(x, eps)
        return np.abs(dy * x * rho[:, None] * o._gain(w, weight_offset)[None, :] * o.sigmoid(z))
    o.rmsnorm_dz_scale = rmsnorm_dz_scale


def m_general_dz_scale_silu_factor_for_sigmoid(o):
    real = o.rmsnorm_dz_scale
    o.rmsnorm_dz_scale = lambda x, w, dy, eps, off, z, act: real(x, w, dy, eps, off, z, "silu")


# --- the empty sum --------------------------------------------------------
def m_empty_sum_is_positive_zero(o):
    o._sum_over_rows = lambda c: np.sum(np.asarray(c, dtype=np.float64), axis=0)


MUTANTS = [m for name, m in sorted(globals().items()) if name.startswith("m_")]


def test_real_oracle_passes_every_pin():
    assert oracle_pins.failing_pins(fresh()) == []


@pytest.mark.parametrize("mutate", MUTANTS, ids=lambda m: m.__name__)
def test_mutant_is_caught(mutate):
    o = fresh()
    mutate(o)
    bad = oracle_pins.failing_pins(o)
    assert bad, f"no pin catches {mutate.__name__}"
