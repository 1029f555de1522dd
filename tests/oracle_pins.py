"""Pins that tie the fp64 oracle to facts other than itself.

Each ``pin_*`` takes an oracle-like module and raises AssertionError when the
module disagrees with a closed form, an exact hand-derived worked example, a
finite-difference derivative, an identity or a brute-force loop.
``test_oracle_pins.py`` runs them on the real oracle; ``test_oracle_mutations.py``
plants plausible mistakes in copies of the oracle and checks that at least one
pin fails for each.

The operators are those of RL-Kernel PR #468 ("[WS1][CUDA][Qwen3-Next] Gated
RMSNorm CUDA kernel for the GDN block", Summary): zero-centred RMSNorm
y = x*rstd*(1+w) and gated RMSNorm y = x*rstd*w*silu(z), and their gradients.
RFC #415 and PR #468 print no worked numeric example, so the worked examples here are
derived by hand with exact rational arithmetic; the derivations are written out
next to each one.
"""
from __future__ import annotations

import math

import numpy as np

L3 = math.log(3.0)


def _close(got, want, rtol=1e-13, atol=1e-15, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, f"{what}: shape {got.shape} != {want.shape}"
    err = np.abs(got - want)
    lim = atol + rtol * np.abs(want)
    assert np.all(err <= lim), f"{what}: max err {err.max():.3e}\n got={got}\nwant={want}"


# --------------------------------------------------------------------------
# worked examples (exact)
# --------------------------------------------------------------------------
def pin_worked_example_norm(orc):
    """H=4, x=[1,2,2,4], eps=0: sum x^2 = 25, ms = 25/4, rho = 2/5,
    xh = [2/5, 4/5, 4/5, 8/5].  w = [0, 1/2, -1, 1] -> g = 1+w = [1, 3/2, 0, 2],
    y = xh*g = [2/5, 6/5, 0, 16/5].
    dy = [1, -1, 2, 1/2]: g*dy = [1, -3/2, 0, 1]; g*dy*xh = [2/5, -6/5, 0, 8/5],
    sum = 4/5, m = 1/5; xh*m = [2, 4, 4, 8]/25;
    g*dy - xh*m = [23/25, -83/50, -4/25, 17/25];
    dx = rho*(...) = [46, -83, -8, 34]/125;  dw = dy*xh = [2/5, -4/5, 8/5, 4/5]."""
    x = [[1.0, 2.0, 2.0, 4.0]]
    w = [0.0, 0.5, -1.0, 1.0]
    dy = [[1.0, -1.0, 2.0, 0.5]]
    y, rho = orc.norm_fwd(x, w, 0.0)
    _close(rho, [0.4], what="rho")
    _close(y, [[0.4, 1.2, 0.0, 3.2]], what="y")
    _close(orc.rstd(x, 0.0), [0.4], what="rstd")
    dx, dw = orc.norm_bwd(x, w, dy, 0.0)
    _close(dx, [[46 / 125, -83 / 125, -8 / 125, 34 / 125]], what="dx")
    _close(dw, [0.4, -0.8, 1.6, 0.8], what="dw")


def pin_worked_example_eps(orc):
    """eps sits inside the square root, added to the mean square.
    H=2, x=[3,4]: ms = 25/2; eps = 7/2 -> ms+eps = 16, rho = 1/4, xh = [3/4, 1].
    w = [1, -1/2] -> g = [2, 1/2], y = [3/2, 1/2].  dy = [1, 1]:
    g*dy*xh = [3/2, 1/2], m = 2/2 = 1; g*dy - xh*m = [5/4, -1/2];
    dx = [5/16, -1/8]; dw = dy*xh = [3/4, 1]."""
    x = [[3.0, 4.0]]
    w = [1.0, -0.5]
    dy = [[1.0, 1.0]]
    y, rho = orc.norm_fwd(x, w, 3.5)
    _close(rho, [0.25], what="rho")
    _close(y, [[1.5, 0.5]], what="y")
    dx, dw = orc.norm_bwd(x, w, dy, 3.5)
    _close(dx, [[5 / 16, -1 / 8]], what="dx")
    _close(dw, [0.75, 1.0], what="dw")


def pin_worked_example_gated(orc):
    """Gated, H=4, x=[1,2,2,4], eps=0 (rho=2/5, xh=[2,4,4,8]/5), L = ln 3,
    z = [L, -L, 0, L] so s(z) = [3/4, 1/4, 1/2, 3/4] and
    silu(z) = [3L/4, -L/4, 0, 3L/4];  w = [1, 2, 5, -1].
    y = xh*w*silu = [3L/10, -2L/5, 0, -6L/5].
    dy = [1, -1, 2, 1/2]: g = w*silu = [3L/4, -L/2, 0, -3L/4];
    g*dy*xh = [3L/10, 2L/5, 0, -3L/5], sum = L/10, m = L/40;
    g*dy - xh*m = [37L/50, 12L/25, -L/50, -83L/200];
    dx = [37L/125, 24L/125, -L/125, -83L/500];
    dz = dy*xh*w*s*(1+z*(1-s)) = [(3/10)(1+L/4), -(2/5)(1-3L/4), 4, -(3/5)(1+L/4)];
    dw = dy*xh*silu = [3L/10, L/5, 0, 3L/5]."""
    L = L3
    x = [[1.0, 2.0, 2.0, 4.0]]
    z = [[L, -L, 0.0, L]]
    w = [1.0, 2.0, 5.0, -1.0]
    dy = [[1.0, -1.0, 2.0, 0.5]]
    y, rho = orc.gated_norm_fwd(x, z, w, 0.0)
    _close(rho, [0.4], what="rho")
    _close(y, [[3 * L / 10, -2 * L / 5, 0.0, -6 * L / 5]], what="y")
    dx, dz, dw = orc.gated_norm_bwd(x, z, w, dy, 0.0)
    _close(dx, [[37 * L / 125, 24 * L / 125, -L / 125, -83 * L / 500]], what="dx")
    _close(dz, [[0.3 * (1 + L / 4), -0.4 * (1 - 3 * L / 4), 4.0, -0.6 * (1 + L / 4)]],
           what="dz")
    _close(dw, [3 * L / 10, L / 5, 0.0, 3 * L / 5], what="dw")


def pin_sigmoid_points(orc):
    """s(ln k) = k/(k+1); s(0) = 1/2; saturates without NaN at +-800."""
    ks = np.array([1.0, 3.0, 1 / 3, 7.0, 0.125])
    _close(orc.sigmoid(np.log(ks)), ks / (ks + 1.0), what="sigmoid")
    _close(orc.silu(np.log(ks)), np.log(ks) * ks / (ks + 1.0), what="silu")
    s = orc.sigmoid(np.array([800.0, -800.0]))
    assert s[0] == 1.0 and s[1] == 0.0, s
    assert np.all(np.isfinite(orc.silu(np.array([800.0, -800.0]))))


# --------------------------------------------------------------------------
# closed forms and invariants on random data
# --------------------------------------------------------------------------
def pin_constant_row(orc):
    """A constant row c gives ms = c^2, so y = c/sqrt(c^2+eps) * (1+w), and
    gated y = c/sqrt(c^2+eps) * w * silu(z) with silu at exact ln(k) points."""
    rng = np.random.default_rng(11)
    H = 16
    for c in (1e-3, -0.7, 2.5, 40.0):
        for eps in (0.0, 1e-6, 0.3):
            x = np.full((1, H), c)
            w = rng.normal(0.0, 0.5, H)
            base = c / math.sqrt(c * c + eps)
            y, rho = orc.norm_fwd(x, w, eps)
            _close(rho, [1.0 / math.sqrt(c * c + eps)], rtol=1e-14, what="rho")
            _close(y, base * (1.0 + w)[None, :], rtol=1e-14, what="y")
            ks = rng.choice([0.25, 1 / 3, 1.0, 3.0, 9.0], size=H)
            z = np.log(ks)[None, :]
            silu_exact = np.log(ks) * ks / (ks + 1.0)
            yg, _ = orc.gated_norm_fwd(x, z, w, eps)
            _close(yg, base * (w * silu_exact)[None, :], rtol=1e-13, atol=1e-15, what="yg")


def pin_unit_rms(orc):
    """At eps = 0 the normalised row has mean square exactly 1 (mean over H, not
    H-1), and with w = 0 the zero-centred output is that normalised row."""
    rng = np.random.default_rng(12)
    for H in (3, 8, 128):
        x = rng.normal(0.0, 2.0, (5, H))
        y, rho = orc.norm_fwd(x, np.zeros(H), 0.0)
        _close(np.mean(y * y, axis=1), np.ones(5), rtol=1e-14, what="ms(xh)")
        _close(y, x * rho[:, None], rtol=1e-15, what="xh")
        yg, rg = orc.gated_norm_fwd(x, np.zeros((5, H)), np.ones(H), 0.0)
        _close(rg, rho, rtol=0, atol=0, what="gated rstd == plain rstd")


def pin_eps_shrinks_rms(orc):
    """With eps > 0 the normalised row's mean square is ms/(ms+eps)."""
    rng = np.random.default_rng(13)
    x = rng.normal(0.0, 0.01, (4, 32))
    eps = 1e-4
    ms = np.mean(x * x, axis=1)
    y, _ = orc.norm_fwd(x, np.zeros(32), eps)
    _close(np.mean(y * y, axis=1), ms / (ms + eps), rtol=1e-13, what="ms(xh)")


def pin_scale_invariance(orc):
    """At eps = 0 the outputs do not change when a row is scaled by a > 0."""
    rng = np.random.default_rng(14)
    x = rng.normal(size=(3, 24))
    z = rng.normal(size=(3, 24))
    w = rng.normal(size=24)
    for a in (1e-3, 0.5, 7.0, 1e4):
        _close(orc.norm_fwd(a * x, w, 0.0)[0], orc.norm_fwd(x, w, 0.0)[0], rtol=1e-13,
               atol=1e-14, what="norm y(ax)")
        _close(orc.gated_norm_fwd(a * x, z, w, 0.0)[0], orc.gated_norm_fwd(x, z, w, 0.0)[0],
               rtol=1e-13, atol=1e-14, what="gated y(ax)")


def pin_scale_identity(orc):
    """sum_j x_j dx_j = rho * S * eps / (ms + eps), S = sum_j g_j dy_j x_j:
    the derivative of L along x itself, from y(a x) at eps = 0 being flat.
    Checked through the zero-centred op (g = 1+w) and the gated op."""
    rng = np.random.default_rng(15)
    R, H = 6, 40
    x = rng.normal(size=(R, H))
    z = rng.normal(size=(R, H))
    w = rng.normal(size=H)
    dy = rng.normal(size=(R, H))
    for eps in (0.0, 1e-3, 0.5):
        ms = np.mean(x * x, axis=1)
        rho = 1.0 / np.sqrt(ms + eps)
        dx, _ = orc.norm_bwd(x, w, dy, eps)
        S = np.sum((1.0 + w)[None, :] * dy * x, axis=1)
        _close(np.sum(x * dx, axis=1), rho * S * eps / (ms + eps), rtol=1e-10, atol=1e-12,
               what="norm identity")
        dxg, _, _ = orc.gated_norm_bwd(x, z, w, dy, eps)
        zs = z / (1.0 + np.exp(-z))
        Sg = np.sum(w[None, :] * zs * dy * x, axis=1)
        _close(np.sum(x * dxg, axis=1), rho * Sg * eps / (ms + eps), rtol=1e-10, atol=1e-12,
               what="gated identity")


def _fd(f, a, h=1e-5):
    """Central differences with one Richardson step, elementwise over ``a``."""
    g = np.zeros_like(a)
    it = np.nditer(a, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        def d(step):
            ap = a.copy(); ap[i] += step
            am = a.copy(); am[i] -= step
            return (f(ap) - f(am)) / (2 * step)
        g[i] = (4 * d(h / 2) - d(h)) / 3
    return g


def pin_finite_differences(orc):
    """dx, dz, dw equal the numerical gradient of L = sum(y * dy)."""
    rng = np.random.default_rng(16)
    R, H, eps = 3, 8, 1e-2
    x = rng.normal(size=(R, H))
    z = rng.normal(size=(R, H)) * 2.0
    w = rng.normal(size=H)
    dy = rng.normal(size=(R, H))

    def L_norm(x_, w_):
        return float(np.sum(orc.norm_fwd(x_, w_, eps)[0] * dy))

    def L_gated(x_, z_, w_):
        return float(np.sum(orc.gated_norm_fwd(x_, z_, w_, eps)[0] * dy))

    dx, dw = orc.norm_bwd(x, w, dy, eps)
    _close(dx, _fd(lambda a: L_norm(a, w), x), rtol=1e-7, atol=1e-8, what="norm dx")
    _close(dw, _fd(lambda a: L_norm(x, a), w), rtol=1e-7, atol=1e-8, what="norm dw")
    dx, dz, dw = orc.gated_norm_bwd(x, z, w, dy, eps)
    _close(dx, _fd(lambda a: L_gated(a, z, w), x), rtol=1e-7, atol=1e-8, what="gated dx")
    _close(dz, _fd(lambda a: L_gated(x, a, w), z), rtol=1e-7, atol=1e-8, what="gated dz")
    _close(dw, _fd(lambda a: L_gated(x, z, a), w), rtol=1e-7, atol=1e-8, what="gated dw")


def pin_dw_brute_force(orc):
    """dw recomputed by an explicit loop over rows and columns, using the
    per-row forward outputs (dy * y / (1+w) is dy * xh for the zero-centred op;
    gated: dy * y / w is dy * xh * silu(z))."""
    rng = np.random.default_rng(17)
    R, H, eps = 9, 5, 1e-6
    x = rng.normal(size=(R, H))
    z = rng.normal(size=(R, H))
    w = rng.uniform(0.5, 1.5, size=H)          # nonzero so the ratios exist
    dy = rng.normal(size=(R, H))
    _, dw = orc.norm_bwd(x, w, dy, eps)
    _, _, dwg = orc.gated_norm_bwd(x, z, w, dy, eps)
    want = [0.0] * H
    want_g = [0.0] * H
    for r in range(R):
        y, _ = orc.norm_fwd(x[r:r + 1], w, eps)
        yg, _ = orc.gated_norm_fwd(x[r:r + 1], z[r:r + 1], w, eps)
        for j in range(H):
            want[j] += dy[r, j] * y[0, j] / (1.0 + w[j])
            want_g[j] += dy[r, j] * yg[0, j] / w[j]
    _close(dw, want, rtol=1e-12, atol=1e-14, what="norm dw")
    _close(dwg, want_g, rtol=1e-12, atol=1e-14, what="gated dw")


def pin_rows_independent(orc):
    """Each row's outputs depend only on that row (computed alone == in batch)."""
    rng = np.random.default_rng(18)
    x = rng.normal(size=(5, 12)); z = rng.normal(size=(5, 12))
    w = rng.normal(size=12); dy = rng.normal(size=(5, 12))
    y, _ = orc.gated_norm_fwd(x, z, w, 1e-6)
    dx, dz, _ = orc.gated_norm_bwd(x, z, w, dy, 1e-6)
    for r in range(5):
        s = slice(r, r + 1)
        _close(orc.gated_norm_fwd(x[s], z[s], w, 1e-6)[0], y[s], rtol=0, atol=0, what="y row")
        a, b, _ = orc.gated_norm_bwd(x[s], z[s], w, dy[s], 1e-6)
        _close(a, dx[s], rtol=0, atol=0, what="dx row")
        _close(b, dz[s], rtol=0, atol=0, what="dz row")


# --------------------------------------------------------------------------
# the general operator: weight offset and gate activation
# --------------------------------------------------------------------------
def pin_worked_example_sigmoid_offset(orc):
    """Sigmoid gate with offset 1, H=4, x=[1,2,2,4], eps=0 (rho=2/5,
    xh=[2,4,4,8]/5), L = ln 3, z = [L, -L, 0, L]: a = s(z) = [3/4, 1/4, 1/2, 3/4],
    a' = s(1-s) = [3/16, 3/16, 1/4, 3/16].  w = [0, 1/2, -1, 1] -> u = w+1 =
    [1, 3/2, 0, 2];  y = xh*u*a = [3/10, 3/10, 0, 12/5].
    dy = [1, -1, 2, 1/2]: g = u*a = [3/4, 3/8, 0, 3/2]; g*dy*xh = [3/10, -3/10,
    0, 6/5], sum = 6/5, m = 3/10; xh*m = [3, 6, 6, 12]/25;
    g*dy - xh*m = [63/100, -123/200, -6/25, 27/100];
    dx = [63/250, -123/500, -12/125, 27/250];
    dz = dy*xh*u*a' = [3/40, -9/40, 0, 3/10];  dw = dy*xh*a = [3/10, -1/5, 4/5, 3/5]."""
    L = L3
    x = [[1.0, 2.0, 2.0, 4.0]]
    z = [[L, -L, 0.0, L]]
    w = [0.0, 0.5, -1.0, 1.0]
    dy = [[1.0, -1.0, 2.0, 0.5]]
    y, rho = orc.rmsnorm_fwd(x, w, 0.0, weight_offset=1.0, z=z, act="sigmoid")
    _close(rho, [0.4], what="rho")
    _close(y, [[0.3, 0.3, 0.0, 2.4]], what="y")
    dx, dz, dw = orc.rmsnorm_bwd(x, w, dy, 0.0, weight_offset=1.0, z=z, act="sigmoid")
    _close(dx, [[63 / 250, -123 / 500, -12 / 125, 27 / 250]], what="dx")
    _close(dz, [[3 / 40, -9 / 40, 0.0, 0.3]], what="dz")
    _close(dw, [0.3, -0.2, 0.8, 0.6], what="dw")


def pin_general_special_cases(orc):
    """Offset 1 without a gate is the zero-centred operator; offset 0 with the
    silu gate is the gated operator (both pinned above by worked examples)."""
    rng = np.random.default_rng(19)
    x = rng.normal(size=(3, 8)); z = rng.normal(size=(3, 8))
    w = rng.normal(size=8); dy = rng.normal(size=(3, 8))
    _close(orc.rmsnorm_fwd(x, w, 1e-6)[0], orc.norm_fwd(x, w, 1e-6)[0], what="plain y")
    dx, dz, dw = orc.rmsnorm_bwd(x, w, dy, 1e-6)
    assert dz is None
    dx0, dw0 = orc.norm_bwd(x, w, dy, 1e-6)
    _close(dx, dx0, what="plain dx"); _close(dw, dw0, what="plain dw")
    _close(orc.rmsnorm_fwd(x, w, 1e-6, 0.0, z, "silu")[0], orc.gated_norm_fwd(x, z, w, 1e-6)[0],
           what="gated y")
    for got, want, n in zip(orc.rmsnorm_bwd(x, w, dy, 1e-6, 0.0, z, "silu"),
                            orc.gated_norm_bwd(x, z, w, dy, 1e-6), ("dx", "dz", "dw")):
        _close(got, want, what="gated " + n)


def pin_general_finite_differences(orc):
    """dx, dz, dw of every (activation, offset) equal the numerical gradient of
    L = sum(y * dy)."""
    rng = np.random.default_rng(20)
    R, H, eps = 2, 6, 1e-2
    x = rng.normal(size=(R, H)); z = rng.normal(size=(R, H)) * 2.0
    w = rng.normal(size=H); dy = rng.normal(size=(R, H))
    for act in ("none", "silu", "sigmoid"):
        for off in (0.0, 1.0, 0.5):
            zz = None if act == "none" else z

            def L(x_, z_, w_):
                return float(np.sum(orc.rmsnorm_fwd(x_, w_, eps, off, z_, act)[0] * dy))

            dx, dz, dw = orc.rmsnorm_bwd(x, w, dy, eps, off, zz, act)
            tag = f"{act} offset {off}"
            _close(dx, _fd(lambda a: L(a, zz, w), x), rtol=1e-7, atol=1e-8, what=tag + " dx")
            _close(dw, _fd(lambda a: L(x, zz, a), w), rtol=1e-7, atol=1e-8, what=tag + " dw")
            if act != "none":
                _close(dz, _fd(lambda a: L(x, a, w), z), rtol=1e-7, atol=1e-8, what=tag + " dz")


def pin_autograd_gradients(orc):
    """dx, dz, dw of every (activation, offset) equal torch.autograd's gradient
    (fp64, CPU) of L = sum(y * dy) for the forward written here in torch ops
    (not the oracle's): exact up to rounding, so a bound about a million times
    tighter than the finite differences above."""
    import torch
    rng = np.random.default_rng(23)
    R, H, eps = 3, 16, 1e-3
    x = rng.normal(size=(R, H)); z = rng.normal(size=(R, H)) * 3.0
    w = rng.normal(size=H); dy = rng.normal(size=(R, H))
    for act in ("none", "silu", "sigmoid"):
        for off in (0.0, 1.0, 0.5):
            xt, zt, wt = (torch.tensor(a, dtype=torch.float64, requires_grad=True)
                          for a in (x, z, w))
            y = xt * torch.rsqrt((xt * xt).mean(dim=1, keepdim=True) + eps) * (wt + off)
            if act == "silu":
                y = y * (zt * torch.sigmoid(zt))
            elif act == "sigmoid":
                y = y * torch.sigmoid(zt)
            loss = (y * torch.tensor(dy, dtype=torch.float64)).sum()
            gx, gz, gw = torch.autograd.grad(loss, [xt, zt, wt], allow_unused=True)
            dx, dz, dw = orc.rmsnorm_bwd(x, w, dy, eps, off, None if act == "none" else z, act)
            tag = f"{act} offset {off}"
            for got, want, n in ((dx, gx, "dx"), (dw, gw, "dw")) + \
                    (((dz, gz, "dz"),) if act != "none" else ()):
                want = want.detach().numpy()
                _close(got, want, rtol=1e-11, atol=1e-13 * float(np.max(np.abs(want))),
                       what=f"{tag} {n} vs autograd")


def pin_signed_zero_weight(orc):
    """The offset is added only when it is nonzero, so with offset 0 a -0.0
    weight stays -0.0 and flips the sign of the zero it multiplies into (y and
    dz); w + 0.0 would have made it +0.0.  With offset 1, -0.0 becomes 1."""
    x = [[1.0, 2.0, -3.0, 4.0]]
    z = [[0.5, -1.0, 2.0, 1.5]]
    w = [-0.0, 0.0, -0.0, 2.0]
    dy = [[1.0, 1.0, -1.0, 1.0]]
    for act in ("none", "silu", "sigmoid"):
        zz = None if act == "none" else z
        y, _ = orc.rmsnorm_fwd(x, w, 0.0, 0.0, zz, act)
        a = np.ones(4) if act == "none" else (orc.sigmoid(np.array(z[0])) if act == "sigmoid"
                                             else orc.silu(np.array(z[0])))
        pos = np.array(x[0]) * a > 0
        assert y[0, 0] == 0 and bool(np.signbit(y[0, 0])) == bool(pos[0]), (act, y)
        assert y[0, 1] == 0 and bool(np.signbit(y[0, 1])) != bool(pos[1]), (act, y)
        assert y[0, 2] == 0 and bool(np.signbit(y[0, 2])) == bool(pos[2]), (act, y)
        if act != "none":
            _, dz, _ = orc.rmsnorm_bwd(x, w, dy, 0.0, 0.0, zz, act)
            # dz = dy*xh*w*a'(z) with a' > 0 at these z: sign of dy*x flipped by -0.0
            sdx = np.array(dy[0]) * np.array(x[0]) > 0
            assert dz[0, 0] == 0 and bool(np.signbit(dz[0, 0])) == bool(sdx[0]), (act, dz)
            assert dz[0, 2] == 0 and bool(np.signbit(dz[0, 2])) == bool(sdx[2]), (act, dz)
        y1, _ = orc.rmsnorm_fwd(x, w, 0.0, 1.0, zz, act)
        assert y1[0, 0] != 0 and y1[0, 2] != 0, (act, y1)


def pin_row_mask(orc):
    """dw over the rows a mask selects: all-ones is no mask; a loop over the
    selected rows using one-row forward outputs (dy * y / u is dy * xh * a(z));
    masked rows with non-finite values change nothing else; the mask and its
    complement add up to the whole batch; dx and dz ignore the mask."""
    rng = np.random.default_rng(21)
    R, H, eps = 11, 6, 1e-3
    x = rng.normal(size=(R, H)); z = rng.normal(size=(R, H)); dy = rng.normal(size=(R, H))
    w = rng.uniform(0.5, 1.5, size=H)
    mask = np.array([1, 0, 1, 1, 0, 0, 1, 0, 1, 1, 0], dtype=np.uint8)
    for act, off in (("none", 1.0), ("silu", 0.0), ("sigmoid", 1.0)):
        zz = None if act == "none" else z
        full = orc.rmsnorm_bwd(x, w, dy, eps, off, zz, act)
        ones = orc.rmsnorm_bwd(x, w, dy, eps, off, zz, act, row_mask=np.ones(R, np.uint8))
        _close(ones[2], full[2], rtol=0, atol=0, what=f"{act} all-ones mask dw")
        dx, dz, dw = orc.rmsnorm_bwd(x, w, dy, eps, off, zz, act, row_mask=mask)
        _close(dx, full[0], rtol=0, atol=0, what=f"{act} dx ignores the mask")
        if dz is not None:
            _close(dz, full[1], rtol=0, atol=0, what=f"{act} dz ignores the mask")
        want = np.zeros(H)
        u = w + off if off != 0 else w
        for r in range(R):
            if mask[r]:
                y, _ = orc.rmsnorm_fwd(x[r:r + 1], w, eps, off, None if zz is None else z[r:r + 1], act)
                want += dy[r] * y[0] / u
        _close(dw, want, rtol=1e-12, atol=1e-14, what=f"{act} masked dw brute force")
        _, _, dwc = orc.rmsnorm_bwd(x, w, dy, eps, off, zz, act, row_mask=1 - mask)
        _close(dw + dwc, full[2], rtol=1e-12, atol=1e-14, what=f"{act} mask + complement")
        xb = x.copy(); xb[1] = np.nan; xb[4, 2] = np.inf
        with np.errstate(all="ignore"):
            dxb, _, dwb = orc.rmsnorm_bwd(xb, w, dy, eps, off, zz, act, row_mask=mask)
        assert np.all(np.isfinite(dwb)), f"{act}: masked non-finite rows leaked into dw"
        _close(dwb, dw, rtol=0, atol=0, what=f"{act} masked non-finite rows")
        keep = [r for r in range(R) if r not in (1, 4)]
        _close(dxb[keep], dx[keep], rtol=0, atol=0, what=f"{act} other rows' dx")


def pin_round_to_format(orc):
    """fp32 -> bf16 / fp16 rounding equals torch's conversions (a library
    routine) on random values across magnitudes, and hand-checked ties."""
    import torch
    rng = np.random.default_rng(22)
    a = np.concatenate([rng.standard_normal(4000).astype(np.float32) * s
                        for s in (1e-6, 1e-3, 1.0, 300.0, 3e4)])
    # exact ties: a kept value plus half its last place
    a = np.concatenate([a, np.float32([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(2 + 2.0 ** -7),
                                       1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11])])
    t = torch.from_numpy(a)
    for fmt, dt in (("bf16", torch.bfloat16), ("f16", torch.float16)):
        got = orc.round_to_format(a, fmt)
        want = t.to(dt).double().numpy()          # fp16 overflows to inf past 65504
        assert np.array_equal(got, want), f"{fmt} rounding differs at " \
            f"{np.flatnonzero(got != want)[:5]}"
    _close(orc.round_to_format(np.float32([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8]), "bf16"),
           [1.0, 1 + 2.0 ** -6], rtol=0, atol=0, what="bf16 ties to even")
    _close(orc.round_to_format(np.float32([1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11]), "f16"),
           [1.0, 1 + 2.0 ** -9], rtol=0, atol=0, what="f16 ties to even")


def pin_residual_add_example(orc):
    """x = [1, 2, 2, 4], r = [2^-9, 0, 0, 0]: the fp32 sum 1 + 2^-9 is below half
    a bf16 place of 1, so h is x itself and y is the first worked example's
    ([2/5, 6/5, 0, 16/5] at w = [0, 1/2, -1, 1], offset 1, eps = 0); in fp32 the
    sum is kept and h differs.  r = 0 reduces to the plain forward."""
    x = [[1.0, 2.0, 2.0, 4.0]]
    r = [[2.0 ** -9, 0.0, 0.0, 0.0]]
    w = [0.0, 0.5, -1.0, 1.0]
    h, y, rho = orc.rmsnorm_add_fwd(x, r, w, 0.0, 1.0, None, "none", fmt="bf16")
    _close(h, x, rtol=0, atol=0, what="bf16 h")
    _close(y, [[0.4, 1.2, 0.0, 3.2]], what="y from the rounded h")
    _close(rho, [0.4], what="rho")
    h32, _, _ = orc.rmsnorm_add_fwd(x, r, w, 0.0, 1.0, None, "none", fmt="f32")
    _close(h32, [[1 + 2.0 ** -9, 2.0, 2.0, 4.0]], rtol=0, atol=0, what="f32 h")
    rng = np.random.default_rng(23)
    xs = rng.normal(size=(3, 8)); zs = rng.normal(size=(3, 8)); ws = rng.normal(size=8)
    h0, y0, _ = orc.rmsnorm_add_fwd(xs, np.zeros_like(xs), ws, 1e-6, 0.0, zs, "silu", fmt="f64")
    _close(h0, xs, rtol=0, atol=0, what="r = 0 keeps x")
    _close(y0, orc.gated_norm_fwd(xs, zs, ws, 1e-6)[0], what="r = 0 is the plain forward")


def pin_residual_finite_differences(orc):
    """With the sum unrounded (f64), dx equals the numerical gradient of
    L = sum(y * dy) + sum(h * dh) in x and in r (both get the same gradient)."""
    rng = np.random.default_rng(24)
    R, H, eps = 2, 6, 1e-2
    x = rng.normal(size=(R, H)); r = rng.normal(size=(R, H)); z = rng.normal(size=(R, H))
    w = rng.normal(size=H); dy = rng.normal(size=(R, H)); dh = rng.normal(size=(R, H))
    for act, off in (("none", 1.0), ("silu", 0.0), ("sigmoid", 1.0)):
        zz = None if act == "none" else z

        def L(x_, r_):
            h, y, _ = orc.rmsnorm_add_fwd(x_, r_, w, eps, off, zz, act, fmt="f64")
            return float(np.sum(y * dy) + np.sum(h * dh))

        h, _, _ = orc.rmsnorm_add_fwd(x, r, w, eps, off, zz, act, fmt="f64")
        dx, _, _ = orc.rmsnorm_add_bwd(h, w, dy, dh, eps, off, zz, act)
        _close(dx, _fd(lambda a: L(a, r), x), rtol=1e-7, atol=1e-8, what=f"{act} d/dx")
        _close(dx, _fd(lambda a: L(x, a), r), rtol=1e-7, atol=1e-8, what=f"{act} d/dr")


# --------------------------------------------------------------------------
# the cancellation scales behind the dx / dz tolerance
# --------------------------------------------------------------------------
L7 = math.log(7.0)


def pin_cancellation_scales_worked(orc):
    """The scale T of the dx / dz tolerance (|gpu - ref| <= 2 ulp + 2^-16 T),
    hand-derived on the worked examples above.
    dx: T = max(|rho*g*dy|, |rho*xh| * mean_k |g_k dy_k xh_k|).
      Zero-centred example (rho = 2/5, xh = [2,4,4,8]/5, g*dy = [1,-3/2,0,1]):
      |rho*g*dy| = [2/5, 3/5, 0, 2/5]; |g*dy*xh| = [2/5, 6/5, 0, 8/5], mean 4/5;
      |rho*xh| * 4/5 = [16, 32, 32, 64]/125  ->  T = [2/5, 3/5, 32/125, 64/125]
      (with |m| = 1/5 in place of the mean of magnitudes the last two would be
      8/125 and 2/5).
      Gated example (g = [3L/4, -L/2, 0, -3L/4], L = ln 3): |rho*g*dy| =
      [3L/10, L/5, 0, 3L/20]; |g*dy*xh| = [3L/10, 2L/5, 0, 3L/5], mean 13L/40;
      |rho*xh| * 13L/40 = [13L/250, 13L/125, 13L/125, 26L/125]
      ->  T = [3L/10, L/5, 13L/125, 26L/125].
      Sigmoid gate, offset 1 (g = [3/4, 3/8, 0, 3/2]): |rho*g*dy| =
      [3/10, 3/20, 0, 3/10]; |g*dy*xh| = [3/10, 3/10, 0, 6/5], mean 9/20;
      |rho*xh| * 9/20 = [9, 18, 18, 36]/125  ->  T = [3/10, 3/20, 18/125, 3/10].
    dz: T = |dy*xh*u*s| * max(1, |z(1-s)|) (silu), |dy*xh*u*s| (sigmoid).
      Gated example: dy*xh*w*s = [3/10, -2/5, 4, -3/5] and |z(1-s)| =
      [L/4, 3L/4, 0, L/4], all below 1  ->  T = [3/10, 2/5, 4, 3/5].
      Sigmoid, offset 1: dy*xh*u*s = [3/10, -3/10, 0, 6/5].
    A second example where the silu factor exceeds 1: H = 2, x = [3, 4],
      eps = 7/2 (rho = 1/4, xh = [3/4, 1]), z = [-ln 7, ln 3] (s = [1/8, 3/4],
      |z(1-s)| = [7 ln7/8 > 1, ln3/4 < 1]), w = [2, -1], dy = [1, -4]:
      dy*xh*w*s = [3/16, 3]  ->  dz T = [21 ln7/128, 3];
      with offset 1 (u = [3, 0]): silu T = [63 ln7/256, 0], sigmoid [9/32, 0];
      dx (gated): g*dy = [-ln7/4, 3 ln3], |rho*g*dy| = [ln7/16, 3 ln3/4];
      |g*dy*xh| = [3 ln7/16, 3 ln3], mean (3 ln7/16 + 3 ln3)/2;
      |rho*xh| * mean = [(3/32), (1/8)] * (3 ln7/16 + 3 ln3)
      ->  T = [(9/32)(ln7/16 + ln3), 3 ln3/4]."""
    L = L3
    x = [[1.0, 2.0, 2.0, 4.0]]
    w = [0.0, 0.5, -1.0, 1.0]
    dy = [[1.0, -1.0, 2.0, 0.5]]
    z = [[L, -L, 0.0, L]]
    wg = [1.0, 2.0, 5.0, -1.0]
    t_norm = [[2 / 5, 3 / 5, 32 / 125, 64 / 125]]
    _close(orc.dx_cancellation_scale(x, w, dy, 0.0), t_norm, what="dx T, zero-centred")
    _close(orc.rmsnorm_dx_scale(x, w, dy, 0.0, 1.0), t_norm, what="general dx T, offset 1")
    t_gated = [[3 * L / 10, L / 5, 13 * L / 125, 26 * L / 125]]
    _close(orc.dx_cancellation_scale(x, wg, dy, 0.0, z=z), t_gated, what="dx T, gated")
    _close(orc.rmsnorm_dx_scale(x, wg, dy, 0.0, 0.0, z, "silu"), t_gated,
           what="general dx T, silu")
    _close(orc.dz_cancellation_scale(x, z, wg, dy, 0.0), [[0.3, 0.4, 4.0, 0.6]],
           what="dz T, gated")
    _close(orc.rmsnorm_dz_scale(x, wg, dy, 0.0, 0.0, z, "silu"), [[0.3, 0.4, 4.0, 0.6]],
           what="general dz T, silu")
    _close(orc.rmsnorm_dx_scale(x, w, dy, 0.0, 1.0, z, "sigmoid"),
           [[3 / 10, 3 / 20, 18 / 125, 3 / 10]], what="general dx T, sigmoid offset 1")
    _close(orc.rmsnorm_dz_scale(x, w, dy, 0.0, 1.0, z, "sigmoid"), [[0.3, 0.3, 0.0, 1.2]],
           what="general dz T, sigmoid offset 1")
    x2, z2, w2, dy2 = [[3.0, 4.0]], [[-L7, L]], [2.0, -1.0], [[1.0, -4.0]]
    _close(orc.dz_cancellation_scale(x2, z2, w2, dy2, 3.5), [[21 * L7 / 128, 3.0]],
           what="dz T, silu factor above 1")
    _close(orc.rmsnorm_dz_scale(x2, w2, dy2, 3.5, 0.0, z2, "silu"), [[21 * L7 / 128, 3.0]],
           what="general dz T, silu factor above 1")
    _close(orc.rmsnorm_dz_scale(x2, w2, dy2, 3.5, 1.0, z2, "silu"), [[63 * L7 / 256, 0.0]],
           what="general dz T, silu offset 1")
    _close(orc.rmsnorm_dz_scale(x2, w2, dy2, 3.5, 1.0, z2, "sigmoid"), [[9 / 32, 0.0]],
           what="general dz T, sigmoid offset 1")
    t2 = [[(9 / 32) * (L7 / 16 + L), 3 * L / 4]]
    _close(orc.dx_cancellation_scale(x2, w2, dy2, 3.5, z=z2), t2, what="dx T, second example")
    _close(orc.rmsnorm_dx_scale(x2, w2, dy2, 3.5, 0.0, z2, "silu"), t2,
           what="general dx T, second example")


def _f32_backward(x, z, w, dy, eps, act, offset):
    """An fp32 evaluation of dx and dz, independent of the oracle and of the
    kernels: numpy float32 arithmetic, sums in plain ascending order (the
    order whose rounding error grows fastest), the sigmoid in its
    overflow-free form."""
    f = np.float32
    x, dy, w = x.astype(f), dy.astype(f), w.astype(f)
    R, H = x.shape
    u = (w + f(offset)).astype(f) if offset != 0 else w
    ss = np.zeros(R, f)
    for j in range(H):
        ss = (ss + x[:, j] * x[:, j]).astype(f)
    rho = (f(1) / np.sqrt((ss / f(H) + f(eps)).astype(f))).astype(f)
    xh = (x * rho[:, None]).astype(f)
    if act == "none":
        a, c, s = np.ones_like(x), None, None
    else:
        z = z.astype(f)
        e = np.exp(-np.abs(z)).astype(f)
        s = np.where(z >= 0, f(1) / (f(1) + e), e / (f(1) + e)).astype(f)
        a = (z * s).astype(f) if act == "silu" else s
        c = (f(1) + z * (f(1) - s)).astype(f) if act == "silu" else (f(1) - s).astype(f)
    gd = ((u[None, :] * a).astype(f) * dy).astype(f)
    acc = np.zeros(R, f)
    for j in range(H):
        acc = (acc + gd[:, j] * xh[:, j]).astype(f)
    m = (acc / f(H)).astype(f)
    dx = (rho[:, None] * (gd - (xh * m[:, None]).astype(f)).astype(f)).astype(f)
    dz = None if act == "none" else \
        (((((dy * xh).astype(f) * u[None, :]).astype(f) * s).astype(f) * c).astype(f))
    return dx, dz


def pin_cancellation_scales_bound_fp32_error(orc):
    """The scale is large enough: an fp32 evaluation of dx and dz (ascending
    sums; rows with 1% of channels x50 in x, z and dy, as the outlier workload
    has) stays within 2^-16 * T of the fp64 result, at widths 128 and 2048,
    for every gate: dx in every element, dz wherever the sigmoid is an fp32
    normal number (z > -87).  Below that s(z) = e^z keeps fewer than 24 bits in
    fp32, or none past z < -103; those dz are below 1e-37, where the bf16 and
    fp16 tolerances' own spacing (2^-133, 2^-24) is far larger than dz."""
    rng = np.random.default_rng(31)
    for H in (128, 2048):
        for act, off in (("none", 1.0), ("silu", 0.0), ("sigmoid", 1.0)):
            R = 16
            x, z, dy = (rng.normal(size=(R, H)) for _ in range(3))
            w = rng.normal(1.0 if off == 0.0 else 0.0, 0.3, H)
            cols = rng.choice(H, max(1, round(0.01 * H)), replace=False)
            for a in (x, z, dy):
                a[:, cols] *= 50.0
            x, z, dy, w = (a.astype(np.float32).astype(np.float64) for a in (x, z, dy, w))
            zz = None if act == "none" else z
            dx64, dz64, _ = orc.rmsnorm_bwd(x, w, dy, 1e-6, off, zz, act)
            dx32, dz32 = _f32_backward(x, z, w, dy, 1e-6, act, off)
            T = orc.rmsnorm_dx_scale(x, w, dy, 1e-6, off, zz, act)
            assert np.all(np.abs(dx32 - dx64) <= 2.0 ** -16 * T), (H, act, "dx")
            if act != "none":
                Tz = orc.rmsnorm_dz_scale(x, w, dy, 1e-6, off, z, act)
                normal = z > -87.0
                assert np.all((np.abs(dz32 - dz64) <= 2.0 ** -16 * Tz)[normal]), (H, act, "dz")
                if act == "silu" and off == 0.0:
                    assert np.array_equal(Tz, orc.dz_cancellation_scale(x, z, w, dy, 1e-6))
                    assert np.array_equal(T, orc.dx_cancellation_scale(x, w, dy, 1e-6, z=z))
            if act == "none" and off == 1.0:
                assert np.array_equal(T, orc.dx_cancellation_scale(x, w, dy, 1e-6))


# --------------------------------------------------------------------------
# the empty sum
# --------------------------------------------------------------------------
def pin_empty_and_signed_zero_sums(orc):
    """dw over no row -- a batch of no rows, or a mask selecting none -- is
    -0.0 in every column (IEEE addition's identity: the reading taken where the
    pages fix no value).  Sums that have terms follow IEEE's sign rules: a
    column whose every term is -0.0 sums to -0.0, and one +0.0 term among them
    makes +0.0 (IEEE 754, section 6.3)."""
    H = 4
    for act, off in (("none", 1.0), ("silu", 0.0), ("sigmoid", 1.0)):
        x0 = np.zeros((0, H))
        zz = None if act == "none" else x0
        _, _, dw = orc.rmsnorm_bwd(x0, np.ones(H), x0, 1e-6, off, zz, act)
        assert dw.shape == (H,) and np.all(dw == 0) and np.all(np.signbit(dw)), (act, dw)
        x = np.array([[1.0, 2.0, 0.0, 0.0], [3.0, -1.0, 0.0, 0.0], [2.0, 2.0, 0.0, 0.0]])
        dy = np.array([[1.0, 1.0, -1.0, -1.0], [2.0, -1.0, -2.0, 3.0], [1.0, 1.0, -1.0, -1.0]])
        z = np.full_like(x, 0.5)
        zz = None if act == "none" else z
        _, _, dwm = orc.rmsnorm_bwd(x, np.ones(H), dy, 1e-6, off, zz, act,
                                    row_mask=np.zeros(3, np.uint8))
        assert np.all(dwm == 0) and np.all(np.signbit(dwm)), (act, dwm)
        # column 2: x = +0 and dy < 0 in every row: every term is -0.0;
        # column 3: one row has dy > 0, a +0.0 term among -0.0 terms
        _, _, dws = orc.rmsnorm_bwd(x, np.ones(H), dy, 1e-6, off, zz, act)
        assert dws[2] == 0 and np.signbit(dws[2]), (act, dws)
        assert dws[3] == 0 and not np.signbit(dws[3]), (act, dws)
    _, dw = orc.norm_bwd(np.zeros((0, H)), np.ones(H), np.zeros((0, H)), 1e-6)
    assert np.all(np.signbit(dw)) and np.all(dw == 0), dw
    _, _, dw = orc.gated_norm_bwd(np.zeros((0, H)), np.zeros((0, H)), np.ones(H),
                                  np.zeros((0, H)), 1e-6)
    assert np.all(np.signbit(dw)) and np.all(dw == 0), dw


ALL_PINS = [
    pin_worked_example_norm,
    pin_worked_example_eps,
    pin_worked_example_gated,
    pin_sigmoid_points,
    pin_constant_row,
    pin_unit_rms,
    pin_eps_shrinks_rms,
    pin_scale_invariance,
    pin_scale_identity,
    pin_finite_differences,
    pin_dw_brute_force,
    pin_rows_independent,
    pin_worked_example_sigmoid_offset,
    pin_general_special_cases,
    pin_general_finite_differences,
    pin_autograd_gradients,
    pin_signed_zero_weight,
    pin_row_mask,
    pin_round_to_format,
    pin_residual_add_example,
    pin_residual_finite_differences,
    pin_cancellation_scales_worked,
    pin_cancellation_scales_bound_fp32_error,
    pin_empty_and_signed_zero_sums,
]


def failing_pins(orc):
    """Names of the pins that ``orc`` fails (an exception counts as a failure)."""
    bad = []
    for p in ALL_PINS:
        try:
            with np.errstate(all="ignore"):
                p(orc)
        except Exception:  # noqa: BLE001 - any failure of a mutant counts
            bad.append(p.__name__)
    return bad
