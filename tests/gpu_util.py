"""Shared helpers of the GPU tests: run the library on a workload and compare
with the fp64 oracle."""
from __future__ import annotations

import json
import os

import numpy as np
import torch

import oracle
from numerics import check_out
from rollout_parity_b200 import workloads

f64 = workloads.as_f64


def is_general(wl) -> bool:
    """True for op "general": its activation and offset are given explicitly,
    so it runs through rmsnorm_fwd / rmsnorm_bwd."""
    return wl.op == "general"


def run(rn, wl, rstd_in_bwd=True):
    """Forward then backward through the C ABI; returns a dict of outputs.
    op "norm" / "gated" use their own entry points, op "general" rmsnorm_fwd /
    rmsnorm_bwd."""
    if is_general(wl):
        y, rstd = rn.rmsnorm_fwd(wl.x, wl.w, wl.eps, wl.weight_offset, wl.z, wl.act)
        dx, dz, dw = rn.rmsnorm_bwd(wl.x, wl.w, wl.dy, rstd if rstd_in_bwd else None, wl.eps,
                                    wl.weight_offset, wl.z, wl.act)
    elif wl.gated:
        y, rstd = rn.gated_norm_fwd(wl.x, wl.z, wl.w, wl.eps)
        dx, dz, dw = rn.gated_norm_bwd(wl.x, wl.z, wl.w, wl.dy, rstd if rstd_in_bwd else None,
                                       wl.eps)
    else:
        y, rstd = rn.norm_fwd(wl.x, wl.w, wl.eps)
        dx, dw = rn.norm_bwd(wl.x, wl.w, wl.dy, rstd if rstd_in_bwd else None, wl.eps)
        dz = None
    return dict(y=y, rstd=rstd, dx=dx, dz=dz, dw=dw)


def oracle_rows(wl, idx=None):
    """fp64 oracle outputs (y, rstd, dx, dz and cancellation scales) for the
    rows ``idx`` (all rows when None)."""
    sel = (lambda t: f64(t)) if idx is None else (lambda t: f64(t[idx]))
    x, dy = sel(wl.x), sel(wl.dy)
    w = f64(wl.w)
    if is_general(wl):
        z = None if wl.z is None else sel(wl.z)
        o, a = wl.weight_offset, wl.act
        y, r = oracle.rmsnorm_fwd(x, w, wl.eps, o, z, a)
        dx, dz, _ = oracle.rmsnorm_bwd(x, w, dy, wl.eps, o, z, a)
        sdx = oracle.rmsnorm_dx_scale(x, w, dy, wl.eps, o, z, a)
        sdz = None if z is None else oracle.rmsnorm_dz_scale(x, w, dy, wl.eps, o, z, a)
    elif wl.gated:
        z = sel(wl.z)
        y, r = oracle.gated_norm_fwd(x, z, w, wl.eps)
        dx, dz, _ = oracle.gated_norm_bwd(x, z, w, dy, wl.eps)
        sdx = oracle.dx_cancellation_scale(x, w, dy, wl.eps, z=z)
        sdz = oracle.dz_cancellation_scale(x, z, w, dy, wl.eps)
    else:
        y, r = oracle.norm_fwd(x, w, wl.eps)
        dx, _ = oracle.norm_bwd(x, w, dy, wl.eps)
        dz, sdz = None, None
        sdx = oracle.dx_cancellation_scale(x, w, dy, wl.eps)
    return dict(y=y, rstd=r, dx=dx, dz=dz, sdx=sdx, sdz=sdz)


def oracle_dw(wl, chunk=4096):
    """fp64 dw over all rows, summed chunk by chunk to bound host memory."""
    w = f64(wl.w)
    tot = np.zeros(wl.width)
    for s in range(0, wl.rows, chunk):
        e = min(wl.rows, s + chunk)
        x, dy = f64(wl.x[s:e]), f64(wl.dy[s:e])
        if is_general(wl):
            z = None if wl.z is None else f64(wl.z[s:e])
            _, _, dw = oracle.rmsnorm_bwd(x, w, dy, wl.eps, wl.weight_offset, z, wl.act)
        elif wl.gated:
            _, _, dw = oracle.gated_norm_bwd(x, f64(wl.z[s:e]), w, dy, wl.eps)
        else:
            _, dw = oracle.norm_bwd(x, w, dy, wl.eps)
        tot += dw
    return tot


def record(wl, stats, idx=None):
    """Appends one JSON line of parity statistics to the file named by the
    RN_ACCURACY_RECORD environment variable, when it is set (the accuracy
    record kept beside the profiles); a no-op otherwise."""
    path = os.environ.get("RN_ACCURACY_RECORD")
    if not path:
        return
    line = {"test": os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0],
            "workload": wl.name, "rows": wl.rows, "width": wl.width, "dtype": wl.dtype,
            "act": wl.act, "weight_offset": wl.weight_offset,
            "rows_checked": wl.rows if idx is None else int(len(idx)), "stats": stats}
    with open(path, "a") as f:
        f.write(json.dumps(line) + "\n")


def compare(out, wl, idx=None, with_dw=True):
    """Assert the parity tolerances; return statistics (and record them, see
    record())."""
    ref = oracle_rows(wl, idx)
    g = (lambda k: out[k]) if idx is None else (lambda k: out[k][idx.to(out[k].device)
                                                                 if torch.is_tensor(idx) else idx])
    stats = {}
    stats["y"] = check_out(g("y"), ref["y"], what="y")
    stats["rstd"] = check_out(g("rstd"), ref["rstd"], what="rstd")
    stats["dx"] = check_out(g("dx"), ref["dx"], scale=ref["sdx"], what="dx")
    if wl.gated:
        stats["dz"] = check_out(g("dz"), ref["dz"], scale=ref["sdz"], what="dz")
    if with_dw:
        stats["dw"] = check_out(out["dw"], oracle_dw(wl), what="dw")
    record(wl, stats, idx)
    return stats


def sample_rows(rows, n=2048, seed=0):
    rng = np.random.default_rng(seed)
    idx = set(rng.choice(rows, size=min(n, rows), replace=False).tolist())
    idx.update([0, rows - 1, min(rows - 1, 31), min(rows - 1, 32)])
    return torch.tensor(sorted(idx), dtype=torch.long)
