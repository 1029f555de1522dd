"""Residual-add RMSNorm on the GPU (rmsnorm_add_fwd / rmsnorm_add_bwd).

RL-Kernel PR #468 (Notes) mentions a norm variant that also adds a residual
and defines nothing more about it; the reading is the usual fused form: h = x + r, formed in
fp32 and rounded once to the tensors' format, stored and normalised; the
backward gives x and r the norm's gradient at h plus dh.  h is a rounding
decision both sides take in fp32, so it is compared bit for bit; the rest
against the oracle's tolerances; and the fused calls must give exactly the
bits of the unfused calls on the stored h."""
import pytest
import torch

import oracle
from numerics import check_out
from rollout_parity_b200 import workloads

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
f64 = workloads.as_f64

CASES = [("silu", 0.0, 1000, 128, "bf16"), ("none", 1.0, 300, 2048, "f32"),
         ("sigmoid", 1.0, 129, 5120, "f16"), ("silu", 0.0, 257, 136, "bf16"),
         ("none", 1.0, 777, 256, "bf16")]
IDS = [f"{a}-off{int(o)}-{r}x{w}-{d}" for a, o, r, w, d in CASES]


def inputs(act, off, rows, width, dtype, seed):
    wl = workloads.make("general", rows, width, dtype, seed=seed, act=act, weight_offset=off,
                        w_mean=1.0 if off == 0.0 else 0.0).to(DEV)
    g = torch.Generator().manual_seed(seed)
    r = (torch.randn(rows, width, generator=g) * 3.0).to(wl.x.dtype).to(DEV)
    dh = torch.randn(rows, width, generator=g).to(wl.x.dtype).to(DEV)
    return wl, r, dh


def bits(t):
    return t.view(torch.int32 if t.dtype == torch.float32 else torch.int16)


@pytest.mark.parametrize("act,off,rows,width,dtype", CASES, ids=IDS)
def test_residual_forward_and_backward(cuda_lib, act, off, rows, width, dtype):
    wl, r, dh = inputs(act, off, rows, width, dtype, seed=rows)
    h, y, rstd = cuda_lib.rmsnorm_add_fwd(wl.x, r, wl.w, wl.eps, off, wl.z, act)
    dx, dz, dw = cuda_lib.rmsnorm_add_bwd(h, wl.w, wl.dy, dh, rstd, wl.eps, off, wl.z, act)
    z64 = None if wl.z is None else f64(wl.z)
    h_ref, y_ref, r_ref = oracle.rmsnorm_add_fwd(f64(wl.x), f64(r), f64(wl.w), wl.eps, off, z64,
                                                 act, fmt=dtype)
    assert torch.equal(h.cpu().double(), torch.from_numpy(h_ref)), "h differs from fmt(x + r)"
    check_out(y, y_ref, what="y")
    check_out(rstd, r_ref, what="rstd")
    dx_ref, dz_ref, dw_ref = oracle.rmsnorm_add_bwd(h_ref, f64(wl.w), f64(wl.dy), f64(dh),
                                                    wl.eps, off, z64, act)
    scale = oracle.rmsnorm_dx_scale(h_ref, f64(wl.w), f64(wl.dy), wl.eps, off, z64, act)
    check_out(dx, dx_ref, scale=scale + abs(f64(dh)), what="dx")
    if dz is not None:
        check_out(dz, dz_ref, scale=oracle.rmsnorm_dz_scale(h_ref, f64(wl.w), f64(wl.dy), wl.eps,
                                                            off, z64, act), what="dz")
    check_out(dw, dw_ref, what="dw")


@pytest.mark.parametrize("act,off,rows,width,dtype", CASES, ids=IDS)
def test_fused_equals_unfused_on_the_stored_h(cuda_lib, act, off, rows, width, dtype):
    wl, r, dh = inputs(act, off, rows, width, dtype, seed=rows + 1)
    h, y, rstd = cuda_lib.rmsnorm_add_fwd(wl.x, r, wl.w, wl.eps, off, wl.z, act)
    y2, rstd2 = cuda_lib.rmsnorm_fwd(h, wl.w, wl.eps, off, wl.z, act)
    assert torch.equal(bits(y), bits(y2)) and torch.equal(bits(rstd), bits(rstd2))
    # without dh the residual backward is rmsnorm_bwd on h
    a = cuda_lib.rmsnorm_add_bwd(h, wl.w, wl.dy, None, rstd, wl.eps, off, wl.z, act)
    b = cuda_lib.rmsnorm_bwd(h, wl.w, wl.dy, rstd, wl.eps, off, wl.z, act)
    for u, v in zip(a, b):
        if u is not None:
            assert torch.equal(bits(u), bits(v))


@pytest.mark.parametrize("act,off,rows,width,dtype", CASES[:3], ids=IDS[:3])
def test_in_place_updates(cuda_lib, act, off, rows, width, dtype):
    wl, r, dh = inputs(act, off, rows, width, dtype, seed=rows + 2)
    h, y, rstd = cuda_lib.rmsnorm_add_fwd(wl.x, r, wl.w, wl.eps, off, wl.z, act)
    r2 = r.clone()
    _, y2, _ = cuda_lib.rmsnorm_add_fwd(wl.x, r2, wl.w, wl.eps, off, wl.z, act, h=r2)   # h is r
    assert torch.equal(bits(r2), bits(h)) and torch.equal(bits(y2), bits(y))
    x2 = wl.x.clone()
    cuda_lib.rmsnorm_add_fwd(x2, r, wl.w, wl.eps, off, wl.z, act, h=x2)                  # h is x
    assert torch.equal(bits(x2), bits(h))
    dx, _, dw = cuda_lib.rmsnorm_add_bwd(h, wl.w, wl.dy, dh, rstd, wl.eps, off, wl.z, act)
    dh2 = dh.clone()
    dx2, _, dw2 = cuda_lib.rmsnorm_add_bwd(h, wl.w, wl.dy, dh2, rstd, wl.eps, off, wl.z, act,
                                           dx=dh2)                                       # dx is dh
    assert torch.equal(bits(dh2), bits(dx)) and torch.equal(bits(dw2), bits(dw))
