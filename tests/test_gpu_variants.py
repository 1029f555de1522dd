"""The operator's variants on the GPU through rmsnorm_fwd / rmsnorm_bwd:
gate activation (none, silu, sigmoid), weight offset, and element format
(fp32, fp16, bf16), element by element against the fp64 oracle.

The matrix is the one RL-Kernel PR #468 ("[WS1][CUDA][Qwen3-Next] Gated RMSNorm
CUDA kernel for the GDN block", Summary, "rstd" bullet) spans with its rstd
identity test: {fp32, fp16, bf16} x H {128, 2048, 5120} x {silu, sigmoid} x
offset {0, 1}, 36 cases; H = 128 and 5120 take different team shapes (4 and 512
threads a row here) and 5120 leaves a ragged last vector slot.  The signed-zero
rule is that page's "Changes to existing code, in detail", "Signed zero" bullet.
Tolerances as in test_gpu_parity.py (tests/numerics.py), fp16 in fp16 ulps.
"""
import dataclasses

import pytest
import torch

import oracle
from gpu_util import compare, run, sample_rows
from numerics import to64
from rollout_parity_b200 import workloads

pytestmark = pytest.mark.gpu
DEV = "cuda:0"

MATRIX = [(dt, h, act, off) for dt in ("f32", "f16", "bf16") for h in (128, 2048, 5120)
          for act in ("silu", "sigmoid") for off in (0.0, 1.0)]
IDS = [f"{dt}-H{h}-{act}-off{int(off)}" for dt, h, act, off in MATRIX]


def general(rows, width, dtype, act, off, seed, **kw):
    # offset 0 multiplies by w itself: centre w at 1 so the gain is not ~0
    return workloads.make("general", rows, width, dtype, seed=seed, act=act, weight_offset=off,
                          w_mean=1.0 if off == 0.0 else 0.0, **kw).to(DEV)


def bits(t):
    return t.view(torch.int32 if t.dtype == torch.float32 else torch.int16)


def sub(wl, s, e):
    """The rows [s, e) as a workload of their own (fresh contiguous copies)."""
    c = lambda t: None if t is None else t[s:e].clone()
    return dataclasses.replace(wl, rows=e - s, x=c(wl.x), z=c(wl.z), dy=c(wl.dy))


@pytest.mark.parametrize("dtype,width,act,off", MATRIX, ids=IDS)
def test_variant_parity(cuda_lib, dtype, width, act, off):
    rows = 300 if width == 128 else 67      # several leaves and tiles, ragged tail
    wl = general(rows, width, dtype, act, off, seed=width + rows)
    compare(run(cuda_lib, wl), wl)


@pytest.mark.parametrize("dtype,width,act,off", MATRIX, ids=IDS)
def test_rstd_is_bitwise_the_plain_rstd(cuda_lib, dtype, width, act, off):
    wl = general(97, width, dtype, act, off, seed=width)
    _, r_plain = cuda_lib.norm_fwd(wl.x, wl.w, wl.eps)
    _, r = cuda_lib.rmsnorm_fwd(wl.x, wl.w, wl.eps, off, wl.z, act)
    assert torch.equal(bits(r), bits(r_plain))


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("off", [0.0, 1.0, 0.5, -1.0])
def test_no_gate_any_offset(cuda_lib, dtype, off):
    wl = general(300, 136, dtype, "none", off, seed=11)
    compare(run(cuda_lib, wl), wl)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("act", ["none", "silu", "sigmoid"])
def test_general_entry_recomputed_rstd_gives_identical_bits(cuda_lib, dtype, act):
    wl = general(200, 2048, dtype, act, 1.0, seed=5)
    a = run(cuda_lib, wl, rstd_in_bwd=True)
    b = run(cuda_lib, wl, rstd_in_bwd=False)
    for k in ("dx", "dz", "dw"):
        if a[k] is not None:
            assert torch.equal(bits(a[k]), bits(b[k])), k


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_general_matches_named_entries_bitwise(cuda_lib, dtype):
    # offset 1 without a gate is norm_*; offset 0 with silu is gated_norm_*
    for op, act, off in (("norm", "none", 1.0), ("gated", "silu", 0.0)):
        named = workloads.make(op, 333, 2048, dtype, seed=9).to(DEV)
        gen = workloads.make("general", 333, 2048, dtype, seed=9, act=act,
                             weight_offset=off).to(DEV)
        a, b = run(cuda_lib, named), run(cuda_lib, gen)
        for k in ("y", "rstd", "dx", "dz", "dw"):
            if a[k] is not None:
                assert torch.equal(bits(a[k]), bits(b[k])), (op, k)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("act", ["none", "silu", "sigmoid"])
def test_signed_zero_weight(cuda_lib, dtype, act):
    # columns whose weight is -0.0 or +0.0: with offset 0 the zero products in
    # y and dz carry the sign the oracle gives them (the weight's own zero);
    # with offset 1 those columns are ordinary
    wl = general(64, 128, dtype, act, 0.0, seed=13)
    w = wl.w.clone()
    neg, pos = torch.arange(0, 128, 7), torch.arange(3, 128, 11)
    w[neg] = -0.0
    w[pos] = 0.0
    wl.w.copy_(w)
    out = run(cuda_lib, wl)
    x, dy = workloads.as_f64(wl.x), workloads.as_f64(wl.dy)
    z = None if wl.z is None else workloads.as_f64(wl.z)
    wf = workloads.as_f64(wl.w)
    y_ref, _ = oracle.rmsnorm_fwd(x, wf, wl.eps, 0.0, z, act)
    _, dz_ref, _ = oracle.rmsnorm_bwd(x, wf, dy, wl.eps, 0.0, z, act)
    cols = torch.cat([neg, pos])
    for name, got, ref in (("y", out["y"], y_ref), ("dz", out["dz"], dz_ref)):
        if got is None:
            continue
        g = to64(got)[:, cols.numpy()]
        r = ref[:, cols.numpy()]
        assert (g == 0).all() and (r == 0).all(), name
        assert (torch.signbit(torch.from_numpy(g)) == torch.signbit(torch.from_numpy(r))).all(), name
    y1, _ = cuda_lib.rmsnorm_fwd(wl.x, wl.w, wl.eps, 1.0, wl.z, act)
    assert (y1[:, cols.to(DEV)] != 0).float().mean() > 0.99


@pytest.mark.parametrize("dtype,width,act", [("f16", 128, "sigmoid"), ("bf16", 5120, "sigmoid"),
                                             ("f32", 2048, "silu"), ("f16", 5120, "none")])
def test_variant_prefix_slices_and_geometry(cuda_lib, dtype, width, act):
    rows = 512 if width == 128 else 96
    wl = general(rows, width, dtype, act, 1.0, seed=21)
    full = run(cuda_lib, wl)
    for b in (1, 2, 33, rows // 2, rows):
        got = run(cuda_lib, sub(wl, 0, b))
        for k in ("y", "rstd", "dx", "dz"):
            if full[k] is not None:
                assert torch.equal(bits(full[k][:b]), bits(got[k])), (k, b)
    try:
        for geo in ((1, 1, 8), (3, 2, 16), (0, 1, 0)):
            cuda_lib.rn_test_set_geometry(*geo)
            again = run(cuda_lib, wl)
            for k in ("y", "rstd", "dx", "dz", "dw"):
                if full[k] is not None:
                    assert torch.equal(bits(full[k]), bits(again[k])), (k, geo)
    finally:
        cuda_lib.rn_test_set_geometry(0, 0, 0)


@pytest.mark.parametrize("op", ["norm", "gated"])
def test_fp16_named_entries(cuda_lib, op):
    for rows, width in ((1000, 128), (77, 24), (257, 1032), (17, 16384)):
        wl = workloads.make(op, rows, width, "f16", seed=rows,
                            w_mean=1.0 if op == "gated" else 0.0).to(DEV)
        compare(run(cuda_lib, wl), wl)


@pytest.mark.slow
@pytest.mark.parametrize("name", sorted(workloads.VARIANTS))
def test_variant_configs_full_size(cuda_lib, name):
    # the benchmark's variant workloads at full size: sampled rows element by
    # element, dw over every row
    wl = workloads.VARIANTS[name]().to(DEV)
    out = run(cuda_lib, wl)
    compare(out, wl, idx=sample_rows(wl.rows, n=1024))


@pytest.mark.parametrize("act,off", [(None, 1.0), ("sigmoid", 0.0), ("swish", 1.0)])
def test_autograd_wrapper_routes_gradients(cuda_lib, act, off):
    from rollout_parity_b200 import autograd
    a = {None: "none", "swish": "silu"}.get(act, act)
    wl = general(96, 256, "bf16", a, off, seed=31)
    x = wl.x.clone().requires_grad_(True)
    w = wl.w.clone().requires_grad_(True)
    z = None if wl.z is None else wl.z.clone().requires_grad_(True)
    y = autograd.rms_norm(x, w, z, wl.eps, off, act)
    y.backward(wl.dy)
    want = run(cuda_lib, wl)
    assert torch.equal(bits(y.detach()), bits(want["y"]))
    assert torch.equal(bits(x.grad), bits(want["dx"]))
    assert torch.equal(bits(w.grad), bits(want["dw"]))
    if z is not None:
        assert torch.equal(bits(z.grad), bits(want["dz"]))
