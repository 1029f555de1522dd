"""Bitwise invariance on the GPU (via the C ABI).

The contract (RL-Kernel RFC #415, section 4 "Numerical contract", points 2, 3
and 6): a row's outputs do not depend on the other rows, its position, the
batch size, packing, padding or launch geometry; dw does not depend on the
launch geometry and is reproducible.  The reuse checks of PR #468 ("Prior art
& reuse decision": every row alone vs in full batches, sub-batches covering
every row, a batch-size sweep; and its prefix-slice and dweight batch tests in
"Summary") are the model; the sub-batch sweep visits every start position
(the review finding on the stride at sub-batch size 1).
"""
import dataclasses

import numpy as np
import pytest
import torch

import fold_model
from gpu_util import run
from rollout_parity_b200 import workloads

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
ROW_KEYS = ("y", "rstd", "dx", "dz")


def sub(wl, s, e):
    """The rows [s, e) as a workload of their own (fresh contiguous copies)."""
    c = lambda t: None if t is None else t[s:e].clone()
    return dataclasses.replace(wl, rows=e - s, x=c(wl.x), z=c(wl.z), dy=c(wl.dy),
                               seq_lens=None)


def bits(t):
    return t.view(torch.int32 if t.dtype == torch.float32 else torch.int16)


def assert_rows_equal(full, part, s, e, what=""):
    for k in ROW_KEYS:
        if full[k] is None:
            continue
        assert torch.equal(bits(full[k][s:e]), bits(part[k])), f"{what}: {k} rows [{s},{e}) differ"


@pytest.fixture(autouse=True)
def default_geometry(cuda_lib):
    cuda_lib.rn_test_set_geometry(0, 0, 0)
    yield
    cuda_lib.rn_test_set_geometry(0, 0, 0)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("width", [8, 128, 136, 2048, 5120, 8192, 16384])
@pytest.mark.parametrize("eps", [1e-6, 0.0, 0.5])
def test_gated_rstd_is_bitwise_the_plain_rstd(cuda_lib, dtype, width, eps):
    rows = 97
    wl = workloads.make("gated", rows, width, dtype, seed=width).to(DEV)
    _, r_plain = cuda_lib.norm_fwd(wl.x, wl.w, eps)
    _, r_gated = cuda_lib.gated_norm_fwd(wl.x, wl.z, wl.w, eps)
    assert torch.equal(r_plain.view(torch.int32), r_gated.view(torch.int32))


@pytest.mark.parametrize("op", ["norm", "gated"])
def test_prefix_slices(cuda_lib, op):
    # prefixes {1, 2, 8, 16, 32, 48, 64, 512} of 512 rows, bf16, width 128
    wl = workloads.make(op, 512, 128, "bf16", seed=1).to(DEV)
    full = run(cuda_lib, wl)
    for b in (1, 2, 8, 16, 32, 48, 64, 512):
        assert_rows_equal(full, run(cuda_lib, sub(wl, 0, b)), 0, b, f"prefix {b}")


@pytest.mark.parametrize("op,width", [("gated", 128), ("norm", 2048)])
def test_every_row_alone(cuda_lib, op, width):
    rows = 1024 if width == 128 else 256
    wl = workloads.make(op, rows, width, "bf16", seed=2).to(DEV)
    full = run(cuda_lib, wl)
    for r in range(rows):
        assert_rows_equal(full, run(cuda_lib, sub(wl, r, r + 1)), r, r + 1, f"row {r} alone")


@pytest.mark.parametrize("sb", [1, 7, 128, 4096])
def test_sub_batches_at_every_start(cuda_lib, sb):
    # sub-batches of size sb tiling the batch, starting at every offset mod sb
    wl = workloads.make("gated", 4096, 128, "bf16", seed=3).to(DEV)
    full = run(cuda_lib, wl)
    shifts = range(sb) if sb <= 7 else (0, 1, sb // 2, sb - 1)
    for shift in shifts:
        starts = [0] + list(range(shift, wl.rows, sb)) if shift else list(range(0, wl.rows, sb))
        starts = sorted(set(starts))
        bounds = starts + [wl.rows]
        for s, e in zip(bounds[:-1], bounds[1:]):
            if e > s:
                assert_rows_equal(full, run(cuda_lib, sub(wl, s, e)), s, e, f"sb {sb} shift {shift}")


def test_permutation(cuda_lib):
    wl = workloads.make("gated", 3000, 128, "bf16", seed=4).to(DEV)
    full = run(cuda_lib, wl)
    perm = torch.randperm(wl.rows, generator=torch.Generator().manual_seed(0)).to(DEV)
    p = lambda t: None if t is None else t[perm].contiguous()
    wp = workloads.Workload(name="perm", op=wl.op, rows=wl.rows, width=wl.width, dtype=wl.dtype,
                            eps=wl.eps, x=p(wl.x), z=p(wl.z), dy=p(wl.dy), w=wl.w)
    out = run(cuda_lib, wp)
    inv = torch.argsort(perm)
    for k in ROW_KEYS:
        assert torch.equal(bits(out[k][inv]), bits(full[k])), k


def test_padding_rows_mutated(cuda_lib):
    # the same 500 rows inside a larger batch whose other rows change between runs
    base = workloads.make("gated", 500, 128, "bf16", seed=5).to(DEV)
    ref = run(cuda_lib, base)
    for seed, (before, after) in enumerate([(3, 0), (0, 45), (37, 11), (256, 300)]):
        pad = workloads.make("gated", before + after, 128, "bf16", seed=100 + seed).to(DEV)
        cat = lambda a, b: None if a is None else torch.cat([b[:before], a, b[before:]]).contiguous()
        wl = workloads.Workload(name="pad", op="gated", rows=500 + before + after, width=128,
                                dtype="bf16", eps=base.eps, x=cat(base.x, pad.x),
                                z=cat(base.z, pad.z), dy=cat(base.dy, pad.dy), w=base.w)
        out = run(cuda_lib, wl)
        for k in ROW_KEYS:
            assert torch.equal(bits(out[k][before:before + 500]), bits(ref[k])), (k, before, after)


@pytest.mark.slow
def test_packed_sequences_alone_and_shifted(cuda_lib):
    wl = workloads.cfg_packed_2048().to(DEV)
    full = run(cuda_lib, wl)
    starts = np.concatenate([[0], np.cumsum(wl.seq_lens)[:-1]])
    rng = np.random.default_rng(0)
    pick = sorted(set(rng.choice(len(starts), size=min(40, len(starts)), replace=False)) |
                  {0, len(starts) - 1})
    for i in pick:
        s, n = int(starts[i]), int(wl.seq_lens[i])
        assert_rows_equal(full, run(cuda_lib, sub(wl, s, s + n)), s, s + n, f"seq {i} alone")
        # the same sequence at a shifted row offset inside other data
        off = int(rng.integers(1, 97))
        pad = workloads.make("norm", off + 5, 2048, "bf16", seed=int(i) + 7).to(DEV)
        cat = lambda a, b: torch.cat([b[:off], a[s:s + n], b[off:]]).contiguous()
        moved = workloads.Workload(name="moved", op="norm", rows=n + off + 5, width=2048,
                                   dtype="bf16", eps=wl.eps, x=cat(wl.x, pad.x), z=None,
                                   dy=cat(wl.dy, pad.dy), w=wl.w)
        out = run(cuda_lib, moved)
        for k in ("y", "rstd", "dx"):
            assert torch.equal(bits(out[k][off:off + n]), bits(full[k][s:s + n])), (k, i)


@pytest.mark.slow
def test_gated_heads_sub_batches(cuda_lib):
    # the full 262144-row batch vs sub-batches covering every row, three sizes
    wl = workloads.cfg_gated_heads().to(DEV)
    full = run(cuda_lib, wl)
    for sb in (4099, 32768, 100000):
        for s in range(0, wl.rows, sb):
            e = min(wl.rows, s + sb)
            assert_rows_equal(full, run(cuda_lib, sub(wl, s, e)), s, e, f"sb {sb}")
    # and a sample of rows alone
    for r in np.random.default_rng(1).choice(wl.rows, 256, replace=False):
        r = int(r)
        assert_rows_equal(full, run(cuda_lib, sub(wl, r, r + 1)), r, r + 1, f"row {r}")


@pytest.mark.parametrize("op,rows,width", [("gated", 4096, 128), ("norm", 16384, 128),
                                           ("gated", 1000, 2048), ("norm", 300, 8192),
                                           ("gated", 70, 5120)])
def test_dw_repeatable_across_geometry(cuda_lib, op, rows, width):
    wl = workloads.make(op, rows, width, "bf16", seed=6).to(DEV)
    ref = run(cuda_lib, wl)
    for _ in range(10):
        assert torch.equal(bits(run(cuda_lib, wl)["dw"]), bits(ref["dw"]))
    for max_ctas in (1, 7, 148, 1024, 0):
        for lpc in (1, 2, 8, 0):
            for fold_rows in (8, 64, 256, 0):
                cuda_lib.rn_test_set_geometry(max_ctas, lpc, fold_rows)
                out = run(cuda_lib, wl)
                for k in ("dw",) + ROW_KEYS:
                    if ref[k] is not None:
                        assert torch.equal(bits(out[k]), bits(ref[k])), (k, max_ctas, lpc, fold_rows)
    cuda_lib.rn_test_set_geometry(0, 0, 0)


def test_row_outputs_across_geometry(cuda_lib):
    wl = workloads.make("gated", 2000, 128, "bf16", seed=7).to(DEV)
    ref = run(cuda_lib, wl)
    for max_ctas in (1, 3, 148):
        for lpc in (1, 2, 8):
            cuda_lib.rn_test_set_geometry(max_ctas, lpc, 0)
            out = run(cuda_lib, wl)
            for k in ROW_KEYS:
                assert torch.equal(bits(out[k]), bits(ref[k])), (k, max_ctas, lpc)


@pytest.mark.parametrize("op,width,dtype", [("gated", 128, "bf16"), ("norm", 128, "bf16"),
                                            ("gated", 2048, "bf16"), ("norm", 128, "f32"),
                                            ("norm", 8192, "bf16")])
@pytest.mark.parametrize("rows", [1, 7, 31, 32, 33, 255, 256, 257, 4096, 16384])
def test_dw_equals_the_declared_tree_over_single_row_dws(cuda_lib, op, width, dtype, rows):
    if width * rows > 16384 * 128 and rows > 300:
        pytest.skip("kept to the sizes the one-row loop runs in seconds")
    wl = workloads.make(op, rows, width, dtype, seed=rows).to(DEV)
    batch_dw = run(cuda_lib, wl)["dw"].cpu().numpy()
    one = np.stack([run(cuda_lib, sub(wl, r, r + 1))["dw"].cpu().numpy() for r in range(rows)])
    model = fold_model.dw_tree(one)
    assert np.array_equal(batch_dw.view(np.uint32), model.view(np.uint32))


def test_gated_sign_symmetry_and_negative_zero_weight(cuda_lib):
    # every gated output is a product with w (dx through the dot, which negates
    # exactly), so w -> -w flips the sign bit of y, dx, dz and leaves dw alone;
    # with w_j = -0.0 column j of y and dz is zero with the flipped sign
    wl = workloads.make("gated", 333, 128, "bf16", seed=8).to(DEV)
    w = wl.w.clone()
    w[5] = 0.0
    w[77] = 0.0
    a = run(cuda_lib, workloads.Workload(**{**wl.__dict__, "w": w}))
    b = run(cuda_lib, workloads.Workload(**{**wl.__dict__, "w": -w}))
    for k in ("y", "dx", "dz"):
        assert torch.equal(a[k].view(torch.int16) ^ torch.tensor(-32768, dtype=torch.int16, device=DEV),
                           b[k].view(torch.int16)), k
    assert torch.equal(bits(a["dw"]), bits(b["dw"]))
    assert torch.equal(bits(a["rstd"]), bits(b["rstd"]))
    for j in (5, 77):
        assert torch.all(b["y"][:, j] == 0) and torch.all(b["dz"][:, j] == 0)
        assert torch.equal(torch.signbit(b["y"][:, j].float()), ~torch.signbit(a["y"][:, j].float()))


def test_norm_input_sign_symmetry(cuda_lib):
    # x -> -x: y and dw flip sign exactly, rstd and dx are unchanged
    wl = workloads.make("norm", 333, 2048, "bf16", seed=9, w_mean=0.0).to(DEV)
    a = run(cuda_lib, wl)
    b = run(cuda_lib, workloads.Workload(**{**wl.__dict__, "x": -wl.x}))
    assert torch.equal(bits(b["y"]), bits(-a["y"])) and torch.equal(bits(b["dw"]), bits(-a["dw"]))
    assert torch.equal(bits(b["rstd"]), bits(a["rstd"])) and torch.equal(bits(b["dx"]), bits(a["dx"]))


def _alone_and_shifted(cuda_lib, wl, full, rows, seed, keys):
    """Each row in ``rows`` computed alone, and inside other data at a shifted
    row offset, gives the bits it has in ``full``."""
    rng = np.random.default_rng(seed)
    for r in rows:
        r = int(r)
        one = run(cuda_lib, sub(wl, r, r + 1))
        for k in keys:
            assert torch.equal(bits(one[k]), bits(full[k][r:r + 1])), (k, r, "alone")
        before, after = int(rng.integers(1, 40)), int(rng.integers(0, 9))
        pad = workloads.make(wl.op, before + after, wl.width, wl.dtype, seed=r + 11,
                             act=wl.act if wl.op == "general" else None,
                             weight_offset=wl.weight_offset if wl.op == "general" else None
                             ).to(DEV)
        cat = lambda a, b: None if a is None else \
            torch.cat([b[:before], a[r:r + 1], b[before:]]).contiguous()
        moved = dataclasses.replace(wl, rows=before + 1 + after, x=cat(wl.x, pad.x),
                                    z=cat(wl.z, pad.z), dy=cat(wl.dy, pad.dy), seq_lens=None)
        out = run(cuda_lib, moved)
        for k in keys:
            assert torch.equal(bits(out[k][before:before + 1]), bits(full[k][r:r + 1])), \
                (k, r, "shifted", before)


def _prefix_sweep(cuda_lib, wl, prefixes, keys):
    """Rows of each prefix batch equal the same rows of the full batch, and the
    prefix's dw is the same across launch geometries and repeats."""
    full = run(cuda_lib, wl)
    for b in prefixes:
        part = run(cuda_lib, sub(wl, 0, b)) if b < wl.rows else full
        for k in keys:
            assert torch.equal(bits(part[k]), bits(full[k][:b])), (k, b)
        ref_dw = bits(part["dw"]).clone()
        for geo in ((1, 1, 8), (7, 2, 64), (148, 0, 0), (0, 8, 256), (0, 0, 0)):
            cuda_lib.rn_test_set_geometry(*geo)
            again = run(cuda_lib, sub(wl, 0, b)) if b < wl.rows else run(cuda_lib, wl)
            assert torch.equal(bits(again["dw"]), ref_dw), (b, geo)
            for k in keys:
                assert torch.equal(bits(again[k]), bits(full[k][:b])), (k, b, geo)
        cuda_lib.rn_test_set_geometry(0, 0, 0)
    return full


@pytest.mark.slow
def test_wide_8192_batch_size_sweep_bitwise(cuda_lib):
    # the 32768 x 8192 bf16 workload: every row of the prefixes 1, 7, 128, 4096
    # equals the same row of the full batch (512-thread teams, the shared-memory
    # warp tree), dw is the same across geometries, and sampled rows alone and
    # at shifted offsets keep their bits
    wl = workloads.cfg_wide_8192().to(DEV)
    full = _prefix_sweep(cuda_lib, wl, workloads.SWEEP_8192, ("y", "rstd", "dx"))
    pick = np.random.default_rng(2).choice(wl.rows, 14, replace=False).tolist() + [0, wl.rows - 1]
    _alone_and_shifted(cuda_lib, wl, full, pick, seed=3, keys=("y", "rstd", "dx"))


@pytest.mark.parametrize("op,rows,width,dtype,act,off", [
    ("general", 3000, 5120, "bf16", "none", 1.0),      # 128 x 5 teams
    ("general", 1200, 5120, "bf16", "silu", 0.0),
    ("gated", 600, 16384, "f32", None, None),          # 1024 x 4 teams
    ("norm", 600, 16384, "bf16", None, None),          # 512 x 4 teams
    ("gated", 2000, 4104, "bf16", None, None),         # 512 x 2, vector slots left idle
])
def test_multiwarp_batch_size_sweep_bitwise(cuda_lib, op, rows, width, dtype, act, off):
    wl = workloads.make(op, rows, width, dtype, seed=width + rows, act=act,
                        weight_offset=off, w_mean=1.0 if off in (None, 0.0) else 0.0).to(DEV)
    keys = ("y", "rstd", "dx") + (("dz",) if wl.gated else ())
    full = _prefix_sweep(cuda_lib, wl, (1, 7, 128, rows // 2 + 3, rows), keys)
    pick = np.random.default_rng(rows).choice(rows, 6, replace=False).tolist() + [rows - 1]
    _alone_and_shifted(cuda_lib, wl, full, pick, seed=width, keys=keys)
