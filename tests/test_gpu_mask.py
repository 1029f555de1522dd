"""The backward's row mask on the GPU: rows with a zero mask byte are left out
of dw (RL-Kernel PR #468, "Changes to existing code, in detail": the dw entry
point takes a mask), dx and dz stay every row's.

A left-out row stands for -0.0, the additive identity, in the declared tree,
so the masked dw must equal, bitwise, the tree model applied to the one-row
dws with the left-out rows replaced by -0.0; it must also meet the parity bar
against the oracle's masked sum, and ignore whatever values the left-out rows
hold (padding)."""
import numpy as np
import pytest
import torch

import fold_model
import oracle
from numerics import check_out
from rollout_parity_b200 import workloads

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
f64 = workloads.as_f64

CASES = [  # (act, offset, rows, width, dtype): stripe and team-per-leaf kernels
    ("silu", 0.0, 1000, 128, "bf16"), ("none", 1.0, 777, 128, "f32"),
    ("sigmoid", 1.0, 300, 2048, "bf16"), ("none", 1.0, 129, 5120, "f16"),
    ("silu", 0.0, 257, 136, "bf16"), ("sigmoid", 0.0, 5000, 256, "bf16"),
]
IDS = [f"{a}-off{int(o)}-{r}x{w}-{d}" for a, o, r, w, d in CASES]


def make(act, off, rows, width, dtype, seed):
    return workloads.make("general", rows, width, dtype, seed=seed, act=act, weight_offset=off,
                          w_mean=1.0 if off == 0.0 else 0.0).to(DEV)


def mask_of(rows, seed, frac=0.3):
    rng = np.random.default_rng(seed)
    m = (rng.random(rows) >= frac).astype(np.uint8)
    m[-1] = 0                       # a left-out last row (ragged leaf)
    return torch.from_numpy(m).to(DEV)


def bwd(rn, wl, mask=None):
    y, rstd = rn.rmsnorm_fwd(wl.x, wl.w, wl.eps, wl.weight_offset, wl.z, wl.act)
    return rn.rmsnorm_bwd(wl.x, wl.w, wl.dy, rstd, wl.eps, wl.weight_offset, wl.z, wl.act,
                          row_mask=mask)


def bits(t):
    return t.view(torch.int32)


@pytest.mark.parametrize("act,off,rows,width,dtype", CASES, ids=IDS)
def test_masked_dw_parity(cuda_lib, act, off, rows, width, dtype):
    wl = make(act, off, rows, width, dtype, seed=rows)
    m = mask_of(rows, seed=rows)
    dx, dz, dw = bwd(cuda_lib, wl, m)
    dx0, dz0, _ = bwd(cuda_lib, wl)
    assert torch.equal(dx.view(torch.int16 if dx.dtype != torch.float32 else torch.int32),
                       dx0.view(torch.int16 if dx.dtype != torch.float32 else torch.int32))
    _, _, want = oracle.rmsnorm_bwd(f64(wl.x), f64(wl.w), f64(wl.dy), wl.eps, off,
                                    None if wl.z is None else f64(wl.z), act,
                                    row_mask=m.cpu().numpy())
    check_out(dw, want, what="masked dw")


@pytest.mark.parametrize("act,off,rows,width,dtype", CASES[:3], ids=IDS[:3])
def test_masked_dw_is_the_tree_with_identity_rows(cuda_lib, act, off, rows, width, dtype):
    wl = make(act, off, rows, width, dtype, seed=rows + 1)
    m = mask_of(rows, seed=rows + 1)
    _, _, dw = bwd(cuda_lib, wl, m)
    mk = m.cpu().numpy()
    ident = np.full(width, -0.0, dtype=np.float32)
    one = []
    for r in range(rows):
        if mk[r]:
            s = slice(r, r + 1)
            sub = workloads.Workload(name="r", op="general", rows=1, width=width, dtype=dtype,
                                     eps=wl.eps, x=wl.x[s].clone(),
                                     z=None if wl.z is None else wl.z[s].clone(),
                                     dy=wl.dy[s].clone(), w=wl.w, act=act, weight_offset=off)
            one.append(bwd(cuda_lib, sub)[2].cpu().numpy())
        else:
            one.append(ident)
    model = fold_model.dw_tree(np.stack(one))
    assert np.array_equal(dw.cpu().numpy().view(np.uint32), model.view(np.uint32))


@pytest.mark.parametrize("act,off,rows,width,dtype", CASES, ids=IDS)
def test_left_out_rows_may_hold_anything(cuda_lib, act, off, rows, width, dtype):
    wl = make(act, off, rows, width, dtype, seed=rows + 2)
    m = mask_of(rows, seed=rows + 2)
    _, _, dw_clean = bwd(cuda_lib, wl, m)
    out = m == 0
    wl.x[out] = float("nan")
    wl.dy[out] = float("inf")
    if wl.z is not None:
        wl.z[out] = float("nan")
    dx, _, dw = bwd(cuda_lib, wl, m)
    assert torch.isfinite(dw).all()
    assert torch.equal(bits(dw), bits(dw_clean))


@pytest.mark.parametrize("act,off,rows,width,dtype", CASES[:3], ids=IDS[:3])
def test_everything_left_out_is_the_oracles_empty_sum(cuda_lib, act, off, rows, width, dtype):
    # no row contributes: the oracle's empty sum, sign included (-0.0), and the
    # same bits as a call with no rows at all
    wl = make(act, off, rows, width, dtype, seed=3)
    m = torch.zeros(rows, dtype=torch.uint8, device=DEV)
    _, _, dw = bwd(cuda_lib, wl, m)
    _, _, want = oracle.rmsnorm_bwd(f64(wl.x), f64(wl.w), f64(wl.dy), wl.eps, off,
                                    None if wl.z is None else f64(wl.z), act,
                                    row_mask=m.cpu().numpy())
    got = dw.cpu().numpy()
    assert np.array_equal(got, want) and np.array_equal(np.signbit(got), np.signbit(want))
    e = wl.x[:0]
    dw0 = torch.full_like(dw, 7.0)
    cuda_lib.rmsnorm_bwd(e, wl.w, e, None, wl.eps, off, None if wl.z is None else wl.z[:0], act,
                         dw=dw0)
    assert torch.equal(bits(dw0), bits(dw))


def test_all_ones_mask_is_no_mask(cuda_lib):
    for act, off, rows, width, dtype in CASES[:4]:
        wl = make(act, off, rows, width, dtype, seed=7)
        _, _, a = bwd(cuda_lib, wl, torch.ones(rows, dtype=torch.bool, device=DEV))
        _, _, b = bwd(cuda_lib, wl)
        assert torch.equal(bits(a), bits(b))
