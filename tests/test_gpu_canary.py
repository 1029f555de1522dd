"""Guard words around every output buffer (the host-side stand-in for a
memory checker, which this pool does not offer).

Each output -- y, rstd, h, dx, dz, dw and the backward's workspace -- is a
view into a larger device buffer whose 256 bytes before and after it hold a
sentinel bit pattern.  After the forward and backward calls the guards must be
bitwise unchanged: a store past either end of a ragged row, a row count that
is not a multiple of the 32-row leaf, or a partial vector slot would show up
as a changed guard word.  The outputs are also checked against the
unguarded call's, bitwise.
"""
import pytest
import torch

from rollout_parity_b200 import workloads

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
GUARD = 256                    # bytes on each side of every output
SENTINEL = 0x5A                # byte pattern of the guards (and of the outputs before the call)

CASES = [  # (act, offset, rows, width, dtype, residual, mask)
    ("silu", 0.0, 1000, 128, "bf16", False, False),
    ("silu", 0.0, 33, 1032, "bf16", False, False),      # ragged width: idle vector slots
    ("none", 1.0, 257, 4104, "bf16", False, True),
    ("sigmoid", 1.0, 95, 136, "f16", True, False),
    ("none", 1.0, 63, 1032, "f32", True, True),
    ("silu", 0.0, 31, 16384, "bf16", False, False),
    ("none", 1.0, 17, 16384, "f32", False, False),
    ("silu", 0.0, 300, 5120, "bf16", True, False),
    ("none", 1.0, 1, 8, "bf16", False, False),
    ("sigmoid", 0.0, 4129, 256, "bf16", False, True),
]
IDS = [f"{a}-off{int(o)}-{r}x{w}-{d}{'-res' if res else ''}{'-mask' if m else ''}"
       for a, o, r, w, d, res, m in CASES]


class Guarded:
    """Device buffers with GUARD sentinel bytes on both sides of the view."""

    def __init__(self):
        self.bufs = []

    def make(self, shape, dtype):
        n = 1
        for s in shape:
            n *= s
        nbytes = n * torch.empty(0, dtype=dtype).element_size()
        raw = torch.full((GUARD + nbytes + GUARD,), SENTINEL, dtype=torch.uint8, device=DEV)
        self.bufs.append((raw, nbytes))
        return raw[GUARD:GUARD + nbytes].view(dtype).view(shape)

    def check(self, what):
        for raw, nbytes in self.bufs:
            head, tail = raw[:GUARD], raw[GUARD + nbytes:]
            assert bool((head == SENTINEL).all()), f"{what}: guard before a buffer changed"
            assert bool((tail == SENTINEL).all()), f"{what}: guard after a buffer changed"


def bits(t):
    return t.contiguous().view(torch.uint8)


@pytest.mark.parametrize("act,off,rows,width,dtype,resid,use_mask", CASES, ids=IDS)
def test_outputs_stay_inside_their_buffers(cuda_lib, act, off, rows, width, dtype, resid,
                                           use_mask):
    wl = workloads.make("general", rows, width, dtype, seed=rows + width, act=act,
                        weight_offset=off, w_mean=1.0 if off == 0.0 else 0.0).to(DEV)
    r = workloads.make("general", rows, width, dtype, seed=rows + width + 1, act="none",
                       weight_offset=1.0).x.to(DEV) if resid else None
    mask = (torch.arange(rows, device=DEV) % 3 != 1).to(torch.uint8) if use_mask else None
    g = Guarded()
    shape = (rows, width)
    tdt = wl.x.dtype
    y, rstd = g.make(shape, tdt), g.make((rows,), torch.float32)
    dx, dw = g.make(shape, tdt), g.make((width,), torch.float32)
    dz = g.make(shape, tdt) if act != "none" else None
    ws = g.make((cuda_lib.norm_bwd_workspace_bytes(rows, width),), torch.uint8)
    if resid:
        h = g.make(shape, tdt)
        cuda_lib.rmsnorm_add_fwd(wl.x, r, wl.w, wl.eps, off, wl.z, act, h=h, y=y, rstd=rstd)
        cuda_lib.rmsnorm_add_bwd(h, wl.w, wl.dy, wl.dy, rstd, wl.eps, off, wl.z, act,
                                 row_mask=mask, dx=dx, dz=dz, dw=dw, ws=ws)
        ref_h, ref_y, ref_r = cuda_lib.rmsnorm_add_fwd(wl.x, r, wl.w, wl.eps, off, wl.z, act)
        ref = cuda_lib.rmsnorm_add_bwd(ref_h, wl.w, wl.dy, wl.dy, ref_r, wl.eps, off, wl.z, act,
                                       row_mask=mask)
        assert torch.equal(bits(h), bits(ref_h))
    else:
        cuda_lib.rmsnorm_fwd(wl.x, wl.w, wl.eps, off, wl.z, act, y=y, rstd=rstd)
        cuda_lib.rmsnorm_bwd(wl.x, wl.w, wl.dy, rstd, wl.eps, off, wl.z, act, row_mask=mask,
                             dx=dx, dz=dz, dw=dw, ws=ws)
        ref_y, ref_r = cuda_lib.rmsnorm_fwd(wl.x, wl.w, wl.eps, off, wl.z, act)
        ref = cuda_lib.rmsnorm_bwd(wl.x, wl.w, wl.dy, ref_r, wl.eps, off, wl.z, act,
                                   row_mask=mask)
    torch.cuda.synchronize()
    g.check("after the calls")
    assert torch.equal(bits(y), bits(ref_y)) and torch.equal(bits(rstd), bits(ref_r))
    for got, want in zip((dx, dz, dw), ref):
        if want is not None:
            assert torch.equal(bits(got), bits(want))

