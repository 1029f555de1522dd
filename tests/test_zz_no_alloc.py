"""gated_norm_bwd_static_ws: the gated backward that allocates nothing.

Some callers cannot allocate device memory: hosts that give a library only
each call's input and output buffers and own all other device memory (plugin
interfaces, runtimes with a fixed memory plan), or code where cudaMalloc's
device synchronisation or its bypass of the host's memory accounting is not
allowed.  For them the library keeps the backward's dw-partial scratch in its
own static 8 MiB device block.  These tests call that entry point through the
C ABI and compare it with gated_norm_bwd (caller workspace) on the same
inputs; both run the same kernels, so the tolerance is bitwise equality.

This file is collected last so that a run stopping at its first failure has
already run every other test; it also passes when run alone.
"""
import pytest
import torch

from rollout_parity_b200 import workloads
from rollout_parity_b200._lib import DType, Status

STATIC_SCRATCH_BYTES = 8 << 20


def _bits(t):
    return t.view(torch.int16 if t.dtype == torch.bfloat16 else torch.int32)


def _static_bwd(lib, wl, rstd, dx, dz, dw):
    return lib.gated_norm_bwd_static_ws(
        wl.rows, wl.width, wl.eps, int(DType.BF16 if wl.dtype == "bf16" else DType.F32),
        wl.x.data_ptr(), wl.z.data_ptr(), wl.w.data_ptr(), wl.dy.data_ptr(),
        rstd.data_ptr() if rstd is not None else None, dx.data_ptr(), dz.data_ptr(),
        dw.data_ptr(), torch.cuda.current_stream().cuda_stream)


@pytest.mark.gpu
def test_static_scratch_backward_matches_workspace_backward_twice(cuda_lib):
    lib = cuda_lib.load()
    dev = torch.device("cuda:0")
    # two calls in a row on different shapes: the second finds the first's
    # partials in the shared scratch and must not depend on them
    for call, (rows, width, dtype) in enumerate([(262144, 128, "bf16"), (3000, 2048, "bf16")]):
        wl = workloads.make("gated", rows, width, dtype, seed=40 + call).to(dev)
        assert lib.norm_bwd_workspace_bytes(rows, width) <= STATIC_SCRATCH_BYTES
        _, rstd = cuda_lib.gated_norm_fwd(wl.x, wl.z, wl.w, wl.eps)
        ref_dx, ref_dz, ref_dw = cuda_lib.gated_norm_bwd(wl.x, wl.z, wl.w, wl.dy, rstd, wl.eps)
        dx, dz = torch.empty_like(wl.x), torch.empty_like(wl.x)
        dw = torch.full((width,), float("nan"), device=dev)
        assert _static_bwd(lib, wl, rstd, dx, dz, dw) == Status.OK
        torch.cuda.synchronize()
        for got, want, name in ((dx, ref_dx, "dx"), (dz, ref_dz, "dz"), (dw, ref_dw, "dw")):
            assert torch.equal(_bits(got), _bits(want)), f"call {call}: {name} differs"


def test_static_scratch_backward_rejects_shapes_beyond_its_scratch():
    # the size check comes before any CUDA call, so this runs without a GPU
    import rollout_parity_b200 as rn
    from rollout_parity_b200 import build as rn_build
    rn_build.build()                       # a fresh checkout has no librn.so yet
    lib = rn.load()
    rows = 262144 * 2                      # 9.4 MiB of partials at width 128
    assert lib.norm_bwd_workspace_bytes(rows, 128) > STATIC_SCRATCH_BYTES
    fake = 1 << 40                         # never dereferenced: the call returns first
    st = lib.gated_norm_bwd_static_ws(rows, 128, 1e-6, int(DType.BF16), fake, fake, fake, fake,
                                      None, fake, fake, fake, None)
    assert st == Status.E_WORKSPACE


@pytest.mark.gpu
def test_static_scratch_backward_writes_only_its_outputs(cuda_lib):
    # dx, dz and dw sit between 256-byte guards of a sentinel pattern; a ragged
    # width (1032) and row count (3001) must leave the guards unchanged
    lib = cuda_lib.load()
    dev = torch.device("cuda:0")
    rows, width, guard = 3001, 1032, 256
    wl = workloads.make("gated", rows, width, "bf16", seed=9).to(dev)
    bufs = []

    def guarded(n_elems, dtype):
        nbytes = n_elems * torch.empty(0, dtype=dtype).element_size()
        raw = torch.full((2 * guard + nbytes,), 0x5A, dtype=torch.uint8, device=dev)
        bufs.append((raw, nbytes))
        return raw[guard:guard + nbytes].view(dtype)

    dx = guarded(rows * width, torch.bfloat16).view(rows, width)
    dz = guarded(rows * width, torch.bfloat16).view(rows, width)
    dw = guarded(width, torch.float32)
    _, rstd = cuda_lib.gated_norm_fwd(wl.x, wl.z, wl.w, wl.eps)
    assert _static_bwd(lib, wl, rstd, dx, dz, dw) == Status.OK
    torch.cuda.synchronize()
    for raw, nbytes in bufs:
        assert bool((raw[:guard] == 0x5A).all()) and bool((raw[guard + nbytes:] == 0x5A).all())
    ref_dx, ref_dz, ref_dw = cuda_lib.gated_norm_bwd(wl.x, wl.z, wl.w, wl.dy, rstd, wl.eps)
    for got, want in ((dx, ref_dx), (dz, ref_dz), (dw, ref_dw)):
        assert torch.equal(_bits(got), _bits(want))
