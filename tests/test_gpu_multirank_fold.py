"""rn_fold_rows on the GPU, and data-parallel sharding emulated on one GPU:
the dw of equal power-of-two-leaf shards, folded in shard order, equals the dw
of one backward call over the whole batch, bitwise (no collective involved;
the two-rank gather itself is covered by tests/test_parallel_cpu.py)."""
import numpy as np
import pytest
import torch

import fold_model
from rollout_parity_b200 import workloads

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _bits(t):
    return t.view(torch.int32)


@pytest.mark.parametrize("n", [1, 2, 3, 7, 8, 9, 64, 200, 256])
@pytest.mark.parametrize("width", [8, 128, 2056])
def test_fold_rows_is_the_declared_tree(cuda_lib, n, width):
    rng = np.random.default_rng(n * width)
    rows = (rng.standard_normal((n, width)) * 100).astype(np.float32)
    got = cuda_lib.rn_fold_rows(torch.from_numpy(rows).to(DEV)).cpu().numpy()
    want = np.asarray(fold_model.pairwise_tree(list(rows), lambda a, b: (a + b).astype(np.float32)),
                      dtype=np.float32)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


@pytest.mark.parametrize("op,shards,rows_per_shard,width", [
    ("gated", 4, 4096, 128), ("gated", 2, 32, 128), ("norm", 2, 1024, 2048),
    ("norm", 8, 256, 8192), ("gated", 3, 2048, 5120)])
def test_sharded_dw_folds_to_the_whole_batch_dw(cuda_lib, op, shards, rows_per_shard, width):
    wl = workloads.make(op, shards * rows_per_shard, width, "bf16", seed=shards).to(DEV)
    if op == "gated":
        whole = cuda_lib.gated_norm_bwd(wl.x, wl.z, wl.w, wl.dy, None, wl.eps)[2]
    else:
        whole = cuda_lib.norm_bwd(wl.x, wl.w, wl.dy, None, wl.eps)[1]
    parts = []
    for r in range(shards):
        s = slice(r * rows_per_shard, (r + 1) * rows_per_shard)
        x, dy = wl.x[s].contiguous(), wl.dy[s].contiguous()
        if op == "gated":
            parts.append(cuda_lib.gated_norm_bwd(x, wl.z[s].contiguous(), wl.w, dy, None, wl.eps)[2])
        else:
            parts.append(cuda_lib.norm_bwd(x, wl.w, dy, None, wl.eps)[1])
    folded = cuda_lib.rn_fold_rows(torch.stack(parts))
    assert torch.equal(_bits(folded), _bits(whole))


def test_fold_rows_rejects_bad_counts(cuda_lib):
    from rollout_parity_b200._lib import Status
    lib = cuda_lib.load()
    x = torch.zeros(257, 128, device=DEV)
    out = torch.zeros(128, device=DEV)
    assert lib.rn_fold_rows(0, 128, x.data_ptr(), out.data_ptr(), None) == Status.E_ARG
    assert lib.rn_fold_rows(257, 128, x.data_ptr(), out.data_ptr(), None) == Status.E_ARG
    assert lib.rn_fold_rows(4, 100, x.data_ptr(), out.data_ptr(), None) == Status.E_WIDTH


# --- any split on 256-row chunk boundaries ------------------------------------
@pytest.mark.parametrize("n", [1, 2, 9, 256, 257, 1000, 1025, 2049, 3000, 70000])
@pytest.mark.parametrize("width", [8, 128, 2056, 4104, 5120])
def test_fold_tree_is_the_declared_tree(cuda_lib, n, width):
    # 257..1024 rows take the one-pass fold, whose CTAs have 32, 16 or 8 warps
    # as the width needs (128, 2056: 32; 4104: 16; 5120: 8 on a 148-SM B200)
    if n * width > 70000 * 128:
        pytest.skip("kept to a few MB")
    rng = np.random.default_rng(n + width)
    rows = (rng.standard_normal((n, width)) * 100).astype(np.float32)
    want = np.asarray(fold_model.pairwise_tree(list(rows), lambda a, b: (a + b).astype(np.float32)),
                      dtype=np.float32)
    t = torch.from_numpy(rows).to(DEV)
    for fold_rows in (0, 8, 256):
        cuda_lib.rn_test_set_geometry(0, 0, fold_rows)
        got = cuda_lib.rn_fold_tree(t).cpu().numpy()
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), fold_rows
    cuda_lib.rn_test_set_geometry(0, 0, 0)


def _general(op, rows, width, dtype, seed):
    act, off = {"gated": ("silu", 0.0), "norm": ("none", 1.0), "sigmoid": ("sigmoid", 1.0)}[op]
    return workloads.make("general", rows, width, dtype, seed=seed, act=act, weight_offset=off,
                          w_mean=1.0 if off == 0.0 else 0.0).to(DEV)


SPLITS = [  # (op, width, dtype, rows per emulated rank): 256-row boundaries, last ragged
    ("gated", 128, "bf16", [4096, 4096]), ("gated", 128, "bf16", [256, 768, 1000]),
    ("gated", 128, "bf16", [0, 3001]), ("norm", 2048, "bf16", [512, 256, 77]),
    ("sigmoid", 136, "f16", [256, 0, 513]), ("norm", 8192, "bf16", [256, 300]),
    ("gated", 5120, "bf16", [768, 256]), ("norm", 16384, "f32", [256, 31]),
    ("gated", 1032, "bf16", [1280, 5]), ("norm", 128, "f32", [2560, 2560, 2560])]


@pytest.mark.parametrize("op,width,dtype,split", SPLITS,
                         ids=[f"{o}-{w}-{d}-{'-'.join(map(str, s))}" for o, w, d, s in SPLITS])
@pytest.mark.parametrize("masked", [False, True], ids=["nomask", "mask"])
def test_chunk_split_dw_is_the_one_call_dw(cuda_lib, op, width, dtype, split, masked):
    rows = sum(split)
    wl = _general(op, rows, width, dtype, seed=rows + width)
    z = wl.z
    mask = (torch.arange(rows, device=DEV) % 5 != 2).to(torch.uint8) if masked else None
    dx, dz, dw = cuda_lib.rmsnorm_bwd(wl.x, wl.w, wl.dy, None, wl.eps, wl.weight_offset, z,
                                      wl.act, row_mask=mask)
    _, _, whole_chunks = cuda_lib.rmsnorm_bwd_chunks(wl.x, wl.w, wl.dy, None, wl.eps,
                                                     wl.weight_offset, z, wl.act, row_mask=mask)
    assert whole_chunks.shape == (-(-rows // 256), width)
    parts, s0 = [], 0
    for n in split:
        sl = slice(s0, s0 + n)
        c = lambda t: None if t is None else t[sl].contiguous()
        pdx, pdz, ch = cuda_lib.rmsnorm_bwd_chunks(c(wl.x), wl.w, c(wl.dy), None, wl.eps,
                                                   wl.weight_offset, c(z), wl.act,
                                                   row_mask=c(mask))
        assert torch.equal(pdx.view(torch.uint8), dx[sl].contiguous().view(torch.uint8))
        if pdz is not None:
            assert torch.equal(pdz.view(torch.uint8), dz[sl].contiguous().view(torch.uint8))
        # a rank's chunk partials are the whole call's partials of the same chunks
        assert torch.equal(_bits(ch), _bits(whole_chunks[s0 // 256:s0 // 256 + ch.shape[0]]))
        parts.append(ch)
        s0 += n
    folded = cuda_lib.rn_fold_tree(torch.cat(parts).contiguous())
    assert torch.equal(_bits(folded), _bits(dw))


@pytest.mark.parametrize("width,dtype", [(128, "bf16"), (2048, "bf16"), (5120, "bf16")])
def test_chunk_partials_across_geometry(cuda_lib, width, dtype):
    wl = _general("gated", 3000, width, dtype, seed=width)
    ref = cuda_lib.rmsnorm_bwd_chunks(wl.x, wl.w, wl.dy, None, wl.eps, 0.0, wl.z, "silu")[2]
    for geo in ((1, 0, 0), (7, 1, 0), (148, 8, 0), (0, 1, 8), (0, 0, 0)):
        cuda_lib.rn_test_set_geometry(*geo)
        got = cuda_lib.rmsnorm_bwd_chunks(wl.x, wl.w, wl.dy, None, wl.eps, 0.0, wl.z, "silu")[2]
        assert torch.equal(_bits(got), _bits(ref)), geo
    cuda_lib.rn_test_set_geometry(0, 0, 0)


def test_chunk_partials_are_the_model_of_one_row_dws(cuda_lib):
    # chunk c = the declared tree over the one-row dws of rows [256c, 256c+256)
    rows, width = 700, 128
    wl = _general("gated", rows, width, "bf16", seed=5)
    got = cuda_lib.rmsnorm_bwd_chunks(wl.x, wl.w, wl.dy, None, wl.eps, 0.0, wl.z, "silu")[2]
    one = np.stack([cuda_lib.rmsnorm_bwd(wl.x[r:r + 1].contiguous(), wl.w,
                                         wl.dy[r:r + 1].contiguous(), None, wl.eps, 0.0,
                                         wl.z[r:r + 1].contiguous(), "silu")[2].cpu().numpy()
                    for r in range(rows)])
    want = fold_model.chunk_partials(one)
    assert np.array_equal(got.cpu().numpy().view(np.uint32), want.view(np.uint32))


def test_last_launches_counts_the_calls_kernels(cuda_lib):
    lib = cuda_lib.load()
    from rollout_parity_b200._lib import DType
    wl = _general("gated", 262144, 128, "bf16", seed=1)
    _, rstd = cuda_lib.rmsnorm_fwd(wl.x, wl.w, wl.eps, 0.0, wl.z, "silu")
    assert lib.rn_last_launches() == 1
    cuda_lib.rmsnorm_bwd(wl.x, wl.w, wl.dy, rstd, wl.eps, 0.0, wl.z, "silu")
    assert lib.rn_last_launches() == lib.rn_bwd_launches(262144, 128, int(DType.BF16))
    _, _, ch = cuda_lib.rmsnorm_bwd_chunks(wl.x, wl.w, wl.dy, rstd, wl.eps, 0.0, wl.z, "silu")
    assert lib.rn_last_launches() >= 1
    cuda_lib.rn_fold_tree(ch)
    assert lib.rn_last_launches() >= 1
    e = wl.x[:0]
    cuda_lib.rmsnorm_bwd(e, wl.w, e, None, wl.eps, 0.0, wl.z[:0], "silu")
    assert lib.rn_last_launches() == 1        # the -0.0 fill of dw
