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
