"""Multi-rank dw on CPU (gloo, two ranks): the all-gather-then-fold of the
ranks' dw equals the declared tree over the whole batch, bitwise, and
unsupported shard shapes are refused on every rank.

The per-rank dw here comes from the fp32 tree model (tests/fold_model.py), which
the GPU tests tie bitwise to the kernels; this test covers the host logic:
rank order, the gather, the shape checks and the subtree property."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import fold_model

WIDTH = 24


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _leaf_partials(n_leaves, seed=0):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((n_leaves, WIDTH)) * 10).astype(np.float32)


def _tree_fold(t: torch.Tensor) -> torch.Tensor:
    add = lambda a, b: (a + b).astype(np.float32)
    rows = [r for r in t.numpy().astype(np.float32)]
    return torch.from_numpy(np.asarray(fold_model.pairwise_tree(rows, add), dtype=np.float32))


def _worker(rank, world, port, leaves_per_rank, rows_override, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from rollout_parity_b200 import parallel
        leaves = _leaf_partials(leaves_per_rank * world)
        mine = leaves[rank * leaves_per_rank:(rank + 1) * leaves_per_rank]
        add = lambda a, b: (a + b).astype(np.float32)
        dw_local = torch.from_numpy(np.asarray(fold_model.pairwise_tree(list(mine), add),
                                               dtype=np.float32))
        rows = rows_override[rank] if rows_override else leaves_per_rank * 32
        try:
            got = parallel.allgather_fold_dw(dw_local, rows, fold=_tree_fold)
            np.save(os.path.join(out_dir, f"r{rank}.npy"), got.numpy())
        except ValueError as e:
            open(os.path.join(out_dir, f"r{rank}.err"), "w").write(str(e))
    finally:
        dist.destroy_process_group()


def _run(tmp_path, world, leaves_per_rank, rows_override=None):
    mp.spawn(_worker, args=(world, _free_port(), leaves_per_rank, rows_override, str(tmp_path)),
             nprocs=world, join=True)


@pytest.mark.parametrize("leaves_per_rank", [1, 2, 8])
def test_two_ranks_fold_equals_whole_batch_tree(tmp_path, leaves_per_rank):
    _run(tmp_path, 2, leaves_per_rank)
    whole = np.asarray(fold_model.pairwise_tree(list(_leaf_partials(2 * leaves_per_rank)),
                                                lambda a, b: (a + b).astype(np.float32)),
                       dtype=np.float32)
    for r in range(2):
        got = np.load(tmp_path / f"r{r}.npy")
        assert np.array_equal(got.view(np.uint32), whole.view(np.uint32)), r


@pytest.mark.parametrize("rows", [[128, 96], [96, 96], [100, 100]])
def test_unsupported_shards_are_refused_on_every_rank(tmp_path, rows):
    _run(tmp_path, 2, 4, rows_override=rows)
    for r in range(2):
        assert (tmp_path / f"r{r}.err").exists(), r
        assert not (tmp_path / f"r{r}.npy").exists()


# --- any split on 256-row chunk boundaries ------------------------------------
def _contribs(rows, seed=1):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((rows, WIDTH)) * 10).astype(np.float32)


def _chunk_worker(rank, world, port, split, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from rollout_parity_b200 import parallel
        c = _contribs(sum(split))
        s0 = sum(split[:rank])
        mine = c[s0:s0 + split[rank]]
        local = (torch.from_numpy(fold_model.chunk_partials(mine)) if split[rank]
                 else torch.zeros(0, WIDTH))
        try:
            got = parallel.chunk_split_dw(local, split[rank], fold=_tree_fold)
            np.save(os.path.join(out_dir, f"r{rank}.npy"), got.numpy())
        except ValueError as e:
            open(os.path.join(out_dir, f"r{rank}.err"), "w").write(str(e))
    finally:
        dist.destroy_process_group()


def _run_chunks(tmp_path, split):
    mp.spawn(_chunk_worker, args=(len(split), _free_port(), split, str(tmp_path)),
             nprocs=len(split), join=True)


@pytest.mark.parametrize("split", [[256, 256], [512, 300], [256, 1000], [0, 777], [768, 0],
                                   [256, 512, 33], [1024, 256, 256]],
                         ids=lambda s: "-".join(map(str, s)))
def test_chunk_split_equals_whole_batch_tree(tmp_path, split):
    _run_chunks(tmp_path, split)
    whole = fold_model.dw_tree(_contribs(sum(split)))
    for r in range(len(split)):
        got = np.load(tmp_path / f"r{r}.npy")
        assert np.array_equal(got.view(np.uint32), whole.view(np.uint32)), (split, r)


@pytest.mark.parametrize("split", [[300, 256], [255, 1], [256, 100, 256]],
                         ids=lambda s: "-".join(map(str, s)))
def test_chunk_split_off_boundaries_is_refused_on_every_rank(tmp_path, split):
    _run_chunks(tmp_path, split)
    for r in range(len(split)):
        assert (tmp_path / f"r{r}.err").exists(), r
        assert not (tmp_path / f"r{r}.npy").exists()


def test_chunk_model_is_the_leaf_tree_from_its_third_level():
    # the model's own claim, checked on ragged row counts: the tree over chunk
    # partials is the declared tree over leaves
    for rows in (1, 31, 256, 257, 1000, 2048, 4100):
        c = _contribs(rows, seed=rows)
        got = fold_model.pairwise_tree(list(fold_model.chunk_partials(c)), fold_model._f32_add)
        assert np.array_equal(np.asarray(got).view(np.uint32), fold_model.dw_tree(c).view(np.uint32))
