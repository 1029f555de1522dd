"""CPU checks of the test-side helpers: bf16 rounding/ulp and the dw tree model."""
import numpy as np
import pytest
import torch

import fold_model as fm
from numerics import F16, bf16_round, bf16_ulp, round16, ulp16


def test_bf16_round_matches_torch_on_fp32_values():
    # fp32 -> bf16 in torch is round-to-nearest-even in one step: for inputs that
    # are fp32 values the two must agree bit for bit
    rng = np.random.default_rng(0)
    a = np.concatenate([rng.normal(size=20000).astype(np.float32),
                        (rng.normal(size=2000) * 1e-39).astype(np.float32),   # subnormals
                        (rng.normal(size=2000) * 1e30).astype(np.float32)])
    want = torch.from_numpy(a).to(torch.bfloat16).to(torch.float64).numpy()
    got = bf16_round(a.astype(np.float64))
    assert np.array_equal(got, want)


def test_bf16_round_ties_to_even_without_double_rounding():
    one = 1.0
    step = 2.0 ** -7
    assert bf16_round(one + step / 2) == one                     # tie -> even (1.0)
    assert bf16_round(one + 3 * step / 2) == one + 2 * step      # tie -> even
    # just above the tie: fp64 keeps the excess that an fp32 detour would drop
    x = one + step / 2 + 2.0 ** -40
    assert bf16_round(x) == one + step
    assert bf16_round(-x) == -(one + step)
    assert np.signbit(bf16_round(-0.0))


def test_bf16_ulp():
    assert bf16_ulp(1.0) == 2.0 ** -7
    assert bf16_ulp(0.75) == 2.0 ** -8
    assert bf16_ulp(-3.0) == 2.0 ** -6
    assert bf16_ulp(0.0) == 2.0 ** -133
    assert bf16_ulp(1e-40) == 2.0 ** -133


@pytest.mark.parametrize("n,shape", [
    (1, "0"), (2, "(0+1)"), (3, "((0+1)+2)"), (4, "((0+1)+(2+3))"),
    (5, "(((0+1)+(2+3))+4)"), (6, "(((0+1)+(2+3))+(4+5))"),
    (7, "(((0+1)+(2+3))+((4+5)+6))"),
    (8, "(((0+1)+(2+3))+((4+5)+(6+7)))"),
])
def test_tree_shapes(n, shape):
    assert fm.tree_shape(n) == shape


@pytest.mark.parametrize("n", list(range(1, 70)) + [255, 256, 257, 1000, 1024, 1025])
@pytest.mark.parametrize("b", [1, 2, 3, 5])
def test_tree_over_aligned_blocks_is_the_same_tree(n, b):
    # the property the GPU fold relies on: reduce aligned blocks of 2**b nodes
    # with the same level-by-level rule, then the block results -> same tree
    blk = 2 ** b
    names = [str(i) for i in range(n)]
    add = lambda x, y: f"({x}+{y})"
    inner = [fm.pairwise_tree(names[s:s + blk], add) for s in range(0, n, blk)]
    assert fm.pairwise_tree(inner, add) == fm.pairwise_tree(names, add)


def test_tree_equals_split_at_largest_power_of_two():
    # and the recursive reading: left = perfect tree over the largest power of two
    # below n, right = the same rule on the rest
    add = lambda x, y: f"({x}+{y})"

    def split(names):
        if len(names) == 1:
            return names[0]
        p = 1
        while p * 2 < len(names):
            p *= 2
        return add(split(names[:p]), split(names[p:]))

    for n in range(1, 300):
        names = [str(i) for i in range(n)]
        assert split(names) == fm.pairwise_tree(names, add)


def test_dw_tree_exact_on_integers():
    rng = np.random.default_rng(3)
    c = rng.integers(-50, 50, size=(1000, 16)).astype(np.float32)
    assert np.array_equal(fm.dw_tree(c), c.sum(axis=0, dtype=np.int64).astype(np.float32))


def test_dw_tree_leaf_is_left_fold():
    # inside a leaf the order is ascending rows from the first one: (((a+b)+c)+...)
    big = np.float32(2.0 ** 25)
    c = np.array([[big], [1.0], [1.0], [-big]], dtype=np.float32)
    # left fold: big+1 -> big (rounded), +1 -> big, -big -> 0
    assert fm.dw_tree(c)[0] == 0.0
    # a pairwise tree over the same four would give (big+1)+(1-big) = big + (1-big) = 0 too,
    # so check a case that separates them: rows 32 apart form two leaves
    c2 = np.zeros((33, 1), dtype=np.float32)
    c2[0] = big; c2[1] = 1.0; c2[32] = 1.0
    # leaf0 = big+1 -> big (ties to even), leaf1 = 1; big + 1 -> big
    assert fm.dw_tree(c2)[0] == big


def test_f16_round_matches_torch_on_fp32_values():
    rng = np.random.default_rng(3)
    a = np.concatenate([rng.standard_normal(20000).astype(np.float32) * s
                        for s in (1e-7, 1e-5, 1e-2, 1.0, 300.0, 6e4)])
    want = torch.from_numpy(a).to(torch.float16).to(torch.float64).numpy()
    np.testing.assert_array_equal(round16(a.astype(np.float64), F16), want)


def test_f16_ulp_and_range():
    assert ulp16(1.0, F16) == 2.0 ** -10
    assert ulp16(0.0, F16) == 2.0 ** -24 and ulp16(1e-7, F16) == 2.0 ** -24
    assert round16(65504.0, F16) == 65504.0
    assert round16(65519.0, F16) == 65504.0
    assert np.isinf(round16(65520.0, F16))            # the tie rounds to even: 2**16
    assert round16(2.0 ** -25, F16) == 0.0            # tie between 0 and 2**-24 -> even (0)
    assert round16(3 * 2.0 ** -25, F16) == 2.0 ** -23
