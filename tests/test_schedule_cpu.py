"""Host-side schedule of librn, checked without a GPU against a plain restatement:
the forward team shape (rn_describe) for every supported width and element size,
and the number of kernels a backward call enqueues (rn_bwd_launches) for many
row counts.  The team shape fixes the declared reduction order, so it must
depend on (width, element size) only and cover the row exactly."""
import re

import pytest

import rollout_parity_b200 as rn
from rollout_parity_b200._lib import DType


def pow2ceil(v):
    p = 1
    while p < v:
        p <<= 1
    return p


def fwd_shape(width, ve):
    nv = width // ve
    if nv == 16 and ve == 8:
        return 8, 2
    if nv <= 32:
        t = max(1, pow2ceil(nv) // 4)
        return t, -(-nv // t)
    if nv <= 128:
        return 32, -(-nv // 32)
    if nv <= 512:
        return 128, -(-nv // 128)
    if nv <= 2048:
        if nv % 512 == 0:
            return 512, nv // 512
        if nv % 128 == 0 and nv // 128 <= 5:
            return 128, nv // 128
        if nv % 256 == 0 and nv // 256 <= 5:
            return 256, nv // 256
        return 512, -(-nv // 512)
    return 1024, -(-nv // 1024)


@pytest.fixture(scope="module")
def lib():
    return rn.load()


@pytest.mark.parametrize("dt,ve", [(DType.BF16, 8), (DType.F16, 8), (DType.F32, 4)])
def test_forward_team_shape_for_every_width(lib, dt, ve):
    for width in range(8, 16385, 8):
        d = lib.rn_describe(width, dt).decode()
        t = int(re.search(r"team_threads=(\d+)", d).group(1))
        k = int(re.search(r"vectors_per_thread=(\d+)", d).group(1))
        assert int(re.search(r"elems_per_vector=(\d+)", d).group(1)) == ve
        assert (t, k) == fwd_shape(width, ve), width
        assert t * k * ve >= width and (t * (k - 1) * ve < width), width   # no idle vector column
        assert k <= 5


def fold_passes(n):
    passes = 0
    while n > 1:
        if 256 < n <= 1024:
            return passes + 1          # one k_fold1 pass
        s = 32 if n > 256 else max(8, pow2ceil(n))
        n = -(-n // s)
        passes += 1
    return passes


def bwd_shape(width, ve):
    t, k = fwd_shape(width, ve)
    if ve == 8 and width // 8 == 16:
        return 4, 4
    return t, k


def leaves_per_cta(width, ve, rows, sms=148):
    t, k = bwd_shape(width, ve)
    nv = width // ve
    stripe = nv == t * k and t <= 8 and (t * k * ve) % 128 == 0
    leaves = -(-rows // 32)
    if stripe:
        lpc = 1
        while lpc < 8 and -(-leaves // lpc) > 8 * sms:
            lpc *= 2
        return lpc
    return None   # the team-per-leaf kernel's CTA size depends on its shared memory


@pytest.mark.parametrize("width,dt,ve", [(128, DType.BF16, 8), (256, DType.BF16, 8),
                                         (128, DType.F32, 4), (128, DType.F16, 8)])
def test_backward_launch_count_narrow_rows(lib, width, dt, ve):
    for rows in (1, 31, 32, 33, 255, 256, 257, 4096, 8191, 65536, 262144, 262145, 1 << 20,
                 (1 << 22) + 5):
        lpc = leaves_per_cta(width, ve, rows)
        groups = -(-(-(-rows // 32)) // lpc)
        assert lib.rn_bwd_launches(rows, width, dt) == 1 + fold_passes(groups), rows
