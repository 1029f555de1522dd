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


# ---- shared memory: every launch shape fits the 227 KB a CTA may use -------------
SMEM_LIMIT = 227 * 1024


def fwd_block(t, k):
    return (128 if k <= 2 else 64) if t <= 16 else (128 if t == 32 else t)


def fwd_stages(t, gated, resid, ve):
    if t <= 32 or (t == 128 and gated and not resid and ve == 8):
        return 3
    return 2 if t <= 512 else 1


def bwd_stages(t, k, gated=True):
    if t <= 16:
        return 3
    if t <= 128:
        return 2 if gated and t == 32 else (3 if gated and t == 128 and k >= 3 else 4)
    return (3 if k <= 2 else 2) if t <= 512 else 1


def gain_in_smem(t, k, ve):
    """The gain is staged in shared memory for sub-warp teams and for threads
    of more than 16 elements in rows of at most 8192 elements."""
    return t <= 16 or (k * ve > 16 and t * k * ve <= 8192)


def fwd_smem(t, k, ve, gated, resid):
    b = fwd_block(t, k)
    nt, w = b // t, (t // 32 if t > 32 else 1)
    red = 2 * nt * w * 4 if t > 32 else 0
    gain = k * t * ve * 4 if gain_in_smem(t, k, ve) else 0
    return red + gain + fwd_stages(t, gated, resid, ve) * (1 + gated + resid) * k * b * 16


def bwd_smem(t, k, ve, lpc, width, tensors):
    bd, w = lpc * t, (t // 32 if t > 32 else 1)
    red = 2 * lpc * w * 4 if t > 32 else 0
    gain = k * t * ve * 4 if gain_in_smem(t, k, ve) else 0
    gated = tensors == 3
    stages = bwd_stages(t, k, gated) * tensors * k * bd * 16
    leaves = lpc * width * 4 if lpc > 1 else 0
    return red + gain + stages + leaves + bwd_stages(t, k, gated) * bd * 4


def bwd_lpc(t, k, ve, width):
    lpc = (8 * t if t <= 32 else (256 if t <= 128 else t)) // t
    if t > 32 and width > 2048:
        lpc = 1
    lpc = min(lpc, 8)
    while lpc > 1 and bwd_smem(t, k, ve, lpc, width, 3) > 96 * 1024:
        lpc //= 2
    return lpc


@pytest.mark.parametrize("ve", [8, 4])
def test_every_shape_fits_shared_memory(ve):
    worst = 0
    for width in range(8, 16385, 8):
        t, k = fwd_shape(width, ve)
        for gated in (False, True):          # x; + z; + r; + both
            for resid in (False, True):
                worst = max(worst, fwd_smem(t, k, ve, gated, resid))
        tb, kb = bwd_shape(width, ve)
        stripe = width // ve == tb * kb and tb <= 8 and (tb * kb * ve) % 128 == 0
        if stripe:                            # gain, stages, rstd stages, transpose buffer
            s = kb * tb * ve * 4 + 3 * 3 * kb * 32 * 16 + 3 * 32 * 4 + (32 // tb) * (width + 4) * 4
        else:                                 # dh is read into registers, not staged
            lpc = bwd_lpc(tb, kb, ve, width)
            s = max(bwd_smem(tb, kb, ve, lpc, width, 3), bwd_smem(tb, kb, ve, lpc, width, 2))
        worst = max(worst, s)
    assert worst <= SMEM_LIMIT, worst
