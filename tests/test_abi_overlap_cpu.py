"""CPU, property-based: the backward's and the residual forward's buffer checks.

The C ABI refuses any output that overlaps an input or another output
(RN_E_ARG), except the in-place forms its header allows: dx may be exactly dh
in rmsnorm_add_bwd, and h may be exactly x or exactly r in rmsnorm_add_fwd.
Here buffers are laid out at random -- most apart, one output moved onto
another buffer at a random 16-byte-aligned offset -- and the library's answer
(validate-only mode: fake addresses, never dereferenced) is compared with that
rule written out in Python over the byte ranges each argument covers.
"""
import contextlib

import pytest

hypothesis = pytest.importorskip("hypothesis")
from hypothesis import given, settings, strategies as st  # noqa: E402

import rollout_parity_b200 as rn  # noqa: E402
from rollout_parity_b200 import build as rn_build  # noqa: E402
from rollout_parity_b200._lib import Act, DType, Status  # noqa: E402

BASE = 1 << 40
GAP = 1 << 34          # apart: far larger than any buffer drawn here
ESIZE = {DType.BF16: 2, DType.F16: 2, DType.F32: 4}


@pytest.fixture(scope="module")
def lib():
    rn_build.build()
    return rn.load()


@contextlib.contextmanager
def validate_only(lib):
    lib.rn_test_set_validate_only(1)
    try:
        yield
    finally:
        lib.rn_test_set_validate_only(0)


def overlaps(a, b):
    (pa, na), (pb, nb) = a, b
    return na > 0 and nb > 0 and pa < pb + nb and pb < pa + na


def rule(inputs, outputs, allowed=()):
    """Status the ranges call for: RN_E_ARG when an output overlaps an input
    (unless the pair is an allowed exact alias) or another output."""
    for i, (on, orange) in enumerate(outputs):
        for iname, irange in inputs:
            if (on, iname) in allowed and orange == irange:
                continue
            if overlaps(orange, irange):
                return Status.E_ARG
        for _, other in outputs[i + 1:]:
            if overlaps(orange, other):
                return Status.E_ARG
    return Status.OK


@st.composite
def layouts(draw, names, outputs):
    """Addresses for `names`: slot i at BASE + i*GAP, then maybe one output
    moved onto another buffer at a 16-byte-aligned offset (possibly negative)."""
    addr = {n: BASE + i * GAP for i, n in enumerate(names)}
    if draw(st.booleans()):
        mover = draw(st.sampled_from(outputs))
        target = draw(st.sampled_from([n for n in names if n != mover]))
        off = 16 * draw(st.integers(min_value=-4096, max_value=1 << 16))
        addr[mover] = addr[target] + off
    return addr


SHAPES = st.tuples(st.integers(1, 3000), st.sampled_from([8, 16, 128, 136, 1024, 2048]),
                   st.sampled_from([DType.BF16, DType.F16, DType.F32]))
BWD_NAMES = ["x", "z", "w", "dy", "dh", "rstd", "mask", "dx", "dz", "dw", "ws"]


@settings(max_examples=400, deadline=None)
@given(shape=SHAPES, addr=layouts(BWD_NAMES, ["dx", "dz", "dw", "ws"]),
       same_dx_dh=st.booleans())
def test_add_bwd_overlap_rule(lib, shape, addr, same_dx_dh):
    rows, width, dt = shape
    if same_dx_dh:
        addr = dict(addr, dx=addr["dh"])
    tb = rows * width * ESIZE[dt]
    ws = lib.norm_bwd_workspace_bytes(rows, width)
    size = dict(x=tb, z=tb, w=width * 4, dy=tb, dh=tb, rstd=rows * 4, mask=rows, dx=tb, dz=tb,
                dw=width * 4, ws=ws)
    rng = {n: (addr[n], size[n]) for n in BWD_NAMES}
    inputs = [(n, rng[n]) for n in ("x", "z", "w", "dy", "rstd", "mask", "dh")]
    outputs = [(n, rng[n]) for n in ("dx", "dz", "dw", "ws")]
    want = rule(inputs, outputs, allowed={("dx", "dh")})
    with validate_only(lib):
        got = lib.rmsnorm_add_bwd(rows, width, 1e-6, 0.0, int(Act.SILU), int(dt), addr["x"],
                                  addr["z"], addr["w"], addr["dy"], addr["dh"], addr["rstd"],
                                  addr["mask"], addr["dx"], addr["dz"], addr["dw"], addr["ws"],
                                  ws, None)
    assert got == want, (rows, width, dt, {k: hex(v) for k, v in addr.items()})


FWD_NAMES = ["x", "r", "z", "w", "h", "y", "rstd"]


@settings(max_examples=400, deadline=None)
@given(shape=SHAPES, addr=layouts(FWD_NAMES, ["h", "y", "rstd"]),
       in_place=st.sampled_from([None, "x", "r"]))
def test_add_fwd_overlap_rule(lib, shape, addr, in_place):
    rows, width, dt = shape
    if in_place is not None:
        addr = dict(addr, h=addr[in_place])
    tb = rows * width * ESIZE[dt]
    size = dict(x=tb, r=tb, z=tb, w=width * 4, h=tb, y=tb, rstd=rows * 4)
    rng = {n: (addr[n], size[n]) for n in FWD_NAMES}
    inputs = [(n, rng[n]) for n in ("x", "z", "w", "r")]
    outputs = [(n, rng[n]) for n in ("y", "rstd", "h")]
    # h may be exactly x or exactly r -- the one it starts at, when it starts at x
    allowed = {("h", "x")} if addr["h"] == addr["x"] else {("h", "r")}
    want = rule(inputs, outputs, allowed=allowed)
    with validate_only(lib):
        got = lib.rmsnorm_add_fwd(rows, width, 1e-6, 0.0, int(Act.SILU), int(dt), addr["x"],
                                  addr["r"], addr["z"], addr["w"], addr["h"], addr["y"],
                                  addr["rstd"], None)
    assert got == want, (rows, width, dt, {k: hex(v) for k, v in addr.items()})
