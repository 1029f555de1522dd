"""The C ABI without a GPU: the library loads, exports every function
include/rn.h declares, and its argument checks return the documented status
without touching CUDA (validate-only mode; the fake pointers below are never
dereferenced)."""
import contextlib
import os
import re
import subprocess

import pytest

import rollout_parity_b200 as rn
from rollout_parity_b200 import build as rn_build
from rollout_parity_b200._lib import SIGNATURES, Act, DType, Status

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rn.h")


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(
        r"^(?:rn_status|size_t|const char\s*\*|int64_t|int32_t|int|void)\s+(\w+)\s*\(", text,
        flags=re.M)))


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


def test_header_declares_the_expected_api():
    assert header_functions() == sorted(SIGNATURES)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", rn.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if ln.strip()}
    for name in header_functions():
        assert name in exported, name
        assert hasattr(lib, name)


# fake device addresses, 4 GiB apart so nothing overlaps unless a test says so
BASE = 1 << 40
def P(i, off=0):
    return BASE + (i << 32) + off


R, H = 64, 128
X, Z, W, Y, RS, DY, DX, DZ, DW, WS = range(10)


def fwd(lib, rows=R, width=H, eps=1e-6, dt=DType.BF16, x=None, w=None, y=None, rstd=None):
    return lib.norm_fwd(rows, width, eps, dt, P(X) if x is None else x, P(W) if w is None else w,
                        P(Y) if y is None else y, P(RS) if rstd is None else rstd, None)


def gfwd(lib, rows=R, width=H, eps=1e-6, dt=DType.BF16, x=None, z=None, w=None, y=None,
         rstd=None):
    return lib.gated_norm_fwd(rows, width, eps, dt, P(X) if x is None else x,
                              P(Z) if z is None else z, P(W) if w is None else w,
                              P(Y) if y is None else y, P(RS) if rstd is None else rstd, None)


def gbwd(lib, rows=R, width=H, eps=1e-6, dt=DType.BF16, ws_bytes=None, **kw):
    ptr = dict(x=P(X), z=P(Z), w=P(W), dy=P(DY), rstd=P(RS), dx=P(DX), dz=P(DZ), dw=P(DW),
               ws=P(WS))
    ptr.update(kw)
    nws = lib.norm_bwd_workspace_bytes(rows, width) if ws_bytes is None else ws_bytes
    return lib.gated_norm_bwd(rows, width, eps, dt, ptr["x"], ptr["z"], ptr["w"], ptr["dy"],
                              ptr["rstd"], ptr["dx"], ptr["dz"], ptr["dw"], ptr["ws"], nws, None)


def bwd(lib, rows=R, width=H, eps=1e-6, dt=DType.BF16, ws_bytes=None, **kw):
    ptr = dict(x=P(X), w=P(W), dy=P(DY), rstd=P(RS), dx=P(DX), dw=P(DW), ws=P(WS))
    ptr.update(kw)
    nws = lib.norm_bwd_workspace_bytes(rows, width) if ws_bytes is None else ws_bytes
    return lib.norm_bwd(rows, width, eps, dt, ptr["x"], ptr["w"], ptr["dy"], ptr["rstd"],
                        ptr["dx"], ptr["dw"], ptr["ws"], nws, None)


FWD_CASES = [
    ("valid", {}, Status.OK),
    ("valid f32", dict(dt=DType.F32), Status.OK),
    ("rstd NULL", dict(rstd=0), Status.OK),
    ("rstd 4-byte aligned", dict(rstd=P(RS, 4)), Status.OK),
    ("rows 0, no tensors", dict(rows=0, x=0, y=0), Status.OK),
    ("rows < 0", dict(rows=-1), Status.E_ARG),
    ("rows too large", dict(rows=(1 << 36) + 1), Status.E_ARG),
    ("eps < 0", dict(eps=-1e-6), Status.E_ARG),
    ("eps nan", dict(eps=float("nan")), Status.E_ARG),
    ("eps inf", dict(eps=float("inf")), Status.E_ARG),
    ("dtype", dict(dt=7), Status.E_DTYPE),
    ("width 0", dict(width=0), Status.E_WIDTH),
    ("width 4", dict(width=4), Status.E_WIDTH),
    ("width 12", dict(width=12), Status.E_WIDTH),
    ("width 16392", dict(width=16392), Status.E_WIDTH),
    ("width < 0", dict(width=-8), Status.E_WIDTH),
    ("x NULL", dict(x=0), Status.E_ARG),
    ("w NULL", dict(w=0), Status.E_ARG),
    ("y NULL", dict(y=0), Status.E_ARG),
    ("x misaligned", dict(x=P(X, 2)), Status.E_ALIGN),
    ("w misaligned", dict(w=P(W, 4)), Status.E_ALIGN),
    ("y misaligned", dict(y=P(Y, 8)), Status.E_ALIGN),
    ("rstd misaligned", dict(rstd=P(RS, 2)), Status.E_ALIGN),
    ("y aliases x", dict(y=P(X)), Status.E_ARG),
    ("y overlaps x tail", dict(y=P(X, R * H * 2 - 16)), Status.E_ARG),
    ("y just after x", dict(y=P(X, R * H * 2)), Status.OK),
    ("rstd inside y", dict(rstd=P(Y, 64)), Status.E_ARG),
    ("y overlaps w", dict(y=P(W, -16)), Status.E_ARG),
]


@pytest.mark.parametrize("name,kw,want", FWD_CASES, ids=[c[0] for c in FWD_CASES])
def test_norm_fwd_checks(lib, name, kw, want):
    with validate_only(lib):
        assert fwd(lib, **kw) == want


GFWD_CASES = [
    ("valid", {}, Status.OK),
    ("z NULL", dict(z=0), Status.E_ARG),
    ("z misaligned", dict(z=P(Z, 2)), Status.E_ALIGN),
    ("z == x is allowed", dict(z=P(X)), Status.OK),
    ("y aliases z", dict(y=P(Z)), Status.E_ARG),
    ("rows 0", dict(rows=0, x=0, z=0, y=0), Status.OK),
]


@pytest.mark.parametrize("name,kw,want", GFWD_CASES, ids=[c[0] for c in GFWD_CASES])
def test_gated_norm_fwd_checks(lib, name, kw, want):
    with validate_only(lib):
        assert gfwd(lib, **kw) == want


GBWD_CASES = [
    ("valid", {}, Status.OK),
    ("rstd NULL recomputes", dict(rstd=0), Status.OK),
    ("ws NULL", dict(ws=0), Status.E_WORKSPACE),
    ("ws too small", dict(ws_bytes=1024), Status.E_WORKSPACE),
    ("ws misaligned", dict(ws=P(WS, 8)), Status.E_ALIGN),
    ("ws overlaps dx", dict(ws=P(DX, 256)), Status.E_ARG),
    ("ws overlaps x", dict(ws=P(X)), Status.E_ARG),
    ("dw NULL", dict(dw=0), Status.E_ARG),
    ("dz NULL", dict(dz=0), Status.E_ARG),
    ("dx aliases dy", dict(dx=P(DY)), Status.E_ARG),
    ("dz aliases dx", dict(dz=P(DX)), Status.E_ARG),
    ("dw overlaps w", dict(dw=P(W)), Status.E_ARG),
    ("dw inside dz", dict(dw=P(DZ, 4096)), Status.E_ARG),
    ("dy misaligned", dict(dy=P(DY, 2)), Status.E_ALIGN),
    ("dw misaligned", dict(dw=P(DW, 4)), Status.E_ALIGN),
    ("rows 0 only needs dw", dict(rows=0, x=0, z=0, dy=0, dx=0, dz=0, ws=0, rstd=0), Status.OK),
    ("rows 0 still needs dw", dict(rows=0, dw=0), Status.E_ARG),
    ("width", dict(width=20), Status.E_WIDTH),
    ("dtype", dict(dt=7), Status.E_DTYPE),
    ("fp16", dict(dt=DType.F16), Status.OK),
]


@pytest.mark.parametrize("name,kw,want", GBWD_CASES, ids=[c[0] for c in GBWD_CASES])
def test_gated_norm_bwd_checks(lib, name, kw, want):
    with validate_only(lib):
        assert gbwd(lib, **kw) == want


BWD_CASES = [
    ("valid", {}, Status.OK),
    ("ws too small by one byte", dict(ws_bytes="need-1"), Status.E_WORKSPACE),
    ("dx aliases x", dict(dx=P(X)), Status.E_ARG),
    ("rstd overlaps dx", dict(rstd=P(DX, 16)), Status.E_ARG),
]


@pytest.mark.parametrize("name,kw,want", BWD_CASES, ids=[c[0] for c in BWD_CASES])
def test_norm_bwd_checks(lib, name, kw, want):
    if kw.get("ws_bytes") == "need-1":
        kw = dict(kw, ws_bytes=lib.norm_bwd_workspace_bytes(R, H) - 1)
    with validate_only(lib):
        assert bwd(lib, **kw) == want


def rfwd(lib, rows=R, width=H, eps=1e-6, woff=1.0, act=Act.SIGMOID, dt=DType.BF16, **kw):
    ptr = dict(x=P(X), z=P(Z), w=P(W), y=P(Y), rstd=P(RS))
    ptr.update(kw)
    return lib.rmsnorm_fwd(rows, width, eps, woff, act, dt, ptr["x"], ptr["z"], ptr["w"],
                           ptr["y"], ptr["rstd"], None)


def rbwd(lib, rows=R, width=H, eps=1e-6, woff=1.0, act=Act.SIGMOID, dt=DType.BF16, **kw):
    ptr = dict(x=P(X), z=P(Z), w=P(W), dy=P(DY), rstd=P(RS), dx=P(DX), dz=P(DZ), dw=P(DW),
               ws=P(WS))
    ptr.update(kw)
    nws = lib.norm_bwd_workspace_bytes(rows, width)
    return lib.rmsnorm_bwd(rows, width, eps, woff, act, dt, ptr["x"], ptr["z"], ptr["w"],
                           ptr["dy"], ptr["rstd"], ptr.get("mask"), ptr["dx"], ptr["dz"],
                           ptr["dw"], ptr["ws"], nws, None)


GENERAL_CASES = [
    ("sigmoid offset 1", {}, Status.OK),
    ("silu offset 0", dict(act=Act.SILU, woff=0.0), Status.OK),
    ("offset -0.0", dict(woff=-0.0), Status.OK),
    ("offset 2.5", dict(woff=2.5), Status.OK),
    ("fp16", dict(dt=DType.F16), Status.OK),
    ("fp32", dict(dt=DType.F32), Status.OK),
    ("no gate, z NULL", dict(act=Act.NONE, z=0, dz=0), Status.OK),
    ("no gate but z given", dict(act=Act.NONE, dz=0), Status.E_ARG),
    ("gate without z", dict(z=0), Status.E_ARG),
    ("activation 3", dict(act=3), Status.E_ARG),
    ("activation -1", dict(act=-1), Status.E_ARG),
    ("offset nan", dict(woff=float("nan")), Status.E_ARG),
    ("offset inf", dict(woff=float("inf")), Status.E_ARG),
    ("dtype 3", dict(dt=3), Status.E_DTYPE),
    ("y aliases z", dict(y=P(Z), dx=P(Z)), Status.E_ARG),
    ("rows 0", dict(rows=0, x=0, z=0, y=0, dy=0, dx=0, dz=0, ws=0, rstd=0), Status.OK),
]


MASK_CASES = [
    ("row mask", dict(mask=P(10)), Status.OK),
    ("row mask unaligned is fine", dict(mask=P(10, 3)), Status.OK),
    ("row mask inside dx", dict(mask=P(DX, 64)), Status.E_ARG),
    ("row mask over ws", dict(mask=P(WS, 16)), Status.E_ARG),
    ("row mask may share x", dict(mask=P(X, 64)), Status.OK),
]


@pytest.mark.parametrize("name,kw,want", MASK_CASES, ids=[c[0] for c in MASK_CASES])
def test_row_mask_checks(lib, name, kw, want):
    with validate_only(lib):
        assert rbwd(lib, **kw) == want


@pytest.mark.parametrize("name,kw,want", GENERAL_CASES, ids=[c[0] for c in GENERAL_CASES])
def test_general_entry_checks(lib, name, kw, want):
    fk = {k: v for k, v in kw.items() if k in ("rows", "width", "eps", "woff", "act", "dt", "x",
                                               "z", "w", "y", "rstd")}
    bk = {k: v for k, v in kw.items() if k not in ("y",)}
    with validate_only(lib):
        assert rfwd(lib, **fk) == want
        if name != "no gate but z given" or "dz" in kw:
            assert rbwd(lib, **bk) == want


def test_general_backward_rejects_dz_without_gate(lib):
    with validate_only(lib):
        assert rbwd(lib, act=Act.NONE, z=0) == Status.E_ARG          # dz given
        assert rbwd(lib, act=Act.NONE, z=0, dz=0) == Status.OK


def test_binding_activation_names():
    assert rn.act_code(None) == Act.NONE and rn.act_code("none") == Act.NONE
    assert rn.act_code("silu") == Act.SILU and rn.act_code("swish") == Act.SILU
    assert rn.act_code("SiLU") == Act.SILU and rn.act_code("sigmoid") == Act.SIGMOID
    with pytest.raises(ValueError):
        rn.act_code("gelu")


HH, RR, DH = 11, 12, 13


def afwd(lib, rows=R, width=H, act=Act.SILU, **kw):
    ptr = dict(x=P(X), r=P(RR), z=P(Z), w=P(W), h=P(HH), y=P(Y), rstd=P(RS))
    ptr.update(kw)
    return lib.rmsnorm_add_fwd(rows, width, 1e-6, 0.0, act, DType.BF16, ptr["x"], ptr["r"],
                               ptr["z"], ptr["w"], ptr["h"], ptr["y"], ptr["rstd"], None)


def abwd(lib, rows=R, width=H, act=Act.SILU, **kw):
    ptr = dict(h=P(HH), z=P(Z), w=P(W), dy=P(DY), dh=P(DH), rstd=P(RS), dx=P(DX), dz=P(DZ),
               dw=P(DW), ws=P(WS))
    ptr.update(kw)
    return lib.rmsnorm_add_bwd(rows, width, 1e-6, 0.0, act, DType.BF16, ptr["h"], ptr["z"],
                               ptr["w"], ptr["dy"], ptr["dh"], ptr["rstd"], None, ptr["dx"],
                               ptr["dz"], ptr["dw"], ptr["ws"],
                               lib.norm_bwd_workspace_bytes(rows, width), None)


ADD_FWD_CASES = [
    ("valid", {}, Status.OK),
    ("h is r", dict(h=P(RR)), Status.OK),
    ("h is x", dict(h=P(X)), Status.OK),
    ("h shifted into r", dict(h=P(RR, 16)), Status.E_ARG),
    ("h is y", dict(h=P(Y)), Status.E_ARG),
    ("r NULL", dict(r=0), Status.E_ARG),
    ("h NULL", dict(h=0), Status.E_ARG),
    ("r misaligned", dict(r=P(RR, 2)), Status.E_ALIGN),
    ("no gate", dict(act=Act.NONE, z=0), Status.OK),
]


@pytest.mark.parametrize("name,kw,want", ADD_FWD_CASES, ids=[c[0] for c in ADD_FWD_CASES])
def test_add_fwd_checks(lib, name, kw, want):
    with validate_only(lib):
        assert afwd(lib, **kw) == want


ADD_BWD_CASES = [
    ("valid", {}, Status.OK),
    ("dh NULL", dict(dh=0), Status.OK),
    ("dx is dh", dict(dx=P(DH)), Status.OK),
    ("dx shifted into dh", dict(dx=P(DH, 32)), Status.E_ARG),
    ("dz is dh", dict(dz=P(DH)), Status.E_ARG),
    ("dh misaligned", dict(dh=P(DH, 8)), Status.E_ALIGN),
]


@pytest.mark.parametrize("name,kw,want", ADD_BWD_CASES, ids=[c[0] for c in ADD_BWD_CASES])
def test_add_bwd_checks(lib, name, kw, want):
    with validate_only(lib):
        assert abwd(lib, **kw) == want


@pytest.mark.parametrize("rows", [1, 31, 32, 33, 256, 257, 4096, 262144, 1 << 30])
@pytest.mark.parametrize("width", [8, 128, 2048, 8192, 16384])
def test_workspace_bytes(lib, rows, width):
    leaves = -(-rows // 32)
    assert lib.norm_bwd_workspace_bytes(rows, width) == (leaves + -(-leaves // 8)) * width * 4


def test_workspace_bytes_invalid(lib):
    assert lib.norm_bwd_workspace_bytes(0, 128) == 0
    assert lib.norm_bwd_workspace_bytes(-5, 128) == 0
    assert lib.norm_bwd_workspace_bytes(64, 100) == 0


@pytest.mark.parametrize("width,dt,team", [(128, DType.BF16, 8), (128, DType.F32, 8),
                                           (8, DType.BF16, 1), (2048, DType.BF16, 128),
                                           (8192, DType.BF16, 512), (5120, DType.BF16, 128),
                                           (6144, DType.BF16, 256), (10240, DType.BF16, 256),
                                           (5120, DType.F32, 256), (4104, DType.BF16, 512),
                                           (16384, DType.F32, 1024), (128, DType.F16, 8),
                                           (64, DType.F32, 4), (120, DType.BF16, 4),
                                           (5120, DType.F16, 128), (2048, DType.F16, 128)])
def test_describe(lib, width, dt, team):
    d = lib.rn_describe(width, dt).decode()
    assert f" team_threads={team} " in d
    assert "acc=fp32" in d and "atomics=none" in d and "fast_math=off" in d
    # the backward runs the forward's team, except 16-bit rows of 128 (4 x 4, the
    # forward's 8 x 2 order)
    bwd = 4 if (width == 128 and dt in (DType.BF16, DType.F16)) else team
    assert f" bwd_team_threads={bwd} " in d


def test_describe_unsupported(lib):
    assert lib.rn_describe(100, DType.BF16) == b"unsupported"
    assert lib.rn_describe(128, 9) == b"unsupported"


def test_geometry_knob_checks(lib):
    try:
        assert lib.rn_test_set_geometry(-1, 0, 0) == Status.E_ARG
        assert lib.rn_test_set_geometry(0, 3, 0) == Status.E_ARG
        assert lib.rn_test_set_geometry(0, 0, 4) == Status.E_ARG
        assert lib.rn_test_set_geometry(0, 0, 512) == Status.E_ARG
        assert lib.rn_test_set_geometry(0, 0, 24) == Status.E_ARG
        assert lib.rn_test_set_geometry(7, 2, 64) == Status.OK
    finally:
        assert lib.rn_test_set_geometry(0, 0, 0) == Status.OK


def test_bwd_launch_count(lib):
    # 262144 rows of width 128 (stripe kernel): 8192 leaves, 8 per warp -> 1024 partials
    # -> one fold pass of up to 1024 rows
    assert lib.rn_bwd_launches(262144, 128, DType.BF16) == 2
    # small batches spread one leaf per warp: 8 or 128 partials, one fold pass
    assert lib.rn_bwd_launches(256, 128, DType.BF16) == 2
    assert lib.rn_bwd_launches(4096, 128, DType.BF16) == 2
    # width 136 (team-per-leaf kernel, 8 leaves per CTA): one CTA writes dw itself
    assert lib.rn_bwd_launches(256, 136, DType.BF16) == 1
    # 2^22 rows at width 2048 (one leaf per CTA): 131072 partials -> 4096 -> 128 -> dw
    assert lib.rn_bwd_launches(1 << 22, 2048, DType.BF16) == 1 + 3
    assert lib.rn_bwd_launches(0, 128, DType.BF16) == 1      # the fill of dw with -0.0
    assert lib.rn_bwd_launches(64, 100, DType.BF16) == 0
    try:
        lib.rn_test_set_geometry(0, 1, 8)                         # 8192 leaves, 8 rows/pass
        assert lib.rn_bwd_launches(262144, 128, DType.BF16) == 1 + 5
    finally:
        lib.rn_test_set_geometry(0, 0, 0)


def test_fold_rows_checks(lib):
    with validate_only(lib):
        assert lib.rn_fold_rows(8, 128, P(X), P(Y), None) == Status.OK
        assert lib.rn_fold_rows(256, 128, P(X), P(Y), None) == Status.OK
        assert lib.rn_fold_rows(0, 128, P(X), P(Y), None) == Status.E_ARG
        assert lib.rn_fold_rows(257, 128, P(X), P(Y), None) == Status.E_ARG
        assert lib.rn_fold_rows(8, 12, P(X), P(Y), None) == Status.E_WIDTH
        assert lib.rn_fold_rows(8, 128, P(X, 4), P(Y), None) == Status.E_ALIGN
        assert lib.rn_fold_rows(8, 128, P(X), P(X, 7 * 512), None) == Status.E_ARG   # overlap
        assert lib.rn_fold_rows(8, 128, 0, P(Y), None) == Status.E_ARG


def test_status_strings(lib):
    for s in Status:
        assert lib.rn_status_string(int(s))
    assert lib.rn_last_cuda_error() == 0


def test_binding_rejects_host_tensors(lib):
    import torch
    x = torch.zeros(4, 128, dtype=torch.bfloat16)
    w = torch.zeros(128)
    with pytest.raises(ValueError):
        rn.norm_fwd(x, w)


def cbwd(lib, rows=R, width=H, act=Act.SILU, woff=0.0, dt=DType.BF16, **kw):
    ptr = dict(x=P(X), z=P(Z), w=P(W), dy=P(DY), rstd=P(RS), dx=P(DX), dz=P(DZ), dw=P(DW),
               ws=P(WS))
    ptr.update(kw)
    nws = kw.get("ws_bytes", lib.norm_bwd_workspace_bytes(rows, width))
    return lib.rmsnorm_bwd_chunks(rows, width, 1e-6, woff, act, dt, ptr["x"], ptr["z"], ptr["w"],
                                  ptr["dy"], ptr["rstd"], ptr.get("mask"), ptr["dx"], ptr["dz"],
                                  ptr["dw"], ptr["ws"], nws, None)


def test_chunk_count(lib):
    for rows, want in ((0, 0), (1, 1), (256, 1), (257, 2), (262144, 1024), (-1, 0),
                       ((1 << 36) + 1, 0)):
        assert lib.rmsnorm_bwd_chunk_count(rows) == want, rows


def test_chunk_backward_checks(lib):
    with validate_only(lib):
        assert cbwd(lib) == Status.OK
        assert cbwd(lib, act=Act.NONE, woff=1.0, z=0, dz=0) == Status.OK
        assert cbwd(lib, rows=0, x=0, z=0, dy=0, dx=0, dz=0, ws=0, rstd=0) == Status.OK
        assert cbwd(lib, rows=0, x=0, z=0, dy=0, dx=0, dz=0, ws=0, rstd=0, dw=0) == Status.OK
        assert cbwd(lib, ws=0) == Status.E_WORKSPACE
        assert cbwd(lib, dw=0) == Status.E_ARG
        assert cbwd(lib, width=20) == Status.E_WIDTH
        # the chunk partials span ceil(R/256) rows of width floats: an output
        # that starts inside them overlaps (a [width] dw would not reach it)
        nc = lib.rmsnorm_bwd_chunk_count(1000)
        assert nc == 4
        assert cbwd(lib, rows=1000, dx=P(DW, H * 4 * (nc - 1))) == Status.E_ARG
        assert rbwd(lib, rows=1000, act=Act.SILU, woff=0.0, dx=P(DW, H * 4 * (nc - 1))) == \
            Status.OK


def test_fold_tree_checks(lib):
    need = lib.rn_fold_tree_workspace_bytes(3000, 128)
    assert need == (375 + 47) * 128 * 4
    assert lib.rn_fold_tree_workspace_bytes(0, 128) == 0
    assert lib.rn_fold_tree_workspace_bytes(8, 12) == 0
    with validate_only(lib):
        assert lib.rn_fold_tree(3000, 128, P(X), P(Y), P(WS), need, None) == Status.OK
        assert lib.rn_fold_tree(1, 128, P(X), P(Y), P(WS), 1024, None) == Status.OK
        assert lib.rn_fold_tree(0, 128, P(X), P(Y), P(WS), need, None) == Status.E_ARG
        assert lib.rn_fold_tree(3000, 128, P(X), P(Y), P(WS), need - 1, None) == Status.E_WORKSPACE
        assert lib.rn_fold_tree(3000, 128, P(X), P(Y), 0, need, None) == Status.E_WORKSPACE
        assert lib.rn_fold_tree(3000, 12, P(X), P(Y), P(WS), need, None) == Status.E_WIDTH
        assert lib.rn_fold_tree(3000, 128, P(X, 4), P(Y), P(WS), need, None) == Status.E_ALIGN
        assert lib.rn_fold_tree(3000, 128, P(X), P(X, 512), P(WS), need, None) == Status.E_ARG
        assert lib.rn_fold_tree(3000, 128, P(X), P(Y), P(X, 1024), need, None) == Status.E_ARG
        assert lib.rn_fold_tree(3000, 128, P(X), P(Y), P(Y), need, None) == Status.E_ARG
