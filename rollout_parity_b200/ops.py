"""Python binding of librn, one function per C entry point, same names.

These functions only marshal arguments: they check that torch tensors can be
described by plain pointers (CUDA, contiguous, the right dtype and shape),
allocate outputs the caller did not pass (torch is used for device memory and
streams only), and call the C ABI on the tensors' device and current stream.
Every step of the computation runs in librn's kernels; a failed status raises
RNError.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch

from ._lib import Act, DType, check, load

_DT = {torch.bfloat16: DType.BF16, torch.float16: DType.F16, torch.float32: DType.F32}
# gate activation names; "swish" is another name for silu
_ACT = {None: Act.NONE, "none": Act.NONE, "silu": Act.SILU, "swish": Act.SILU,
        "sigmoid": Act.SIGMOID}


def _dt(x: torch.Tensor) -> DType:
    if x.dtype not in _DT:
        raise TypeError(f"x dtype {x.dtype} not supported (bf16, fp16 or fp32)")
    return _DT[x.dtype]


def act_code(act) -> Act:
    """The C enum for an activation name (None/"none", "silu"/"swish",
    "sigmoid") or an Act value."""
    if isinstance(act, Act):
        return act
    key = act.lower() if isinstance(act, str) else act
    if key not in _ACT:
        raise ValueError(f"unknown activation {act!r} (none, silu, swish or sigmoid)")
    return _ACT[key]


def _mat(name: str, t: Optional[torch.Tensor], like: torch.Tensor) -> torch.Tensor:
    if t is None:
        raise ValueError(f"{name} is required")
    if t.device != like.device or t.dtype != like.dtype or tuple(t.shape) != tuple(like.shape):
        raise ValueError(f"{name} must be {tuple(like.shape)} {like.dtype} on {like.device}, "
                         f"got {tuple(t.shape)} {t.dtype} on {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _vec(name: str, t: Optional[torch.Tensor], n: int, device) -> torch.Tensor:
    if t is None:
        raise ValueError(f"{name} is required")
    if t.device != device or t.dtype != torch.float32 or tuple(t.shape) != (n,) \
            or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous fp32 [{n}] tensor on {device}")
    return t


def _rows_width(x: torch.Tensor) -> Tuple[int, int]:
    if x.dim() != 2:
        raise ValueError("x must be [rows, width]")
    if not x.is_cuda:
        raise ValueError("x must be a CUDA tensor")
    if not x.is_contiguous():
        raise ValueError("x must be contiguous")
    return int(x.shape[0]), int(x.shape[1])


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(x: torch.Tensor, stream) -> int:
    """The cudaStream_t handle: the tensors' current stream when None, a
    torch.cuda.Stream's handle, or a raw handle passed as an int."""
    if isinstance(stream, int):
        return stream
    s = torch.cuda.current_stream(x.device) if stream is None else stream
    return s.cuda_stream


def norm_bwd_workspace_bytes(rows: int, width: int) -> int:
    return int(load().norm_bwd_workspace_bytes(rows, width))


def workspace(rows: int, width: int, device) -> torch.Tensor:
    """A device buffer large enough for the backward's dw partials."""
    n = norm_bwd_workspace_bytes(rows, width)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def rmsnorm_fwd(x: torch.Tensor, w: torch.Tensor, eps: float = 1e-6, weight_offset: float = 1.0,
                z: Optional[torch.Tensor] = None, act=None, *,
                y: Optional[torch.Tensor] = None, rstd: Optional[torch.Tensor] = None,
                want_rstd: bool = True, stream=None):
    """General forward y = x * rstd * (w + weight_offset) * act(z) (the offset
    is added only when nonzero; act None means no gate and no z).  Returns
    (y, rstd)."""
    rows, width = _rows_width(x)
    a = act_code(act)
    if a == Act.NONE:
        if z is not None:
            raise ValueError("z given without a gate activation")
    else:
        _mat("z", z, x)
    _vec("w", w, width, x.device)
    y = torch.empty_like(x) if y is None else _mat("y", y, x)
    if rstd is None and want_rstd:
        rstd = torch.empty(rows, dtype=torch.float32, device=x.device)
    if rstd is not None:
        _vec("rstd", rstd, rows, x.device)
    with torch.cuda.device(x.device):
        check("rmsnorm_fwd",
              load().rmsnorm_fwd(rows, width, eps, weight_offset, int(a), _dt(x), _ptr(x), _ptr(z),
                                 _ptr(w), _ptr(y), _ptr(rstd), _stream(x, stream)))
    return y, rstd


def rmsnorm_add_fwd(x: torch.Tensor, r: torch.Tensor, w: torch.Tensor, eps: float = 1e-6,
                    weight_offset: float = 1.0, z: Optional[torch.Tensor] = None, act=None, *,
                    h: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
                    rstd: Optional[torch.Tensor] = None, want_rstd: bool = True, stream=None):
    """Residual-add forward: h = x + r (rounded once to x's dtype) and the norm
    of h.  Returns (h, y, rstd).  h may be x or r itself (in place)."""
    rows, width = _rows_width(x)
    a = act_code(act)
    _mat("r", r, x)
    if a == Act.NONE:
        if z is not None:
            raise ValueError("z given without a gate activation")
    else:
        _mat("z", z, x)
    _vec("w", w, width, x.device)
    h = torch.empty_like(x) if h is None else _mat("h", h, x)
    y = torch.empty_like(x) if y is None else _mat("y", y, x)
    if rstd is None and want_rstd:
        rstd = torch.empty(rows, dtype=torch.float32, device=x.device)
    if rstd is not None:
        _vec("rstd", rstd, rows, x.device)
    with torch.cuda.device(x.device):
        check("rmsnorm_add_fwd",
              load().rmsnorm_add_fwd(rows, width, eps, weight_offset, int(a), _dt(x), _ptr(x),
                                     _ptr(r), _ptr(z), _ptr(w), _ptr(h), _ptr(y), _ptr(rstd),
                                     _stream(x, stream)))
    return h, y, rstd


def rmsnorm_add_bwd(h: torch.Tensor, w: torch.Tensor, dy: torch.Tensor,
                    dh: Optional[torch.Tensor] = None, rstd: Optional[torch.Tensor] = None,
                    eps: float = 1e-6, weight_offset: float = 1.0,
                    z: Optional[torch.Tensor] = None, act=None, *,
                    row_mask: Optional[torch.Tensor] = None,
                    dx: Optional[torch.Tensor] = None, dz: Optional[torch.Tensor] = None,
                    dw: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                    stream=None):
    """Residual-add backward: the norm's gradient at h plus dh (the gradient
    of the residual output), the gradient of both x and r.  Returns (dx, dz, dw)."""
    rows, width = _rows_width(h)
    a = act_code(act)
    if a == Act.NONE:
        if z is not None or dz is not None:
            raise ValueError("z or dz given without a gate activation")
    else:
        _mat("z", z, h)
        dz = torch.empty_like(h) if dz is None else _mat("dz", dz, h)
    _vec("w", w, width, h.device)
    _mat("dy", dy, h)
    if dh is not None:
        _mat("dh", dh, h)
    if rstd is not None:
        _vec("rstd", rstd, rows, h.device)
    if row_mask is not None:
        if row_mask.dtype not in (torch.bool, torch.uint8) or tuple(row_mask.shape) != (rows,) \
                or row_mask.device != h.device or not row_mask.is_contiguous():
            raise ValueError(f"row_mask must be a contiguous bool/uint8 [{rows}] tensor on {h.device}")
        row_mask = row_mask.view(torch.uint8)
    dx = torch.empty_like(h) if dx is None else _mat("dx", dx, h)
    dw = torch.empty(width, dtype=torch.float32, device=h.device) if dw is None else \
        _vec("dw", dw, width, h.device)
    ws, nws = _ws(rows, width, h.device, ws)
    with torch.cuda.device(h.device):
        check("rmsnorm_add_bwd",
              load().rmsnorm_add_bwd(rows, width, eps, weight_offset, int(a), _dt(h), _ptr(h),
                                     _ptr(z), _ptr(w), _ptr(dy), _ptr(dh), _ptr(rstd),
                                     _ptr(row_mask), _ptr(dx), _ptr(dz), _ptr(dw), _ptr(ws), nws,
                                     _stream(h, stream)))
    return dx, dz, dw


def norm_fwd(x: torch.Tensor, w: torch.Tensor, eps: float = 1e-6, *,
             y: Optional[torch.Tensor] = None, rstd: Optional[torch.Tensor] = None,
             want_rstd: bool = True, stream=None):
    """Zero-centred RMSNorm forward.  Returns (y, rstd); rstd is None when
    want_rstd is False and none was passed."""
    rows, width = _rows_width(x)
    _vec("w", w, width, x.device)
    y = torch.empty_like(x) if y is None else _mat("y", y, x)
    if rstd is None and want_rstd:
        rstd = torch.empty(rows, dtype=torch.float32, device=x.device)
    if rstd is not None:
        _vec("rstd", rstd, rows, x.device)
    with torch.cuda.device(x.device):
        check("norm_fwd", load().norm_fwd(rows, width, eps, _dt(x), _ptr(x), _ptr(w), _ptr(y),
                                          _ptr(rstd), _stream(x, stream)))
    return y, rstd


def gated_norm_fwd(x: torch.Tensor, z: torch.Tensor, w: torch.Tensor, eps: float = 1e-6, *,
                   y: Optional[torch.Tensor] = None, rstd: Optional[torch.Tensor] = None,
                   want_rstd: bool = True, stream=None):
    """Gated RMSNorm forward.  Returns (y, rstd)."""
    rows, width = _rows_width(x)
    _mat("z", z, x)
    _vec("w", w, width, x.device)
    y = torch.empty_like(x) if y is None else _mat("y", y, x)
    if rstd is None and want_rstd:
        rstd = torch.empty(rows, dtype=torch.float32, device=x.device)
    if rstd is not None:
        _vec("rstd", rstd, rows, x.device)
    with torch.cuda.device(x.device):
        check("gated_norm_fwd",
              load().gated_norm_fwd(rows, width, eps, _dt(x), _ptr(x), _ptr(z), _ptr(w), _ptr(y),
                                    _ptr(rstd), _stream(x, stream)))
    return y, rstd


def _ws(rows, width, device, ws):
    if ws is None:
        ws = workspace(rows, width, device)
    if ws.device != device or not ws.is_contiguous():
        raise ValueError("ws must be a contiguous buffer on the tensors' device")
    return ws, ws.numel() * ws.element_size()


def rmsnorm_bwd(x: torch.Tensor, w: torch.Tensor, dy: torch.Tensor,
                rstd: Optional[torch.Tensor] = None, eps: float = 1e-6, weight_offset: float = 1.0,
                z: Optional[torch.Tensor] = None, act=None, *,
                row_mask: Optional[torch.Tensor] = None,
                dx: Optional[torch.Tensor] = None, dz: Optional[torch.Tensor] = None,
                dw: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                stream=None):
    """General backward.  Returns (dx, dz, dw); dz is None without a gate.
    rstd=None recomputes it.  row_mask ([rows] bool or uint8): rows where it is
    zero are left out of dw (dx and dz are still every row's)."""
    rows, width = _rows_width(x)
    a = act_code(act)
    if a == Act.NONE:
        if z is not None or dz is not None:
            raise ValueError("z or dz given without a gate activation")
    else:
        _mat("z", z, x)
        dz = torch.empty_like(x) if dz is None else _mat("dz", dz, x)
    _vec("w", w, width, x.device)
    _mat("dy", dy, x)
    if rstd is not None:
        _vec("rstd", rstd, rows, x.device)
    if row_mask is not None:
        if row_mask.dtype not in (torch.bool, torch.uint8) or tuple(row_mask.shape) != (rows,) \
                or row_mask.device != x.device or not row_mask.is_contiguous():
            raise ValueError(f"row_mask must be a contiguous bool/uint8 [{rows}] tensor on {x.device}")
        row_mask = row_mask.view(torch.uint8)
    dx = torch.empty_like(x) if dx is None else _mat("dx", dx, x)
    dw = torch.empty(width, dtype=torch.float32, device=x.device) if dw is None else \
        _vec("dw", dw, width, x.device)
    ws, nws = _ws(rows, width, x.device, ws)
    with torch.cuda.device(x.device):
        check("rmsnorm_bwd",
              load().rmsnorm_bwd(rows, width, eps, weight_offset, int(a), _dt(x), _ptr(x), _ptr(z),
                                 _ptr(w), _ptr(dy), _ptr(rstd), _ptr(row_mask), _ptr(dx),
                                 _ptr(dz), _ptr(dw), _ptr(ws), nws, _stream(x, stream)))
    return dx, dz, dw


def norm_bwd(x: torch.Tensor, w: torch.Tensor, dy: torch.Tensor,
             rstd: Optional[torch.Tensor] = None, eps: float = 1e-6, *,
             dx: Optional[torch.Tensor] = None, dw: Optional[torch.Tensor] = None,
             ws: Optional[torch.Tensor] = None, stream=None):
    """Zero-centred RMSNorm backward.  Returns (dx, dw).  rstd=None recomputes it."""
    rows, width = _rows_width(x)
    _vec("w", w, width, x.device)
    _mat("dy", dy, x)
    if rstd is not None:
        _vec("rstd", rstd, rows, x.device)
    dx = torch.empty_like(x) if dx is None else _mat("dx", dx, x)
    dw = torch.empty(width, dtype=torch.float32, device=x.device) if dw is None else \
        _vec("dw", dw, width, x.device)
    ws, nws = _ws(rows, width, x.device, ws)
    with torch.cuda.device(x.device):
        check("norm_bwd", load().norm_bwd(rows, width, eps, _dt(x), _ptr(x), _ptr(w), _ptr(dy),
                                          _ptr(rstd), _ptr(dx), _ptr(dw), _ptr(ws), nws,
                                          _stream(x, stream)))
    return dx, dw


def gated_norm_bwd(x: torch.Tensor, z: torch.Tensor, w: torch.Tensor, dy: torch.Tensor,
                   rstd: Optional[torch.Tensor] = None, eps: float = 1e-6, *,
                   dx: Optional[torch.Tensor] = None, dz: Optional[torch.Tensor] = None,
                   dw: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                   stream=None):
    """Gated RMSNorm backward.  Returns (dx, dz, dw).  rstd=None recomputes it."""
    rows, width = _rows_width(x)
    _mat("z", z, x)
    _vec("w", w, width, x.device)
    _mat("dy", dy, x)
    if rstd is not None:
        _vec("rstd", rstd, rows, x.device)
    dx = torch.empty_like(x) if dx is None else _mat("dx", dx, x)
    dz = torch.empty_like(x) if dz is None else _mat("dz", dz, x)
    dw = torch.empty(width, dtype=torch.float32, device=x.device) if dw is None else \
        _vec("dw", dw, width, x.device)
    ws, nws = _ws(rows, width, x.device, ws)
    with torch.cuda.device(x.device):
        check("gated_norm_bwd",
              load().gated_norm_bwd(rows, width, eps, _dt(x), _ptr(x), _ptr(z), _ptr(w), _ptr(dy),
                                    _ptr(rstd), _ptr(dx), _ptr(dz), _ptr(dw), _ptr(ws), nws,
                                    _stream(x, stream)))
    return dx, dz, dw


def rmsnorm_bwd_chunks(x: torch.Tensor, w: torch.Tensor, dy: torch.Tensor,
                       rstd: Optional[torch.Tensor] = None, eps: float = 1e-6,
                       weight_offset: float = 1.0, z: Optional[torch.Tensor] = None, act=None, *,
                       row_mask: Optional[torch.Tensor] = None,
                       dx: Optional[torch.Tensor] = None, dz: Optional[torch.Tensor] = None,
                       dw_chunks: Optional[torch.Tensor] = None,
                       ws: Optional[torch.Tensor] = None, stream=None):
    """rmsnorm_bwd returning dw's 256-row chunk partials [ceil(rows/256), width]
    in place of dw (for the data-parallel fold).  Returns (dx, dz, dw_chunks)."""
    rows, width = _rows_width(x)
    a = act_code(act)
    if a == Act.NONE:
        if z is not None or dz is not None:
            raise ValueError("z or dz given without a gate activation")
    else:
        _mat("z", z, x)
        dz = torch.empty_like(x) if dz is None else _mat("dz", dz, x)
    _vec("w", w, width, x.device)
    _mat("dy", dy, x)
    if rstd is not None:
        _vec("rstd", rstd, rows, x.device)
    if row_mask is not None:
        if row_mask.dtype not in (torch.bool, torch.uint8) or tuple(row_mask.shape) != (rows,) \
                or row_mask.device != x.device or not row_mask.is_contiguous():
            raise ValueError(f"row_mask must be a contiguous bool/uint8 [{rows}] tensor on {x.device}")
        row_mask = row_mask.view(torch.uint8)
    nc = int(load().rmsnorm_bwd_chunk_count(rows))
    dx = torch.empty_like(x) if dx is None else _mat("dx", dx, x)
    if dw_chunks is None:
        dw_chunks = torch.empty(nc, width, dtype=torch.float32, device=x.device)
    elif (dw_chunks.device != x.device or dw_chunks.dtype != torch.float32
          or tuple(dw_chunks.shape) != (nc, width) or not dw_chunks.is_contiguous()):
        raise ValueError(f"dw_chunks must be a contiguous fp32 [{nc}, {width}] tensor on {x.device}")
    ws, nws = _ws(rows, width, x.device, ws)
    with torch.cuda.device(x.device):
        check("rmsnorm_bwd_chunks",
              load().rmsnorm_bwd_chunks(rows, width, eps, weight_offset, int(a), _dt(x), _ptr(x),
                                        _ptr(z), _ptr(w), _ptr(dy), _ptr(rstd), _ptr(row_mask),
                                        _ptr(dx), _ptr(dz), _ptr(dw_chunks), _ptr(ws), nws,
                                        _stream(x, stream)))
    return dx, dz, dw_chunks


def rn_fold_tree(partials: torch.Tensor, *, out: Optional[torch.Tensor] = None,
                 ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """The level-by-level pairwise tree over the rows of a [n, width] fp32 CUDA
    tensor (any n >= 1); returns the [width] result."""
    if partials.dim() != 2 or partials.dtype != torch.float32 or not partials.is_cuda \
            or not partials.is_contiguous():
        raise ValueError("partials must be a contiguous fp32 CUDA tensor [n, width]")
    n, width = int(partials.shape[0]), int(partials.shape[1])
    out = torch.empty(width, dtype=torch.float32, device=partials.device) if out is None else \
        _vec("out", out, width, partials.device)
    if ws is None:
        nb = int(load().rn_fold_tree_workspace_bytes(n, width))
        ws = torch.empty(max(nb, 16), dtype=torch.uint8, device=partials.device)
    with torch.cuda.device(partials.device):
        check("rn_fold_tree", load().rn_fold_tree(n, width, _ptr(partials), _ptr(out), _ptr(ws),
                                                  ws.numel() * ws.element_size(),
                                                  _stream(partials, stream)))
    return out


def rn_fold_rows(partials: torch.Tensor, *, out: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
    """Joins the rows of a [n, width] fp32 CUDA tensor of dw partials with the
    backward's pairwise tree; returns the [width] result."""
    if partials.dim() != 2 or partials.dtype != torch.float32 or not partials.is_cuda \
            or not partials.is_contiguous():
        raise ValueError("partials must be a contiguous fp32 CUDA tensor [n, width]")
    n, width = int(partials.shape[0]), int(partials.shape[1])
    out = torch.empty(width, dtype=torch.float32, device=partials.device) if out is None else \
        _vec("out", out, width, partials.device)
    with torch.cuda.device(partials.device):
        check("rn_fold_rows", load().rn_fold_rows(n, width, _ptr(partials), _ptr(out),
                                                  _stream(partials, stream)))
    return out


def rn_describe(width: int, dtype=torch.bfloat16) -> str:
    """The provenance string for (width, dtype): kernels, team shape, reduction
    order, dw tree, accumulator; "unsupported" for an invalid pair."""
    if isinstance(dtype, torch.dtype):
        if dtype not in _DT:
            return "unsupported"
        dt = _DT[dtype]
    else:
        dt = int(dtype)
    return load().rn_describe(width, dt).decode()


def rn_test_set_geometry(max_ctas: int = 0, leaves_per_cta: int = 0, fold_rows: int = 0) -> None:
    check("rn_test_set_geometry", load().rn_test_set_geometry(max_ctas, leaves_per_cta, fold_rows))


def rn_test_set_validate_only(on: bool) -> None:
    load().rn_test_set_validate_only(1 if on else 0)
