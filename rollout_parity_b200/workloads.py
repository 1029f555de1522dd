"""Seeded synthetic inputs for the norm operators.

This module draws random numbers, rounds them once to the stored dtype and lays
rows out; it does no normalisation arithmetic.  The CUDA path and the fp64
checker both consume exactly the bits it produces (the checker widens them to
fp64 exactly), so a disagreement between them can never come from the inputs.

Shapes and distributions follow the workloads the gated-RMSNorm PR measures
("[WS1][CUDA][Qwen3-Next] Gated RMSNorm CUDA kernel for the GDN block", sections
"Prior art & reuse decision" and "Comparison charts": bf16, head dim 128,
262144 rows) plus the decoder-norm widths of the same model (hidden 2048) and a
large-width stress case.

Recipe (every tensor has its own child stream of ``SeedSequence(seed)``):
  * x, z, dy: standard normal drawn in float32, then rounded to the stored
    dtype (bf16 round-to-nearest-even through torch) -- or kept as float32.
  * w: float32, ``mean + std * N(0,1)``; it is always fp32 [width].
  * outliers: ``max(1, round(frac * width))`` channel indices drawn without
    replacement; those columns of x, z and dy are multiplied by ``scale``
    (before the dtype rounding).
  * ragged packing: sequence lengths uniform on [1, max_len] drawn until the
    rows would exceed ``rows``; the last one is cut to fill exactly ``rows``.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import numpy as np
import torch

DTYPES = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}
# the operator's (activation, weight offset) by op name; "general" takes both
# from the caller
OP_DEFAULTS = {"norm": ("none", 1.0), "gated": ("silu", 0.0)}

# child-stream ids of SeedSequence(seed).spawn(...)
_X, _Z, _DY, _W, _OUTLIER, _PACK = range(6)


@dataclasses.dataclass
class Workload:
    """One batch of synthetic inputs (host tensors, stored dtype)."""

    name: str
    op: str                     # "norm" (zero-centred), "gated" or "general"
    rows: int
    width: int
    dtype: str                  # "bf16", "f16" or "f32"
    eps: float
    x: torch.Tensor             # [rows, width], stored dtype, CPU
    z: Optional[torch.Tensor]   # present when there is a gate
    dy: torch.Tensor            # upstream gradient, stored dtype
    w: torch.Tensor             # [width] fp32
    seq_lens: Optional[List[int]] = None
    outlier_channels: Optional[List[int]] = None
    act: Optional[str] = None   # gate activation: "none", "silu" or "sigmoid"
    weight_offset: Optional[float] = None   # added to w when nonzero

    def __post_init__(self):
        # "norm" and "gated" fix both; "general" must name them
        if self.op in OP_DEFAULTS:
            act, off = OP_DEFAULTS[self.op]
            self.act = act if self.act is None else self.act
            self.weight_offset = off if self.weight_offset is None else self.weight_offset
        assert self.act in ("none", "silu", "sigmoid") and self.weight_offset is not None

    @property
    def gated(self) -> bool:
        return self.act != "none"

    def to(self, device) -> "Workload":
        f = lambda t: None if t is None else t.to(device)
        return dataclasses.replace(self, x=f(self.x), z=f(self.z), dy=f(self.dy), w=f(self.w))


def _streams(seed: int):
    return [np.random.default_rng(s) for s in np.random.SeedSequence(seed).spawn(6)]


def _normal(rng, shape) -> np.ndarray:
    return rng.standard_normal(shape, dtype=np.float32)


def _store(a: np.ndarray, dtype: str) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(DTYPES[dtype])


def make(op: str, rows: int, width: int, dtype: str = "bf16", *, seed: int = 0,
         eps: float = 1e-6, w_mean: float = 1.0, w_std: float = 0.1,
         outlier_frac: float = 0.0, outlier_scale: float = 50.0,
         outlier_round: str = "nearest", name: str = "", act: Optional[str] = None,
         weight_offset: Optional[float] = None) -> Workload:
    """Draw one workload.  ``op`` is "norm" (no gate, offset 1), "gated" (silu,
    offset 0) or "general" (``act`` and ``weight_offset`` given)."""
    assert op in ("norm", "gated", "general") and dtype in DTYPES
    if op == "general":
        assert act in ("none", "silu", "sigmoid") and weight_offset is not None
    else:
        assert act is None and weight_offset is None
        act, weight_offset = OP_DEFAULTS[op]
    rx, rz, rdy, rw, ro, _ = _streams(seed)
    x = _normal(rx, (rows, width))
    z = _normal(rz, (rows, width)) if act != "none" else None
    dy = _normal(rdy, (rows, width))
    w = (np.float32(w_mean) + np.float32(w_std) * _normal(rw, (width,))).astype(np.float32)
    chans = None
    if outlier_frac > 0.0:
        k = outlier_frac * width
        n = int(np.ceil(k)) if outlier_round == "ceil" else int(round(k))
        n = max(1, min(width, n))
        chans = sorted(int(c) for c in ro.choice(width, size=n, replace=False))
        for a in (x, z, dy):
            if a is not None:
                a[:, chans] *= np.float32(outlier_scale)
    return Workload(name=name or f"{op}_{rows}x{width}_{dtype}", op=op, rows=rows,
                    width=width, dtype=dtype, eps=eps, x=_store(x, dtype),
                    z=None if z is None else _store(z, dtype), dy=_store(dy, dtype),
                    w=torch.from_numpy(w), outlier_channels=chans, act=act,
                    weight_offset=float(weight_offset))


def ragged_lengths(total_rows: int, max_len: int, seed: int = 0) -> List[int]:
    """Sequence lengths ~ U[1, max_len] until ``total_rows`` is filled exactly."""
    rng = _streams(seed)[_PACK]
    lens, used = [], 0
    while used < total_rows:
        n = int(rng.integers(1, max_len + 1))
        n = min(n, total_rows - used)
        lens.append(n)
        used += n
    return lens


# The five workloads the benchmark and parity tests are built around.  Each is a
# function so that nothing large is drawn at import time.
def cfg_small_f32(seed: int = 0) -> Workload:
    """Zero-centred, 64 x 128 fp32, w ~ N(0, 0.1): the small exact-check case."""
    return make("norm", 64, 128, "f32", seed=seed, w_mean=0.0, w_std=0.1,
                name="norm_64x128_f32")


def cfg_gated_4k(seed: int = 0) -> Workload:
    """Gated, 4096 x 128 bf16, w ~ N(1, 0.1)."""
    return make("gated", 4096, 128, "bf16", seed=seed, name="gated_4096x128_bf16")


def cfg_packed_2048(seed: int = 0) -> Workload:
    """Zero-centred, 16384 x 2048 bf16, rows packed from ragged sequences."""
    wl = make("norm", 16384, 2048, "bf16", seed=seed, w_mean=0.0, w_std=0.1,
              name="norm_16384x2048_bf16_packed")
    wl.seq_lens = ragged_lengths(16384, 2048, seed)
    return wl


def cfg_gated_heads(seed: int = 0, outlier_round: str = "nearest") -> Workload:
    """Gated, 262144 rows (8192 tokens x 32 heads, row = token*32 + head) x 128
    bf16, with 1% of channels scaled x50 in x, z and dy."""
    return make("gated", 262144, 128, "bf16", seed=seed, outlier_frac=0.01,
                outlier_scale=50.0, outlier_round=outlier_round,
                name="gated_262144x128_bf16_outliers")


def cfg_wide_8192(seed: int = 0, rows: int = 32768) -> Workload:
    """Zero-centred, 32768 x 8192 bf16, w ~ N(0, 0.1)."""
    return make("norm", rows, 8192, "bf16", seed=seed, w_mean=0.0, w_std=0.1,
                name=f"norm_{rows}x8192_bf16")


CONFIGS = {
    "norm_64x128_f32": cfg_small_f32,
    "gated_4096x128_bf16": cfg_gated_4k,
    "norm_16384x2048_bf16_packed": cfg_packed_2048,
    "gated_262144x128_bf16_outliers": cfg_gated_heads,
    "norm_32768x8192_bf16": cfg_wide_8192,
}
SWEEP_8192 = (1, 7, 128, 4096, 32768)


# Variants of the operator (PR #468 Summary: activation silu or sigmoid, weight
# offset 0 or 1, fp32/fp16/bf16, H in {128, 2048, 5120}) at benchmark sizes.
def cfg_sigmoid_heads(seed: int = 0) -> Workload:
    """The 262144 x 128 bf16 head layout with outliers, sigmoid gate, offset 0."""
    return make("general", 262144, 128, "bf16", seed=seed, outlier_frac=0.01,
                outlier_scale=50.0, act="sigmoid", weight_offset=0.0,
                name="sigmoid_262144x128_bf16_outliers")


def cfg_f16_heads(seed: int = 0) -> Workload:
    """The 262144 x 128 head layout with outliers in fp16, silu gate, offset 0."""
    return make("general", 262144, 128, "f16", seed=seed, outlier_frac=0.01,
                outlier_scale=50.0, act="silu", weight_offset=0.0,
                name="silu_262144x128_f16_outliers")


def cfg_norm_5120(seed: int = 0) -> Workload:
    """Zero-centred (offset 1, no gate), 16384 x 5120 bf16, w ~ N(0, 0.1)."""
    return make("general", 16384, 5120, "bf16", seed=seed, w_mean=0.0, w_std=0.1,
                act="none", weight_offset=1.0, name="norm_16384x5120_bf16")


def cfg_sigmoid_f32_2048(seed: int = 0) -> Workload:
    """Sigmoid gate with offset 1, 16384 x 2048 fp32, w ~ N(0, 0.1)."""
    return make("general", 16384, 2048, "f32", seed=seed, w_mean=0.0, w_std=0.1,
                act="sigmoid", weight_offset=1.0, name="sigmoid_off1_16384x2048_f32")


def cfg_qk_norm(width: int, rows: int, seed: int = 0) -> Workload:
    """Per-head RMSNorm of q/k rows at head dim 256 or 512 (offset 1, no gate),
    bf16, w ~ N(0, 0.1): rows = tokens x heads."""
    return make("general", rows, width, "bf16", seed=seed, w_mean=0.0, w_std=0.1, act="none",
                weight_offset=1.0, name=f"qk_norm_{rows}x{width}_bf16")


def cfg_gated_wide(width: int, seed: int = 0) -> Workload:
    """The gated operator (silu, offset 0) on 16384 rows at a model width, bf16,
    w ~ N(1, 0.1): the pages' rstd matrix widths 2048 and 5120 with the gate."""
    return make("general", 16384, width, "bf16", seed=seed, w_mean=1.0, w_std=0.1, act="silu",
                weight_offset=0.0, name=f"silu_16384x{width}_bf16")


VARIANTS = {
    "sigmoid_262144x128_bf16_outliers": cfg_sigmoid_heads,
    "silu_262144x128_f16_outliers": cfg_f16_heads,
    "norm_16384x5120_bf16": cfg_norm_5120,
    "sigmoid_off1_16384x2048_f32": cfg_sigmoid_f32_2048,
    "qk_norm_131072x256_bf16": lambda seed=0: cfg_qk_norm(256, 131072, seed),
    "qk_norm_65536x512_bf16": lambda seed=0: cfg_qk_norm(512, 65536, seed),
    "silu_16384x2048_bf16": lambda seed=0: cfg_gated_wide(2048, seed),
    "silu_16384x5120_bf16": lambda seed=0: cfg_gated_wide(5120, seed),
}
ALL = {**CONFIGS, **VARIANTS}


def as_f64(t: Optional[torch.Tensor]) -> Optional[np.ndarray]:
    """Widen stored values to fp64 exactly (bf16, fp16 and fp32 embed in fp64)."""
    if t is None:
        return None
    return t.detach().to("cpu").to(torch.float64).numpy()
