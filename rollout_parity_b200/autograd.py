"""torch.autograd wrappers over the C entry points (the forward saves rstd; the
backward reuses it, so the statistic the gradient sees is the forward's)."""
from __future__ import annotations

import torch

from . import ops


class ZeroCentredRMSNorm(torch.autograd.Function):
    """y = x * rstd * (1 + w); x [rows, width] bf16/fp16/fp32, w fp32 [width]."""

    @staticmethod
    def forward(ctx, x, w, eps=1e-6):
        y, rstd = ops.norm_fwd(x, w, eps)
        ctx.save_for_backward(x, w, rstd)
        ctx.eps = eps
        return y

    @staticmethod
    def backward(ctx, dy):
        x, w, rstd = ctx.saved_tensors
        dx, dw = ops.norm_bwd(x, w, dy.contiguous(), rstd, ctx.eps)
        return dx, dw, None


class GatedRMSNorm(torch.autograd.Function):
    """y = x * rstd * w * silu(z); x, z [rows, width] bf16/fp16/fp32, w fp32 [width]."""

    @staticmethod
    def forward(ctx, x, z, w, eps=1e-6):
        y, rstd = ops.gated_norm_fwd(x, z, w, eps)
        ctx.save_for_backward(x, z, w, rstd)
        ctx.eps = eps
        return y

    @staticmethod
    def backward(ctx, dy):
        x, z, w, rstd = ctx.saved_tensors
        dx, dz, dw = ops.gated_norm_bwd(x, z, w, dy.contiguous(), rstd, ctx.eps)
        return dx, dz, dw, None


class RMSNorm(torch.autograd.Function):
    """y = x * rstd * (w + weight_offset) * act(z) (the offset added only when
    nonzero); act None/"none" (no z), "silu"/"swish" or "sigmoid"."""

    @staticmethod
    def forward(ctx, x, w, z=None, eps=1e-6, weight_offset=1.0, act=None):
        y, rstd = ops.rmsnorm_fwd(x, w, eps, weight_offset, z, act)
        ctx.save_for_backward(x, w, rstd, *(() if z is None else (z,)))
        ctx.eps, ctx.weight_offset, ctx.act, ctx.gated = eps, weight_offset, act, z is not None
        return y

    @staticmethod
    def backward(ctx, dy):
        saved = ctx.saved_tensors
        x, w, rstd = saved[:3]
        z = saved[3] if ctx.gated else None
        dx, dz, dw = ops.rmsnorm_bwd(x, w, dy.contiguous(), rstd, ctx.eps, ctx.weight_offset, z,
                                     ctx.act)
        return dx, dw, dz, None, None, None


def zero_centred_rms_norm(x, w, eps=1e-6):
    return ZeroCentredRMSNorm.apply(x, w, eps)


def gated_rms_norm(x, z, w, eps=1e-6):
    return GatedRMSNorm.apply(x, z, w, eps)


def rms_norm(x, w, z=None, eps=1e-6, weight_offset=1.0, act=None):
    return RMSNorm.apply(x, w, z, eps, weight_offset, act)
