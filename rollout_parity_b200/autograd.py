"""torch.autograd wrappers over the C entry points (forward saves rstd; the
backward reuses it, so the statistic the gradient sees is the forward's)."""
from __future__ import annotations

import torch

from . import ops


class ZeroCentredRMSNorm(torch.autograd.Function):
    """y = x * rstd * (1 + w); x [rows, width] bf16/fp32, w fp32 [width]."""

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
    """y = x * rstd * w * silu(z); x, z [rows, width] bf16/fp32, w fp32 [width]."""

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


def zero_centred_rms_norm(x, w, eps=1e-6):
    return ZeroCentredRMSNorm.apply(x, w, eps)


def gated_rms_norm(x, z, w, eps=1e-6):
    return GatedRMSNorm.apply(x, z, w, eps)
