"""Straight-through estimator (STE) for the fused fake-quantize.

"AXS-6: Adaptive eXponent Sharing", overview and Key Advantages: the format
trains with simple straight-through gradient estimation. Forward is the
fused fake-quantize kernel (quantize then dequantize in one pass, on the GPU);
backward passes the incoming gradient through unchanged (d fq(x)/dx := 1).
"""
import torch

from . import mxq


class FakeQuantizeSTE(torch.autograd.Function):
    """y = fake_quantize(x, fmt); dy/dx = identity."""

    @staticmethod
    def forward(ctx, x, fmt="axs6"):
        return mxq.fake_quantize(x.contiguous(), fmt)

    @staticmethod
    def backward(ctx, grad_out):
        return grad_out, None


def fake_quantize_ste(x, fmt="axs6", block_size=32):
    """Differentiable fused fake-quantize (blocks of 32 along the last dimension)."""
    if block_size != 32:
        raise mxq.MXQError(4, f"block_size={block_size}")
    return FakeQuantizeSTE.apply(x, fmt)
