"""block_scaled_microscaling_b200 -- libmxq, block-scaled shared-exponent
quantization (AXS-6, MXFP6 E2M3/E3M2, MXFP8 E4M3, MXFP4 E2M1) as hand-written
CUDA kernels for NVIDIA B200 (sm_100a) behind a C ABI (include/mxq.h).

    from block_scaled_microscaling_b200 import quantize, dequantize, fake_quantize
    codes, scales = quantize(w_bf16, "mxfp6_e2m3")
    w2 = dequantize(codes, scales, "mxfp6_e2m3", w_bf16.shape)
    g_q = fake_quantize(g_fp32, "axs6")          # quantize + dequantize, one pass
"""
from .mxq import (EXPORTS, FORMATS, MXQError, batch, check_device, dequantize, dequantize_cols, dequantize_exmy,
                  exp_free_quantize, exp_quantize, fake_quantize, fake_quantize_exmy, lib, quantize, quantize_cols,
                  quantize_exmy, quantize_grouped, quantize_mma, swizzle_scales)


def fake_quantize_ste(x, fmt="axs6", block_size=32):
    """Differentiable fake-quantize: forward = fused kernel, backward = identity (STE)."""
    from .ste import fake_quantize_ste as f
    return f(x, fmt, block_size)


__all__ = ["quantize", "dequantize", "fake_quantize", "fake_quantize_ste", "exp_quantize", "exp_free_quantize",
           "quantize_grouped", "check_device",
           "quantize_cols", "dequantize_cols", "quantize_exmy", "dequantize_exmy", "fake_quantize_exmy",
           "quantize_mma", "swizzle_scales", "batch", "MXQError", "FORMATS", "lib", "EXPORTS"]
