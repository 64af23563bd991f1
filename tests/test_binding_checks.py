"""Host-side checks of the torch helpers in block_scaled_microscaling_b200.mxq, on CPU.

The C entry points take bare pointers; the helpers refuse, before any call, a host tensor (the
library computes on the GPU only: no CPU path) and a caller-supplied buffer that is
non-contiguous or too small for the shape (a kernel would otherwise read or write past the
tensor's end). Host tensors wrapped to report themselves as CUDA tensors let the size checks run
here; every case fails a check before the library or the CUDA runtime is reached (were one to
pass, torch.cuda.current_stream() would raise on this GPU-less host, not a ValueError).
"""
import pytest
import torch

from block_scaled_microscaling_b200 import build as mxq_build
from block_scaled_microscaling_b200 import mxq


@pytest.fixture(scope="module", autouse=True)
def library():
    # the size checks use the library's host-only size queries
    mxq_build.build()
    return mxq.lib()


class FakeCuda:
    """A host tensor that reports is_cuda = True; everything else is the tensor's own."""
    is_cuda = True

    def __init__(self, t):
        self.t = t

    def __getattr__(self, name):
        return getattr(self.t, name)


def u8(n):
    return FakeCuda(torch.zeros(n, dtype=torch.uint8))


def bf16(*shape):
    return FakeCuda(torch.zeros(shape, dtype=torch.bfloat16))


def f32(*shape):
    return FakeCuda(torch.zeros(shape, dtype=torch.float32))


def test_host_tensors_are_refused():
    x = torch.zeros((4, 64), dtype=torch.bfloat16)
    s = torch.zeros((4, 64), dtype=torch.float32)
    for call in [lambda: mxq.quantize(x, "mxfp8"),
                 lambda: mxq.dequantize(torch.zeros(512, dtype=torch.uint8), torch.zeros(8, dtype=torch.uint8),
                                        "mxfp8", (4, 64)),
                 lambda: mxq.fake_quantize(x, "axs6"),
                 lambda: mxq.exp_quantize(s, "mxfp4"),
                 lambda: mxq.exp_free_quantize(s),
                 lambda: mxq.quantize_mma(x, "mxfp8"),
                 lambda: mxq.swizzle_scales(torch.zeros((4, 2), dtype=torch.uint8)),
                 lambda: mxq.quantize_grouped([x], "mxfp8"),
                 lambda: mxq.quantize_cols(torch.zeros((64, 32), dtype=torch.bfloat16), "mxfp8"),
                 lambda: mxq.dequantize_cols(torch.zeros(512, dtype=torch.uint8), torch.zeros(8, dtype=torch.uint8),
                                             "mxfp8", (64, 8)),
                 lambda: mxq.quantize_exmy(x, 3, 3),
                 lambda: mxq.dequantize_exmy(torch.zeros(448, dtype=torch.uint8), torch.zeros(8, dtype=torch.uint8),
                                             3, 3, (4, 64)),
                 lambda: mxq.fake_quantize_exmy(x, 3, 3),
                 lambda: mxq.batch([("fake_quantize", "axs6", x, x)])]:
        with pytest.raises(ValueError, match="CUDA tensor"):
            call()


@pytest.mark.parametrize("fmt,nc,ns", [("axs6", 4 * 2 * 24, 4 * 2 * 2), ("mxfp6_e2m3", 192, 8),
                                      ("mxfp8", 256, 8), ("mxfp4", 128, 8)])
def test_quantize_output_sizes(fmt, nc, ns):
    x = bf16(4, 64)
    with pytest.raises(ValueError, match=f"codes holds {nc - 1} bytes, the call needs {nc}"):
        mxq.quantize(x, fmt, codes=u8(nc - 1), scales=u8(ns))
    with pytest.raises(ValueError, match=f"scales holds {ns - 1} bytes, the call needs {ns}"):
        mxq.quantize(x, fmt, codes=u8(nc), scales=u8(ns - 1))
    wide = FakeCuda(torch.zeros((nc, 2), dtype=torch.uint8)[:, :1])  # enough bytes, not contiguous
    with pytest.raises(ValueError, match="codes must be contiguous"):
        mxq.quantize(x, fmt, codes=wide, scales=u8(ns))
    with pytest.raises(ValueError, match="codes holds"):
        mxq.exp_quantize(f32(4, 64), fmt, codes=u8(nc - 1), scales=u8(ns))
    with pytest.raises(ValueError, match="scales holds"):
        mxq.quantize_grouped([x, bf16(2, 64)], fmt, outs=[(u8(nc), u8(ns)), (u8(nc // 2), u8(ns // 2 - 1))])
    with pytest.raises(ValueError, match="codes holds"):
        mxq.batch([("quantize", fmt, x, u8(nc - 1), u8(ns))])


def test_dequantize_input_and_output_checks():
    # a shape larger than the codes would make the kernel read past them
    with pytest.raises(ValueError, match="codes holds 256 bytes, the call needs 512"):
        mxq.dequantize(u8(256), u8(16), "mxfp8", (8, 64))
    with pytest.raises(ValueError, match="scales holds 15 bytes, the call needs 16"):
        mxq.dequantize(u8(512), u8(15), "mxfp8", (8, 64))
    out = FakeCuda(torch.zeros((64, 16), dtype=torch.bfloat16).t())  # (16, 64), not contiguous
    with pytest.raises(ValueError, match="out must be contiguous"):
        mxq.dequantize(u8(16 * 64), u8(32), "mxfp8", None, out=out)
    with pytest.raises(ValueError, match="codes holds"):
        mxq.batch([("dequantize", "mxfp6_e3m2", u8(100), u8(8), bf16(4, 64))])
    with pytest.raises(ValueError, match="codes holds"):
        mxq.dequantize_cols(u8(511), u8(16), "mxfp8", (64, 8))
    with pytest.raises(ValueError, match="out must be 2-D"):
        mxq.dequantize_cols(u8(512), u8(16), "mxfp8", None, out=bf16(2, 32, 8))


def test_fake_quantize_output_must_match():
    x = bf16(4, 64)
    with pytest.raises(ValueError, match="x's dtype and size"):
        mxq.fake_quantize(x, "axs6", out=f32(4, 64))
    with pytest.raises(ValueError, match="x's dtype and size"):
        mxq.fake_quantize(x, "axs6", out=bf16(4, 32))
    with pytest.raises(ValueError, match="x's dtype and size"):
        mxq.fake_quantize_exmy(x, 2, 3, out=bf16(3, 64))
    with pytest.raises(ValueError, match="x's dtype and size"):
        mxq.batch([("fake_quantize", "axs6", x, bf16(2, 64))])


def test_other_entry_points_sizes():
    with pytest.raises(ValueError, match="codes holds 127 bytes, the call needs 128"):
        mxq.exp_free_quantize(f32(4, 64), codes=u8(127), scales=u8(8))
    with pytest.raises(ValueError, match="scales holds 511 bytes, the call needs 512"):
        mxq.quantize_mma(bf16(4, 64), "mxfp8", codes=u8(256), scales=u8(511))  # 128 x 4 tile, padded
    with pytest.raises(ValueError, match="out holds 511 bytes, the call needs 512"):
        mxq.swizzle_scales(FakeCuda(torch.zeros((4, 2), dtype=torch.uint8)), out=u8(511))
    # quantize_cols writes the transpose: codes [cols, rows/32 * P]
    with pytest.raises(ValueError, match="scales holds 7 bytes, the call needs 8"):
        mxq.quantize_cols(bf16(32, 8), "mxfp8", codes=u8(256), scales=u8(7))
    # eXmY: a block's payload is W 32-bit words
    with pytest.raises(ValueError, match="codes holds 223 bytes, the call needs 224"):
        mxq.quantize_exmy(bf16(4, 64), 3, 3, codes=u8(223), scales=u8(8))
    with pytest.raises(ValueError, match="scales holds 7 bytes, the call needs 8"):
        mxq.dequantize_exmy(u8(224), u8(7), 3, 3, (4, 64))
    with pytest.raises(ValueError, match="one \\(codes, scales\\) pair per tensor"):
        mxq.quantize_grouped([bf16(4, 64), bf16(4, 64)], "mxfp8", outs=[(u8(256), u8(8))])


def test_unknown_format_is_a_value_error():
    with pytest.raises(ValueError, match="unknown format"):
        mxq.quantize(bf16(4, 64), "mxfp5")
