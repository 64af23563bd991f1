"""GPU: E8M0 scales in the tile layout of the block-scaled tensor-core MMA.

- mxq_quantize_mma: codes bit-identical to mxq_quantize and to the oracle; scales equal the
  oracle's layout of the oracle's scales, padding bytes zero (buffers are pre-filled with 0xEE).
- mxq_swizzle_scales: equal to the oracle's layout for ragged and large shapes.
- consumer check: MXFP8 E4M3 codes + tiled scales given to cuBLAS's block-scaled GEMM
  (torch._scaled_mm) give the product of the oracle-dequantized operands, and the same codes with
  row-major (untiled) scales do not -- the check can tell the layouts apart. (This torch build
  accepts packed FP4 operands only with E4M3 scales per 16 values, not MXFP4's E8M0 per 32, so
  the MXFP4 layout is checked against the oracle only; it is the same scale layout.)
The layout itself is not on the pages ("Sonar: Online MXFP6", Current limits: converted weights
feed block-scaled GEMMs with dimensions in multiples of 128)."""
import numpy as np
import pytest

import oracle
import synthetic

torch = pytest.importorskip("torch")
from block_scaled_microscaling_b200 import mxq  # noqa: E402

pytestmark = pytest.mark.gpu

E8M0_FMTS = ["mxfp6_e2m3", "mxfp6_e3m2", "mxfp8", "mxfp4"]
SHAPES = [(1, 32), (127, 96), (128, 128), (129, 160), (300, 1056), (256, 4096)]


def spread_values(rows, cols, seed, dtype):
    """N(0, 1) values, each block of 32 times 2^e with e uniform in [-6, 6] (so a scale put in the
    wrong place changes the result by a power of two)."""
    x = synthetic.gaussian((rows, cols), 1.0, seed, 0, "f32").reshape(-1, 32)
    e = np.asarray(synthetic.uniform_ints(seed, 7, x.shape[0], 13), dtype=np.int64) - 6
    x = (x * np.ldexp(1.0, e)[:, None].astype(np.float32)).astype(np.float32).reshape(rows, cols)
    return x if dtype == "f32" else synthetic.f32_to_bf16_bits(x)


def dev(x):
    if x.dtype == np.float32:
        return torch.from_numpy(np.ascontiguousarray(x)).cuda()
    return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("fmt", E8M0_FMTS)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("shape", SHAPES)
def test_quantize_mma_matches_oracle(fmt, dtype, shape):
    rows, cols = shape
    x = spread_values(rows, cols, rows * 7 + cols, dtype)
    xd = dev(x)
    want_codes, want_scales = oracle.quantize(x, fmt)
    want_tiled = oracle.swizzle_scales(want_scales)
    scales = torch.full((mxq.mxq_mma_scales_bytes(rows, cols),), 0xEE, dtype=torch.uint8, device="cuda")
    codes, scales = mxq.quantize_mma(xd, fmt, scales=scales)
    plain_codes, _ = mxq.quantize(xd, fmt)
    torch.cuda.synchronize()
    assert scales.numel() == want_tiled.size
    assert np.array_equal(codes.cpu().numpy(), want_codes)
    assert torch.equal(codes, plain_codes)
    assert np.array_equal(scales.cpu().numpy(), want_tiled)


@pytest.mark.parametrize("rows,kb", [(1, 1), (3, 5), (127, 3), (128, 4), (129, 9), (1000, 33), (4096, 128),
                                     (16384, 256), (300, 1028)])
def test_swizzle_scales_matches_oracle(rows, kb):
    s = np.asarray(synthetic.uniform_ints(rows + 17 * kb, 3, rows * kb, 256), dtype=np.uint8).reshape(rows, kb)
    out = torch.full((mxq.mxq_mma_scales_bytes(rows, 32 * kb),), 0xEE, dtype=torch.uint8, device="cuda")
    got = mxq.swizzle_scales(torch.from_numpy(s).cuda(), out=out)
    assert np.array_equal(got.cpu().numpy(), oracle.swizzle_scales(s))


def test_swizzle_after_quantize_equals_fused():
    x = dev(spread_values(384, 2048, 5, "bf16"))
    _, plain = mxq.quantize(x, "mxfp8")
    fused_codes, fused = mxq.quantize_mma(x, "mxfp8")
    assert torch.equal(mxq.swizzle_scales(plain), fused)


def test_mma_errors():
    x = torch.zeros((128, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mxq.MXQError) as e:
        mxq.quantize_mma(x, "axs6")
    assert e.value.status == 4
    s = torch.zeros((128, 4), dtype=torch.uint8, device="cuda")
    buf = torch.zeros(mxq.mxq_mma_scales_bytes(128, 128) + 16, dtype=torch.uint8, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert mxq.mxq_swizzle_scales(s.data_ptr(), 128, 4, buf.data_ptr() + 1, st) == 3      # misaligned out
    assert mxq.mxq_swizzle_scales(buf.data_ptr(), 128, 4, buf.data_ptr() + 16, st) == 1   # overlap
    assert mxq.mxq_swizzle_scales(s.data_ptr(), 128, 0, buf.data_ptr(), st) == 2          # kblocks <= 0
    assert mxq.mxq_swizzle_scales(s.data_ptr(), 0, 4, buf.data_ptr(), st) == 0            # empty
    torch.cuda.synchronize()


# ---- consumer check: cuBLAS block-scaled GEMM reads the codes and the tiled scales ----------

def _operand(fmt, rows, K, seed):
    x = spread_values(rows, K, seed, "f32")
    codes, tiled = mxq.quantize_mma(dev(x), fmt)
    _, plain = mxq.quantize(dev(x), fmt)
    o_codes, o_scales = oracle.quantize(x, fmt)
    dq = oracle.dequantize(o_codes, o_scales, fmt, (rows, K), "f32").astype(np.float64)
    return codes.view(torch.float8_e4m3fn), tiled, plain, dq


def _scaled_mm(a, b, sa, sb):
    err = None
    for od in (torch.float32, torch.bfloat16):
        try:
            c = torch._scaled_mm(a, b.t(), sa.view(torch.float8_e8m0fnu), sb.view(torch.float8_e8m0fnu), out_dtype=od)
            torch.cuda.synchronize()
            return c.float().cpu().numpy().astype(np.float64), od
        except RuntimeError as e:  # this torch/cuBLAS lacks the output type
            err = e
    pytest.skip(f"block-scaled GEMM not available here: {err}")


@pytest.mark.parametrize("fmt", ["mxfp8"])
@pytest.mark.parametrize("M,N,K", [(256, 384, 1024), (128, 256, 512), (512, 128, 4096)])
def test_block_scaled_gemm_consumes_codes_and_tiled_scales(fmt, M, N, K):
    a, sa, sa_plain, adq = _operand(fmt, M, K, 101 + M)
    b, sb, sb_plain, bdq = _operand(fmt, N, K, 202 + N)
    c, od = _scaled_mm(a, b, sa, sb)
    ref = adq @ bdq.T
    mag = np.abs(adq) @ np.abs(bdq).T
    tol = 1e-4 * mag + (2.0 ** -8 * np.abs(ref) if od == torch.bfloat16 else 0.0) + 1e-30
    bad = np.abs(c - ref) > tol
    assert not bad.any(), f"{bad.sum()} of {bad.size} outputs off (out dtype {od})"
    # negative control: the same codes with the scales row-major (untiled, zero-padded) are read wrongly
    wrong_a = torch.zeros_like(sa)
    wrong_a[: sa_plain.numel()] = sa_plain.reshape(-1)
    c2, _ = _scaled_mm(a, b, wrong_a, sb)
    assert (np.abs(c2 - ref) > tol).mean() > 0.5
