"""GPU parity of the column-direction path at sizes where its persistent grid walks several
tiles per CTA, bit for bit against the oracle.

Column-direction blocks are 32 consecutive rows of one column; the library lays the result out
as the row-direction quantization of the transpose (codes [cols, rows/32*P], scales
[cols, rows/32]), so the oracle runs on x.T. The converted operands feed block-scaled GEMMs
whose K-contiguous operand is the column direction ("Sonar: Online MXFP6", Start a model and
Current limits).

The quantize kernel cuts the matrix into tiles of 256 rows x 128 bytes and runs a persistent
grid of (SMs x resident CTAs) CTAs that walk their tiles through two tensor-copy buffers, so a
shape with more tiles than twice the grid reuses both buffers and flips their barrier phases
on every CTA. Each test asserts that premise for its shape before comparing.
"""
import functools
import zlib

import numpy as np
import pytest

import oracle

torch = pytest.importorskip("torch")
from block_scaled_microscaling_b200 import mxq  # noqa: E402

from test_parity_gpu import bits, dev, hard_values, host, tdtype  # noqa: E402

pytestmark = pytest.mark.gpu

FMTS = ["axs6", "mxfp6_e2m3", "mxfp6_e3m2", "mxfp8", "mxfp4"]
TILE_ROWS, TILE_BYTES = 256, 128


def tiles(rows, cols, dtype):
    tc = TILE_BYTES // (4 if dtype == "f32" else 2)
    return -(-cols // tc) * -(-rows // TILE_ROWS)


def assert_walks_several_tiles(rows, cols, dtype):
    """Two 32 KB tile buffers per CTA leave room for at most 3 CTAs in an SM's 228 KB of shared
    memory, so the persistent grid has at most 3 x SMs CTAs; more than twice that many tiles
    means every CTA takes at least two."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert tiles(rows, cols, dtype) >= 2 * (3 * sms), (rows, cols, dtype)


@functools.lru_cache(maxsize=1)
def big_values(rows, cols, dtype, seed):
    """Per-block random exponents over +-30 binades and a sprinkling of zero, -0, subnormal and
    NaN / -Inf column blocks (the blocks are 32 rows of a column here), cheap at any size."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows // 32, 32, cols), dtype=np.float32)
    x *= np.exp2(rng.integers(-30, 31, (rows // 32, 1, cols)).astype(np.float32))
    kind = rng.integers(0, 64, (rows // 32, cols))
    rb, c = np.nonzero(kind == 0)
    x[rb, :, c] = 0.0
    rb, c = np.nonzero(kind == 1)
    x[rb, :, c] = -0.0
    rb, c = np.nonzero(kind == 2)
    x[rb, :, c] *= np.float32(2.0 ** -120)
    rb, c = np.nonzero(kind == 3)
    x[rb, c % 32, c] = np.nan
    rb, c = np.nonzero(kind == 4)
    x[rb, c % 32, c] = -np.inf
    x = np.ascontiguousarray(x.reshape(rows, cols))
    if dtype == "f32":
        return x
    return (x.view(np.uint32) >> 16).astype(np.uint16)  # bf16 by truncation: NaN and -Inf stay what they are


def check_full(x, fmt, dtype):
    rows, cols = x.shape
    codes, scales = mxq.quantize_cols(dev(x), fmt)
    xt = np.ascontiguousarray(x.T)
    oc, os_ = oracle.quantize(xt, fmt)
    assert np.array_equal(host(scales), os_)
    assert np.array_equal(host(codes), oc)
    out = mxq.dequantize_cols(codes, scales, fmt, (rows, cols), tdtype(dtype))
    ref = np.ascontiguousarray(oracle.dequantize(oc, os_, fmt, xt.shape, dtype).T)
    assert np.array_equal(bits(host(out)), bits(ref))


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_cols_4096x4096_every_tile(fmt, dtype):
    """4096 x 4096: 1024 bf16 tiles (2048 fp32 tiles) over the persistent grid, compared in full."""
    rows, cols = 4096, 4096
    assert_walks_several_tiles(rows, cols, dtype)
    x = big_values(rows, cols, dtype, seed=zlib.crc32(repr(("c4096", fmt, dtype)).encode()))
    check_full(x, fmt, dtype)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("dtype,shape", [("bf16", (4192, 4128)), ("f32", (2336, 4160)), ("bf16", (2080, 8224))])
def test_cols_ragged_multi_tile(fmt, dtype, shape):
    """rows % 256 != 0 (a last row tile of 3 or 1 row-blocks) and, for bf16, a last column
    strip of 32 columns, at sizes where the grid still walks several tiles per CTA."""
    rows, cols = shape
    assert_walks_several_tiles(rows, cols, dtype)
    assert rows % TILE_ROWS != 0
    x = hard_values(cols, rows, dtype, seed=zlib.crc32(repr(("rag", fmt, dtype, shape)).encode()))
    # hard_values draws its special blocks along the last dim; transposed they become column blocks
    check_full(np.ascontiguousarray(x.T), fmt, dtype)


@pytest.mark.parametrize("fmt", ["mxfp6_e2m3", "mxfp8", "axs6"])
@pytest.mark.parametrize("dtype,shape", [("f32", (8192, 8192)), ("bf16", (16384, 8192))])
def test_cols_large_sampled_columns(fmt, dtype, shape):
    """The sizes the column figures are measured at (fp32 8192x8192: 8192 tiles; bf16
    16384x8192: 8192 tiles): the whole matrix converted in one launch, then 96 sampled columns
    (the first and last included) compared in full with the oracle on those columns, and
    dequantize_cols of the whole result on the same columns."""
    rows, cols = shape
    assert_walks_several_tiles(rows, cols, dtype)
    x = big_values(rows, cols, dtype, seed=zlib.crc32(repr(("big", dtype, shape)).encode()))
    codes, scales = mxq.quantize_cols(dev(x), fmt)
    rng = np.random.default_rng(5)
    sel = np.unique(np.concatenate([rng.choice(cols, 94, replace=False), [0, cols - 1]]))
    xs = np.ascontiguousarray(x[:, sel].T)
    oc, os_ = oracle.quantize(xs, fmt)
    hs, hc = host(scales), host(codes)
    assert np.array_equal(hs[sel], os_)
    assert np.array_equal(hc[sel], oc)
    out = mxq.dequantize_cols(codes, scales, fmt, (rows, cols), tdtype(dtype))
    ref = oracle.dequantize(oc, os_, fmt, xs.shape, dtype)
    assert np.array_equal(bits(host(out)[:, sel].T.copy()), bits(ref))


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("dtype,shape", [("bf16", (4192, 4128)), ("f32", (2336, 4160))])
def test_dequantize_cols_random_codes(fmt, dtype, shape):
    """Every code value (E4M3 NaN codes included) and every scale byte (0 and 0xFF included) in the
    transposed layout, at a ragged multi-tile size: dequantize_cols equals the oracle's dequantize
    of the same codes, transposed back."""
    rows, cols = shape
    assert_walks_several_tiles(rows, cols, dtype)
    rng = np.random.default_rng(zlib.crc32(repr(("rnd", fmt, dtype, shape)).encode()))
    pb = oracle.payload_bytes(fmt)
    codes = rng.integers(0, 256, (cols, rows // 32 * pb), dtype=np.uint8)
    sb = rng.integers(0, 256, (cols, rows // 32)).astype(np.uint16)
    sb.reshape(-1)[:256] = np.arange(256)
    if fmt == "axs6":
        sb |= (rng.integers(0, 4, sb.shape) << 8).astype(np.uint16)  # config bits are ignored on read
        scales, tscales = sb, torch.from_numpy(sb.view(np.int16)).cuda()
    else:
        scales = sb.astype(np.uint8)
        tscales = torch.from_numpy(scales).cuda()
    out = mxq.dequantize_cols(torch.from_numpy(codes).cuda(), tscales, fmt, (rows, cols), tdtype(dtype))
    ref = np.ascontiguousarray(oracle.dequantize(codes, scales, fmt, (cols, rows), dtype).T)
    assert np.array_equal(bits(host(out)), bits(ref))


@pytest.mark.parametrize("dtype,shape", [("bf16", (2080, 8224)), ("f32", (2336, 4160)), ("bf16", (96, 96))])
def test_cols_outputs_stay_inside_their_buffers(dtype, shape):
    """Guard bands: sentinel bytes around the codes, the scales and the values that the column
    kernels write stay untouched, at shapes with a last row band of one row-block and (bf16) a
    last column strip of 32 columns."""
    rows, cols = shape
    x = big_values(rows, cols, dtype, seed=11)
    for fmt in FMTS:
        nc = cols * (rows // 32) * oracle.payload_bytes(fmt)
        ns = cols * (rows // 32) * (2 if fmt == "axs6" else 1)
        cbuf = torch.full((nc + 64,), 0xA5, dtype=torch.uint8, device="cuda")
        sbuf = torch.full((ns + 64,), 0xA5, dtype=torch.uint8, device="cuda")
        codes = cbuf[32:32 + nc]
        scales = sbuf[32:32 + ns].view(torch.int16 if fmt == "axs6" else torch.uint8)
        mxq.quantize_cols(dev(x), fmt, codes=codes, scales=scales, check=True)
        cb, sbh = host(cbuf), host(sbuf)
        assert np.all(cb[:32] == 0xA5) and np.all(cb[32 + nc:] == 0xA5)
        assert np.all(sbh[:32] == 0xA5) and np.all(sbh[32 + ns:] == 0xA5)
        esz = 4 if dtype == "f32" else 2
        obuf = torch.full(((rows * cols * esz + 128) // 4,), 0x5A5A5A5A, dtype=torch.int32, device="cuda")
        ov = obuf.view(torch.uint8)[64:64 + rows * cols * esz].view(tdtype(dtype)).view(rows, cols)
        mxq.dequantize_cols(codes, scales, fmt, (rows, cols), out=ov)
        ob = host(obuf.view(torch.uint8))
        assert np.all(ob[:64] == 0x5A) and np.all(ob[64 + rows * cols * esz:] == 0x5A)
        ref = oracle.dequantize(host(codes).reshape(cols, -1), host(scales).reshape(cols, -1), fmt, (cols, rows), dtype)
        assert np.array_equal(bits(host(ov)), bits(np.ascontiguousarray(ref.T)))


@pytest.mark.parametrize("fmt,dtype,shape", [("mxfp6_e2m3", "f32", (16384, 32768)), ("axs6", "f32", (16384, 32768)),
                                             ("mxfp8", "bf16", (32768, 32768))])
def test_dequantize_cols_beyond_31_bit_offsets(fmt, dtype, shape):
    """A 2 GiB output (2^31 bytes) leaves the persistent dequantize's 32-bit offsets, so the
    launcher takes the one-CTA-per-tile kernel with 64-bit offsets: the whole matrix converted
    there and back, 24 sampled columns (the first and last included) compared in full with the
    oracle. The values come from the device generator (per-column-block exponents over +-30
    binades, zero and NaN column blocks) and are copied back for the oracle."""
    rows, cols = shape
    esz = 4 if dtype == "f32" else 2
    assert rows * cols * esz >= 1 << 31
    g = torch.Generator(device="cuda").manual_seed(zlib.crc32(repr(("wide", fmt, dtype, shape)).encode()))
    x = torch.randn(rows // 32, 32, cols, device="cuda", generator=g)
    x *= torch.exp2(torch.randint(-30, 31, (rows // 32, 1, cols), device="cuda", generator=g).float())
    kind = torch.randint(0, 64, (rows // 32, 1, cols), device="cuda", generator=g)
    x = torch.where(kind == 0, torch.zeros_like(x), x)
    x[:, 5:6, :] = torch.where(kind == 1, torch.full_like(x[:, 5:6, :], float("nan")), x[:, 5:6, :])
    x = x.reshape(rows, cols).to(tdtype(dtype))
    del kind
    codes, scales = mxq.quantize_cols(x, fmt)
    rng = np.random.default_rng(7)
    sel = np.unique(np.concatenate([rng.choice(cols, 22, replace=False), [0, cols - 1]]))
    xs = np.ascontiguousarray(host(x[:, torch.from_numpy(sel).cuda()]).T)
    oc, os_ = oracle.quantize(xs, fmt)
    assert np.array_equal(host(scales[torch.from_numpy(sel).cuda()]), os_)
    assert np.array_equal(host(codes[torch.from_numpy(sel).cuda()]), oc)
    del x
    torch.cuda.empty_cache()
    out = mxq.dequantize_cols(codes, scales, fmt, (rows, cols), tdtype(dtype))
    ref = oracle.dequantize(oc, os_, fmt, xs.shape, dtype)
    assert np.array_equal(bits(host(out[:, torch.from_numpy(sel).cuda()]).T.copy()), bits(ref))
