"""GPU parity: libmxq (through its C ABI) against the CPU oracle, bit for bit.

Tolerance is 0 ULP everywhere: codes, scale bytes and dequantized /
fake-quantized values are compared as raw bits (the method is exact
power-of-two scaling plus integer rounding; the exponential of the softmax
stage is a fixed fp32 algorithm both sides implement).
"""
import zlib

import numpy as np
import pytest

import oracle
import synthetic

torch = pytest.importorskip("torch")
from block_scaled_microscaling_b200 import mxq  # noqa: E402

pytestmark = pytest.mark.gpu

FMTS = ["axs6", "mxfp6_e2m3", "mxfp6_e3m2", "mxfp8", "mxfp4"]
SHAPES = [(1, 32), (3, 64), (7, 160), (129, 416), (1000, 2080), (5, 8192)]


# ---- host <-> device ------------------------------------------------------------------

def dev(x):
    if x.dtype == np.float32:
        return torch.from_numpy(np.ascontiguousarray(x)).cuda()
    assert x.dtype == np.uint16
    return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()


def host(t):
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    if t.dtype == torch.int16:
        return t.cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def bits(a):
    return np.ascontiguousarray(a).view(np.uint32 if a.dtype == np.float32 else np.uint16)


# ---- inputs ------------------------------------------------------------------------------

def hard_values(rows, cols, dtype, seed):
    """Per-block random exponents and special blocks: zeros, -0, NaN, +-Inf,
    subnormals, near-overflow, low-precision values that hit rounding ties."""
    rng = np.random.default_rng(seed)
    nb = rows * cols // 32
    x = rng.standard_normal((nb, 32)) * 2.0 ** rng.integers(-40, 40, nb)[:, None]
    kind = rng.integers(0, 16, nb)
    ties = rng.integers(-64, 65, (nb, 32)) * 2.0 ** rng.integers(-20, 20, nb)[:, None]
    x = np.where((kind == 1)[:, None], ties, x)
    x[kind == 2] = 0.0
    x[kind == 3] = -0.0
    one = rng.integers(0, 32, nb)
    r = np.arange(nb)
    x[r[kind == 4], one[kind == 4]] = np.nan
    x[r[kind == 5], one[kind == 5]] = np.inf
    x[r[kind == 6], one[kind == 6]] = -np.inf
    x[kind == 7] *= 2.0 ** -120  # fp32/bf16 subnormals
    x[kind == 8] = rng.standard_normal((np.sum(kind == 8), 32)) * 3e38
    x[r[kind == 9], one[kind == 9]] *= 1000.0  # one outlier
    with np.errstate(over="ignore", invalid="ignore"):
        f = x.astype(np.float32).reshape(rows, cols)
    if dtype == "f32":
        return f
    h = synthetic.f32_to_bf16_bits(np.nan_to_num(f, nan=0.0, posinf=0.0, neginf=0.0))
    # re-insert the specials as exact bf16 patterns
    fl = f.reshape(-1)
    hl = h.reshape(-1)
    hl[np.isnan(fl)] = 0x7FC0
    hl[np.isposinf(fl)] = 0x7F80
    hl[np.isneginf(fl)] = 0xFF80
    big = np.abs(fl) > 3.3e38
    hl[big] = np.where(fl[big] > 0, 0x7F7F, 0xFF7F)
    return h


def tdtype(dtype):
    return torch.float32 if dtype == "f32" else torch.bfloat16


# ---- quantize / dequantize / fake-quantize ------------------------------------------------

@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", SHAPES)
def test_quantize_matches_oracle(fmt, dtype, shape):
    x = hard_values(*shape, dtype, seed=zlib.crc32(repr((fmt, dtype, shape)).encode()))
    codes, scales = mxq.quantize(dev(x), fmt)
    oc, os_ = oracle.quantize(x, fmt)
    assert np.array_equal(host(scales), os_)
    assert np.array_equal(host(codes), oc)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_dequantize_matches_oracle_on_random_codes(fmt, dtype):
    """Every code value, E4M3 NaN codes, every scale byte including 0 and 0xFF."""
    rows, cols = 300, 256
    rng = np.random.default_rng(17)
    nb = rows * cols // 32
    codes = rng.integers(0, 256, (rows, cols // 32 * oracle.payload_bytes(fmt)), dtype=np.uint8)
    sb = rng.integers(0, 256, (rows, cols // 32)).astype(np.uint16)
    sb.reshape(-1)[:256] = np.arange(256)
    if fmt == "axs6":
        sb |= (rng.integers(0, 4, sb.shape) << 8).astype(np.uint16)  # config bits are ignored on read
        scales = sb
        tscales = torch.from_numpy(sb.view(np.int16)).cuda()
    else:
        scales = sb.astype(np.uint8)
        tscales = torch.from_numpy(scales).cuda()
    out = mxq.dequantize(torch.from_numpy(codes).cuda(), tscales, fmt, (rows, cols), tdtype(dtype))
    ref = oracle.dequantize(codes, scales, fmt, (rows, cols), dtype)
    assert np.array_equal(bits(host(out)), bits(ref))
    assert nb == rows * cols // 32


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(3, 64), (129, 416), (1000, 2080)])
def test_dequantize_matches_oracle(fmt, dtype, shape):
    x = hard_values(*shape, dtype, seed=7)
    oc, os_ = oracle.quantize(x, fmt)
    tsc = torch.from_numpy(os_.view(np.int16) if fmt == "axs6" else os_).cuda()
    out = mxq.dequantize(torch.from_numpy(oc).cuda(), tsc, fmt, shape, tdtype(dtype))
    ref = oracle.dequantize(oc, os_, fmt, shape, dtype)
    assert np.array_equal(bits(host(out)), bits(ref))


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", SHAPES)
def test_fake_quantize_matches_oracle(fmt, dtype, shape):
    x = hard_values(*shape, dtype, seed=11)
    out = mxq.fake_quantize(dev(x), fmt)
    ref = oracle.fake_quantize(x, fmt)
    assert np.array_equal(bits(host(out)), bits(ref))


@pytest.mark.parametrize("fmt", FMTS)
def test_fake_quantize_in_place_and_round_trip(fmt):
    x = hard_values(257, 320, "f32", seed=5)
    t = dev(x)
    codes, scales = mxq.quantize(t, fmt)
    rt = mxq.dequantize(codes, scales, fmt, t.shape, torch.float32)
    mxq.fake_quantize(t, fmt, out=t)
    assert np.array_equal(bits(host(t)), bits(host(rt)))
    assert np.array_equal(bits(host(t)), bits(oracle.fake_quantize(x, fmt)))


@pytest.mark.parametrize("fmt", ["axs6", "mxfp6_e3m2", "mxfp4"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_fake_quantize_bulk_copy_stream(fmt, dtype):
    """Sizes from 2^19 blocks up take the bulk-copy stream kernel: 16411 x 1024 values (525 152
    blocks, 2052 tiles of 256 with a 32-block tail), out of place and in place."""
    x = hard_values(16411, 1024, dtype, seed=17)
    t = dev(x)
    want = bits(oracle.fake_quantize(x, fmt))
    out = mxq.fake_quantize(t, fmt)
    assert np.array_equal(bits(host(out)), want)
    mxq.fake_quantize(t, fmt, out=t)
    assert np.array_equal(bits(host(t)), want)


def test_outputs_stay_inside_their_buffers():
    """Guard bands: sentinel bytes around every output are untouched."""
    x = hard_values(33, 96, "bf16", seed=3)
    for fmt in FMTS:
        nc = 33 * 3 * oracle.payload_bytes(fmt)
        ns = 33 * 3 * (2 if fmt == "axs6" else 1)
        cbuf = torch.full((nc + 64,), 0xA5, dtype=torch.uint8, device="cuda")
        sbuf = torch.full((ns + 64,), 0xA5, dtype=torch.uint8, device="cuda")
        codes = cbuf[32:32 + nc]
        scales = sbuf[32:32 + ns].view(torch.int16 if fmt == "axs6" else torch.uint8)
        mxq.quantize(dev(x), fmt, codes=codes, scales=scales)
        cb, sb = host(cbuf), host(sbuf)
        assert np.all(cb[:32] == 0xA5) and np.all(cb[32 + nc:] == 0xA5)
        assert np.all(sb[:32] == 0xA5) and np.all(sb[32 + ns:] == 0xA5)
        oc, os_ = oracle.quantize(x, fmt)
        assert np.array_equal(cb[32:32 + nc], oc.reshape(-1))
        obuf = torch.full((33 * 96 + 32,), -7.0, dtype=torch.bfloat16, device="cuda")
        mxq.dequantize(codes, scales, fmt, (33, 96), out=obuf[16:16 + 33 * 96].view(33, 96))
        ob = host(obuf)
        assert np.all(ob[:16] == 0xC0E0) and np.all(ob[16 + 33 * 96:] == 0xC0E0)  # bf16 -7.0


def test_deterministic():
    x = dev(hard_values(511, 1024, "bf16", seed=9))
    for fmt in FMTS:
        a = [host(t).copy() for t in mxq.quantize(x, fmt)]
        b = [host(t).copy() for t in mxq.quantize(x, fmt)]
        assert all(np.array_equal(p, q) for p, q in zip(a, b))


def test_errors_with_device_pointers():
    x = torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda")
    c = torch.zeros(4 * 48, dtype=torch.uint8, device="cuda")
    s = torch.zeros(8, dtype=torch.uint8, device="cuda")
    hx = torch.zeros(4, 64, dtype=torch.bfloat16)
    f = mxq.FORMATS["mxfp6_e2m3"]
    st = torch.cuda.current_stream().cuda_stream
    assert mxq.mxq_quantize(f, hx.data_ptr(), 1, 4, 64, c.data_ptr(), s.data_ptr(), st) == 1   # host memory
    assert mxq.mxq_quantize(f, x.data_ptr() + 2, 1, 4, 64, c.data_ptr(), s.data_ptr(), st) == 3  # misaligned
    assert mxq.mxq_quantize(f, x.data_ptr(), 1, 4, 64, c.data_ptr() + 8, s.data_ptr(), st) == 3
    assert mxq.mxq_quantize(f, x.data_ptr(), 1, 4, 64, x.data_ptr(), s.data_ptr(), st) == 1     # overlap
    y = torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda")
    assert mxq.mxq_fake_quantize(f, x.data_ptr(), 1, 4, 64, x.data_ptr(), st) == 0             # in place ok
    assert mxq.mxq_fake_quantize(f, x.data_ptr(), 1, 4, 64, x.data_ptr() + 64, st) == 1        # partial overlap
    torch.cuda.synchronize()
    del y


# ---- exp-then-quantize softmax stage --------------------------------------------------

@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("cols", [32, 96, 1024, 4096, 4992, 32768, 65536, 131072])
def test_exp_quantize_matches_oracle(fmt, cols):
    rows = max(2, min(64, 2 ** 21 // cols))
    s = synthetic.attention_scores(seed=4, heads=1, queries=rows, keys=cols)
    if rows >= 6:
        s[1, 5] = np.nan
        s[2, 7] = np.inf
        s[3, :] = -np.inf
        s[4, ::3] = -np.inf
        s[5, :] = 0.0
    codes, scales = mxq.exp_quantize(dev(s), fmt)
    oc, os_ = oracle.exp_quantize(s, fmt)
    assert np.array_equal(host(scales), os_)
    assert np.array_equal(host(codes), oc)


# ---- grouped quantize (one launch per decoder layer) ------------------------------------

@pytest.mark.parametrize("fmt", ["mxfp6_e2m3", "axs6", "mxfp4"])
def test_grouped_matches_oracle(fmt):
    shapes = [(40, 2560), (1, 32), (9, 96), (33, 4096), (0, 64), (17, 9728), (2, 160)]
    xs = [hard_values(r, c, "bf16", seed=i) if r else np.zeros((0, c), np.uint16) for i, (r, c) in enumerate(shapes)]
    outs = mxq.quantize_grouped([dev(x) for x in xs], fmt)
    for x, (c, s) in zip(xs, outs):
        if x.shape[0] == 0:
            continue
        oc, os_ = oracle.quantize(x, fmt)
        assert np.array_equal(host(s), os_) and np.array_equal(host(c), oc)


@pytest.mark.parametrize("fmt", ["mxfp4", "mxfp8", "mxfp6_e2m3", "axs6"])
@pytest.mark.parametrize("rows,cols", [(3000, 640), (700, 8192), (5, 131072), (3, 262144 + 32), (149, 4128)])
def test_exp_quantize_many_rows_per_cta(fmt, rows, cols):
    """More rows than resident CTAs: each CTA walks several rows (for MXFP4/MXFP8 the row
    stream runs up to three rows ahead of pass B, so the row-slot rings wrap many times; rows of
    one full stage plus a partial one, rows shorter than one stage)."""
    s = synthetic.attention_scores(seed=5, heads=1, queries=rows, keys=cols)
    s[::97, 3] = np.nan
    s[1::89, :] = -np.inf
    s[2::83, 5] = np.inf
    codes, scales = mxq.exp_quantize(dev(s), fmt)
    oc, os_ = oracle.exp_quantize(s, fmt)
    assert np.array_equal(host(scales), os_)
    assert np.array_equal(host(codes), oc)


# ---- column-direction blocks (32 rows of a column), transposed layout --------------------

@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(32, 32), (96, 64), (256, 32), (288, 96), (1024, 160), (4096, 256)])
def test_quantize_cols_matches_oracle_on_transpose(fmt, dtype, shape):
    x = hard_values(*shape, dtype, seed=zlib.crc32(repr(("cols", fmt, dtype, shape)).encode()))
    codes, scales = mxq.quantize_cols(dev(x), fmt)
    xt = np.ascontiguousarray(x.T)
    oc, os_ = oracle.quantize(xt, fmt)
    assert np.array_equal(host(scales), os_)
    assert np.array_equal(host(codes), oc)
    out = mxq.dequantize_cols(codes, scales, fmt, shape, tdtype(dtype))
    ref = oracle.dequantize(oc, os_, fmt, xt.shape, dtype).T
    assert np.array_equal(bits(host(out)), bits(np.ascontiguousarray(ref)))


def test_cols_shape_rules():
    x = torch.zeros(48, 64, dtype=torch.bfloat16, device="cuda")
    c = torch.zeros(64 * 48, dtype=torch.uint8, device="cuda")
    s = torch.zeros(128, dtype=torch.uint8, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert mxq.mxq_quantize_cols(1, x.data_ptr(), 1, 48, 64, c.data_ptr(), s.data_ptr(), st) == 2  # rows % 32
    assert mxq.mxq_quantize_cols(1, x.data_ptr(), 1, 32, 48, c.data_ptr(), s.data_ptr(), st) == 2  # cols % 32
    assert mxq.mxq_quantize_cols(1, x.data_ptr(), 1, 0, 64, c.data_ptr(), s.data_ptr(), st) == 0   # empty
