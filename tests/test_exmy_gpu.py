"""GPU parity for the eXmY formats (integer rounding path) against the oracle, bit for bit."""
import functools

import numpy as np
import pytest

import oracle
import synthetic

torch = pytest.importorskip("torch")
from block_scaled_microscaling_b200 import mxq  # noqa: E402

from test_parity_gpu import bits, dev, hard_values, host, tdtype  # noqa: E402

pytestmark = pytest.mark.gpu

SPLITS = [(E, M) for W in range(3, 10) for E in range(0, 6) for M in [W - 1 - E] if oracle.exmy_valid(E, M)]


@pytest.mark.parametrize("E,M", SPLITS)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_quantize_and_fake_quantize_match_oracle(E, M, dtype):
    x = hard_values(67, 160, dtype, seed=100 * E + M)
    codes, scales = mxq.quantize_exmy(dev(x), E, M)
    oc, os_ = oracle.quantize_exmy(x, E, M)
    assert np.array_equal(host(scales), os_)
    assert np.array_equal(host(codes), oc)
    fq = mxq.fake_quantize_exmy(dev(x), E, M)
    assert np.array_equal(bits(host(fq)), bits(oracle.fake_quantize_exmy(x, E, M)))


@pytest.mark.parametrize("E,M", SPLITS)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_dequantize_random_codes_match_oracle(E, M, dtype):
    rows, cols = 40, 256
    W = 1 + E + M
    rng = np.random.default_rng(7 * E + M)
    codes = rng.integers(0, 256, (rows, cols // 32 * 4 * W), dtype=np.uint8)
    scales = rng.integers(0, 256, (rows, cols // 32), dtype=np.uint8)
    scales.reshape(-1)[:256] = np.arange(256)
    out = mxq.dequantize_exmy(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(), E, M, (rows, cols),
                              tdtype(dtype))
    ref = oracle.dequantize_exmy(codes, scales, E, M, (rows, cols), dtype)
    assert np.array_equal(bits(host(out)), bits(ref))


@pytest.mark.parametrize("E,M,fmt", [(2, 1, "mxfp4"), (2, 3, "mxfp6_e2m3"), (3, 2, "mxfp6_e3m2")])
def test_named_splits_agree_with_the_conversion_instruction_path(E, M, fmt):
    x = hard_values(129, 256, "bf16", seed=3)
    c1, s1 = mxq.quantize_exmy(dev(x), E, M)
    c2, s2 = mxq.quantize(dev(x), fmt)
    assert torch.equal(c1, c2) and torch.equal(s1, s2)


def test_unsupported_split():
    x = torch.zeros(1, 32, device="cuda")
    c = torch.zeros(64, dtype=torch.uint8, device="cuda")
    s = torch.zeros(1, dtype=torch.uint8, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert mxq.mxq_quantize_exmy(6, 2, x.data_ptr(), 0, 1, 32, c.data_ptr(), s.data_ptr(), st) == 4
    assert mxq.mxq_quantize_exmy(1, 8, x.data_ptr(), 0, 1, 32, c.data_ptr(), s.data_ptr(), st) == 4


@pytest.mark.parametrize("E,M", [s for s in SPLITS if s[1] <= 5])
def test_bf16_two_values_per_word_path_at_scale(E, M):
    """bf16 values with M <= 5 round two values per 32-bit word (bf16x2 arithmetic, 16-bit
    lanes): a 2048x8192 tensor with per-block exponents over +-60 binades, zero, -0 and
    subnormal blocks, quantized whole; 48 sampled rows equal the oracle bit for bit."""
    rng = np.random.default_rng(1000 + 10 * E + M)
    rows, cols = 2048, 8192
    nb = rows * cols // 32
    x = rng.standard_normal((nb, 32)) * 2.0 ** rng.integers(-60, 61, nb)[:, None]
    kind = rng.integers(0, 32, nb)
    x[kind == 0] = 0.0
    x[kind == 1] = -0.0
    x[kind == 2] *= 2.0 ** -70  # bf16 subnormals
    ties = rng.integers(-64, 65, (nb, 32)) * 2.0 ** rng.integers(-10, 10, nb)[:, None]
    x = np.where((kind == 3)[:, None], ties, x)
    h = synthetic.f32_to_bf16_bits(x.astype(np.float32).reshape(rows, cols))
    codes, scales = mxq.quantize_exmy(dev(h), E, M)
    sel = np.sort(rng.choice(rows, 48, replace=False))
    oc, os_ = oracle.quantize_exmy(np.ascontiguousarray(h[sel]), E, M)
    assert np.array_equal(host(scales)[sel], os_)
    assert np.array_equal(host(codes)[sel], oc)


@functools.lru_cache(maxsize=1)
def fp32_wide(rows, cols, seed):
    """fp32 values with per-block exponents over +-60 binades, zero, -0 and subnormal blocks."""
    rng = np.random.default_rng(seed)
    nb = rows * cols // 32
    x = rng.standard_normal((nb, 32), dtype=np.float32)
    x *= np.exp2(rng.integers(-60, 61, (nb, 1)).astype(np.float32))
    kind = rng.integers(0, 32, nb)
    x[kind == 0] = 0.0
    x[kind == 1] = -0.0
    x[kind == 2] *= np.float32(2.0 ** -80)  # fp32 subnormals
    return x.reshape(rows, cols)


@pytest.mark.parametrize("E,M", SPLITS)
def test_fp32_quantize_dequantize_fake_quantize_at_scale(E, M):
    """fp32 2048x8192 (524 288 blocks: the persistent fp32 quantize takes several grid-stride
    passes, the one-pass dequantize and fake-quantize grids 2048 CTAs) converted whole by
    quantize, dequantize and fake-quantize; 48 sampled rows of each equal the oracle bit for
    bit."""
    rows, cols = 2048, 8192
    x = fp32_wide(rows, cols, 77)
    t = dev(x)
    codes, scales = mxq.quantize_exmy(t, E, M)
    out = mxq.dequantize_exmy(codes, scales, E, M, (rows, cols), torch.float32)
    fq = mxq.fake_quantize_exmy(t, E, M)
    sel = np.sort(np.random.default_rng(10 * E + M).choice(rows, 48, replace=False))
    xs = np.ascontiguousarray(x[sel])
    oc, os_ = oracle.quantize_exmy(xs, E, M)
    assert np.array_equal(host(scales)[sel], os_)
    assert np.array_equal(host(codes)[sel], oc)
    assert np.array_equal(bits(host(out)[sel]), bits(oracle.dequantize_exmy(oc, os_, E, M, xs.shape, "f32")))
    assert np.array_equal(bits(host(fq)[sel]), bits(oracle.fake_quantize_exmy(xs, E, M)))
