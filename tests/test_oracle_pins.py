"""Pins for the CPU oracle: each test ties it to something other than itself.

- element decode tables: ml_dtypes / torch casts (library routines);
- element rounding: brute-force nearest-code search written here, over an
  independent decode table, exhaustively over bf16 bit patterns, plus the
  library casts (ml_dtypes / torch float8) on the clamped quotient;
- the shared-scale rule: covariance under powers of two and the top-binade
  property of the block maximum;
- packing: an independent big-integer packer and a hand-written vector;
- output rounding: numpy float32 and ml_dtypes bfloat16 casts;
- the fp32 exponential: math.exp within 2 ulp, constants re-derived from ln 2;
- facts the pages print (bits per value, memory ratio, field widths).
"""
import json
import math
import os
from decimal import Decimal, getcontext

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle
import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
FACTS = json.load(open(os.path.join(GOLDEN, "page_facts.json")))

FP_FORMATS = ["mxfp6_e2m3", "mxfp6_e3m2", "mxfp8", "mxfp4"]
ALL_FORMATS = ["axs6"] + FP_FORMATS
ML = {"mxfp6_e2m3": ml_dtypes.float6_e2m3fn, "mxfp6_e3m2": ml_dtypes.float6_e3m2fn,
      "mxfp8": ml_dtypes.float8_e4m3fn, "mxfp4": ml_dtypes.float4_e2m1fn}


def library_table(fmt):
    """Decode table from ml_dtypes (codes stored one per byte, sign at bit w-1)."""
    if fmt == "axs6":
        # the AXS-6 magnitude is the fixed-point number m/16 (sign + 5-bit mantissa)
        mags = np.arange(32) / 16.0
        return np.concatenate([mags, -mags])
    n = 1 << oracle.bits(fmt)
    return np.arange(n, dtype=np.uint8).view(ML[fmt]).astype(np.float64)


# ---- code tables -------------------------------------------------------------------

@pytest.mark.parametrize("fmt", FP_FORMATS)
def test_decode_table_matches_ml_dtypes(fmt):
    ours = oracle.decode_table(fmt)
    ref = library_table(fmt)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])
    assert np.array_equal(np.signbit(ours[ok]), np.signbit(ref[ok]))


def test_e4m3_table_matches_torch_float8():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    ours = oracle.decode_table("mxfp8")
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])


def test_axs6_table_structure():
    f = FACTS["axs6_block"]
    t = oracle.decode_table("axs6")
    assert t.size == 2 ** f["element_bits"]
    mags = t[:32]
    # 5-bit magnitude on a uniform grid, sign in the top bit
    assert np.all(np.diff(mags) == mags[1] - mags[0])
    assert np.array_equal(t[32:], -mags) and np.signbit(t[32])
    assert mags[-1] < 2.0 <= 2 * mags[16]  # block max lands in [1, 2): emax = 0
    assert oracle.emax("axs6") == 0


@pytest.mark.parametrize("fmt", ALL_FORMATS)
def test_tables_monotone_and_round_trip(fmt):
    t = oracle.decode_table(fmt)
    half = t.size // 2
    pos = t[:half]
    finite = pos[~np.isnan(pos)]
    assert np.all(np.diff(finite) > 0)
    assert oracle.maxval(fmt) == finite[-1]
    # encode(decode(c)) == c for every non-NaN magnitude code
    for c in range(finite.size):
        assert oracle.round_mag(fmt, pos[c]) == c


@pytest.mark.parametrize("fmt", ALL_FORMATS)
def test_codes_round_trip_through_blocks_at_extreme_scales(fmt):
    """Every non-NaN code c, of either sign, written as the fp32 value decode(c)·2^k into blocks
    that also hold the largest code (so the block maximum fixes the scale at exactly 2^k), comes
    back as c with scale byte k + 127 for k in {-127, -20, 0, 20, 127 - emax}: the ends of the
    E8M0 range, where a wrong clamp or an fp32 subnormal input would show; and the dequantized
    values are the inputs, bit for bit."""
    w = oracle.bits(fmt)
    t = oracle.decode_table(fmt)
    codes = np.array([c for c in range(1 << w) if not np.isnan(t[c])], dtype=np.uint32)
    top = int(np.argmax(np.where(np.isnan(t), -np.inf, t)))  # the largest positive code
    nblocks = -(-codes.size // 31)
    want = np.full((nblocks, 32), top, dtype=np.uint32)
    want[:, 1:].flat[:codes.size] = codes
    for k in [-127, -20, 0, 20, 127 - oracle.emax(fmt)]:
        v = t[want] * 2.0 ** k
        x = v.astype(np.float32)
        assert np.array_equal(x.astype(np.float64), v)  # every value is an fp32 number
        got_codes, scales = oracle.quantize(x, fmt)
        bytes_ = (scales & 0xFF) if fmt == "axs6" else scales
        assert np.all(bytes_ == k + 127), (fmt, k)
        P = oracle.payload_bytes(fmt)
        for b in range(nblocks):
            assert np.array_equal(oracle.unpack_codes(got_codes[b, :P], fmt), want[b]), (fmt, k, b)
        back = oracle.dequantize(got_codes, scales, fmt, x.shape, "f32")
        assert np.array_equal(back.view(np.uint32), x.view(np.uint32)), (fmt, k)


def test_max_values_and_emax():
    expect = {"axs6": (31 / 16, 0), "mxfp6_e2m3": (7.5, 2), "mxfp6_e3m2": (28.0, 4),
              "mxfp8": (448.0, 8), "mxfp4": (6.0, 2)}
    for fmt, (mx, em) in expect.items():
        assert oracle.maxval(fmt) == mx
        assert oracle.emax(fmt) == em == math.floor(math.log2(mx))
    # library max values
    assert float(torch.finfo(torch.float8_e4m3fn).max) == 448.0
    for fmt in ["mxfp6_e2m3", "mxfp6_e3m2", "mxfp4"]:
        assert float(ml_dtypes.finfo(ML[fmt]).max) == oracle.maxval(fmt)


# ---- facts printed on the pages -----------------------------------------------------

def test_page_facts_bits():
    a = FACTS["axs6_block"]
    block_bits = a["shared_exponent_bits"] + a["config_bits"] + a["block_size"] * a["element_bits"]
    assert block_bits == 202
    bpv = block_bits / a["block_size"]
    assert round(bpv, FACTS["axs6_bits_per_value"]["decimals"]) == FACTS["axs6_bits_per_value"]["value"]
    assert round(100 * (1 - bpv / 8)) == FACTS["axs6_vs_fp8_memory"]["percent"]
    ratio = 2 ** a["mantissa_bits"] / 2 ** FACTS["axs6_vs_fp8_mantissa"]["fp8_mantissa_bits"]
    assert ratio == FACTS["axs6_vs_fp8_mantissa"]["ratio"]
    assert oracle.bits("axs6") == a["element_bits"]
    m = FACTS["mxfp6_layout"]
    for fmt in ["mxfp6_e2m3", "mxfp6_e3m2"]:
        assert oracle.bits(fmt) == m["element_bits"]
        assert oracle.payload_bytes(fmt) == m["element_bits"] * m["block_size"] // 8 == 24
    e = FACTS["e2m1_fields"]
    assert oracle.bits("mxfp4") == e["sign"] + e["exponent"] + e["mantissa"]
    e = FACTS["e4m3_fields"]
    assert oracle.bits("mxfp8") == e["sign"] + e["exponent"] + e["mantissa"]
    r = FACTS["e3m2_vs_e2m3"]
    assert oracle.maxval(r["larger_range"]) > oracle.maxval(r["more_mantissa"])


def test_scale_array_sizes():
    x = synthetic.quickstart_fp32()
    for fmt in ALL_FORMATS:
        codes, scales = oracle.quantize(x, fmt)
        assert scales.size == x.size // 32
        assert codes.nbytes == x.size * oracle.bits(fmt) // 8


# ---- element rounding: brute force ------------------------------------------------

def brute_force_mags(fmt, y):
    """Nearest non-negative grid magnitude to each y >= 0, ties to the even code."""
    table = library_table(fmt)
    half = table.size // 2
    mags = table[:half]
    codes = np.arange(half)
    keep = ~np.isnan(mags)
    mags, codes = mags[keep], codes[keep]
    d = np.abs(y[:, None] - mags[None, :])
    dmin = d.min(axis=1, keepdims=True)
    tie = d == dmin
    # among tied codes prefer the even one (ties are between adjacent codes)
    score = np.where(tie, np.where(codes[None, :] % 2 == 0, 0, 1), 2)
    return codes[np.argmin(score, axis=1)].astype(np.uint32)


def bf16_positive_values():
    h = np.arange(0x0000, 0x7F80, dtype=np.uint16)  # +0 .. largest finite bf16
    return synthetic.bf16_bits_to_f32(h).astype(np.float64)


@pytest.mark.parametrize("fmt", ALL_FORMATS)
def test_round_exhaustive_bf16_patterns(fmt):
    """Every positive bf16 value times 2^k, k chosen so y sweeps the whole grid."""
    x = bf16_positive_values()
    mx = oracle.maxval(fmt)
    for k in range(-12, 12):
        y = np.ldexp(x, k)
        y = y[(y < 2 * mx) & (y >= 2.0 ** -14)]
        if y.size == 0:
            continue
        assert np.array_equal(oracle.round_mags(fmt, y), brute_force_mags(fmt, y)), k


@pytest.mark.parametrize("fmt", ALL_FORMATS)
def test_round_midpoints_and_neighbours(fmt):
    t = oracle.decode_table(fmt)
    mags = t[: t.size // 2]
    mags = mags[~np.isnan(mags)]
    mids = (mags[:-1] + mags[1:]) / 2
    ys = np.concatenate([mids, np.nextafter(mids, 0), np.nextafter(mids, np.inf), mags,
                         [oracle.maxval(fmt) * 1.0001, oracle.maxval(fmt) * 3, 0.0]])
    assert np.array_equal(oracle.round_mags(fmt, ys), brute_force_mags(fmt, ys))


@pytest.mark.parametrize("fmt", ALL_FORMATS)
def test_round_random_fp32(fmt):
    rng = np.random.default_rng(7)
    y = np.abs(rng.standard_normal(200_000).astype(np.float32)).astype(np.float64) * oracle.maxval(fmt) / 2
    assert np.array_equal(oracle.round_mags(fmt, y), brute_force_mags(fmt, y))


@pytest.mark.parametrize("fmt", FP_FORMATS)
def test_round_matches_library_cast(fmt):
    """Clamp to +-max, then the library's round-to-nearest-even cast."""
    rng = np.random.default_rng(11)
    mx = oracle.maxval(fmt)
    y = np.abs(rng.standard_normal(100_000)).astype(np.float32) * np.float32(mx / 1.5)
    y = np.concatenate([y, bf16_positive_values().astype(np.float32)])
    y = y[np.isfinite(y)]
    yc = np.minimum(y, np.float32(mx))
    lib_codes = yc.astype(ML[fmt]).view(np.uint8).astype(np.uint32)
    ours = oracle.round_mags(fmt, y.astype(np.float64))
    assert np.array_equal(ours, lib_codes)
    if fmt == "mxfp8":
        tc = torch.from_numpy(yc).to(torch.float8_e4m3fn).view(torch.uint8).numpy().astype(np.uint32)
        assert np.array_equal(ours, tc)


@pytest.mark.parametrize("fmt", ALL_FORMATS)
def test_round_ten_million_fp32_patterns(fmt):
    """10^7 fp32 bit patterns drawn uniformly between those of 2^-14 and 2·max (every binade
    of the grid and its subnormal range, all 23 mantissa bits random): the oracle's rounding
    equals the library's round-to-nearest-even cast after clamping (ml_dtypes for the OCP
    formats; for AXS-6, whose element is the fixed-point m/16, numpy's rint of 16·y)."""
    rng = np.random.default_rng(2024)
    mx = oracle.maxval(fmt)
    lo = np.array([2.0 ** -14], dtype=np.float32).view(np.uint32)[0]
    hi = np.array([2 * mx], dtype=np.float32).view(np.uint32)[0]
    y = rng.integers(lo, hi, 10_000_000, dtype=np.uint32).view(np.float32)
    yc = np.minimum(y, np.float32(mx))
    if fmt == "axs6":
        lib_codes = np.rint(yc.astype(np.float64) * 16).astype(np.uint32)
    else:
        lib_codes = yc.astype(ML[fmt]).view(np.uint8).astype(np.uint32)
    ours = oracle.round_mags(fmt, y.astype(np.float64))
    bad = np.flatnonzero(ours != lib_codes)
    assert bad.size == 0, (fmt, y[bad[:5]], ours[bad[:5]], lib_codes[bad[:5]])


# ---- the block: scale rule, signs, specials -----------------------------------------

def oracle_block_bruteforce(fmt, x):
    """Independent O2 for one block: scale from frexp, codes by brute force."""
    x = np.asarray(x, dtype=np.float64)
    amax = np.max(np.abs(x))
    if amax == 0:
        es = -127
    else:
        es = int(np.frexp(amax)[1]) - 1 - oracle.emax(fmt)
        es = min(max(es, -127), 127)
    y = np.ldexp(np.abs(x), -es)
    mags = brute_force_mags(fmt, y)
    sign = np.where(np.signbit(x), 1 << (oracle.bits(fmt) - 1), 0).astype(np.uint32)
    return mags | sign, es + 127


@pytest.mark.parametrize("fmt", ALL_FORMATS)
def test_block_bruteforce_tiny(fmt):
    rng = np.random.default_rng(3)
    for trial in range(300):
        scale = 2.0 ** rng.integers(-40, 40)
        x = (rng.standard_normal(32) * scale).astype(np.float32)
        if trial % 5 == 0:
            x[rng.integers(0, 32, 4)] *= 37.0
        if trial % 7 == 0:
            x[rng.integers(0, 32, 3)] = 0.0
            x[0] = -0.0
        codes, byte = oracle.quantize_block(fmt, x)
        c2, b2 = oracle_block_bruteforce(fmt, x)
        assert byte == b2
        assert np.array_equal(codes, c2)


@pytest.mark.parametrize("fmt", ALL_FORMATS)
def test_scale_covariance(fmt):
    rng = np.random.default_rng(5)
    x = rng.standard_normal(32)
    c0, b0 = oracle.quantize_block(fmt, x)
    for k in [-60, -7, -1, 1, 3, 50]:
        c, b = oracle.quantize_block(fmt, np.ldexp(x, k))
        assert b == b0 + k and np.array_equal(c, c0)


@pytest.mark.parametrize("fmt", ALL_FORMATS)
def test_block_max_in_top_binade(fmt):
    rng = np.random.default_rng(9)
    for _ in range(200):
        x = rng.standard_normal(32) * 2.0 ** rng.integers(-30, 30)
        codes, byte = oracle.quantize_block(fmt, x)
        i = int(np.argmax(np.abs(x)))
        v = abs(oracle.decode(fmt, int(codes[i])))
        assert 2.0 ** oracle.emax(fmt) <= v <= oracle.maxval(fmt)


@pytest.mark.parametrize("fmt", ALL_FORMATS)
def test_specials(fmt):
    sm = 1 << (oracle.bits(fmt) - 1)
    codes, byte = oracle.quantize_block(fmt, np.zeros(32))
    assert byte == 0 and not codes.any()
    z = np.zeros(32)
    z[3] = -0.0
    codes, byte = oracle.quantize_block(fmt, z)
    assert codes[3] == sm and byte == 0
    for bad in [np.nan, np.inf, -np.inf]:
        x = np.ones(32)
        x[17] = bad
        codes, byte = oracle.quantize_block(fmt, x)
        assert byte == 0xFF and not codes.any()
    # fp32 subnormal block: scale clamps at 2^-127
    x = np.full(32, 2.0 ** -140)
    codes, byte = oracle.quantize_block(fmt, x)
    assert byte == 0
    # largest finite fp32
    x = np.full(32, float(np.finfo(np.float32).max))
    codes, byte = oracle.quantize_block(fmt, x)
    assert byte == 127 + 127 - oracle.emax(fmt)


@pytest.mark.parametrize("fmt", ALL_FORMATS)
def test_sign_symmetry(fmt):
    rng = np.random.default_rng(2)
    x = rng.standard_normal(32)
    c, b = oracle.quantize_block(fmt, x)
    cn, bn = oracle.quantize_block(fmt, -x)
    sm = 1 << (oracle.bits(fmt) - 1)
    assert b == bn and np.array_equal(c ^ sm, cn)


# ---- packing -------------------------------------------------------------------------

def bigint_pack(codes, w):
    acc = 0
    for j, c in enumerate(codes):
        acc |= int(c) << (w * j)
    return np.frombuffer(acc.to_bytes(32 * w // 8, "little"), dtype=np.uint8)


@pytest.mark.parametrize("fmt", ALL_FORMATS)
def test_packing_bit_order(fmt):
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((3, 64)) * 3).astype(np.float32)
    codes, scales = oracle.quantize(x, fmt)
    pb = oracle.payload_bytes(fmt)
    for b in range(6):
        c, _ = oracle.quantize_block(fmt, x.reshape(-1)[32 * b: 32 * b + 32])
        assert np.array_equal(codes.reshape(-1)[b * pb:(b + 1) * pb], bigint_pack(c, oracle.bits(fmt)))


def test_packing_hand_vector():
    # E2M3 codes 1, 2, 3, 4 (then zeros): bits 000001 000010 000011 000100 LSB first
    # byte0 = 01 | (10 & 11) << 6 = 0x81 ; byte1 = 0b0011_0000 | 0b0000 = 0x30 ; byte2 = 0b0001_0000 >> ... = 0x10
    x = np.zeros(32)
    x[0], x[1], x[2], x[3] = 0.125, 0.25, 0.375, 0.5
    x[4] = 7.5  # sets the scale to 2^0 (amax in [4, 8) for emax = 2)
    codes, scales = oracle.quantize(x.astype(np.float32).reshape(1, 32), "mxfp6_e2m3")
    assert scales[0, 0] == 127
    assert list(codes[0, :3]) == [0x81, 0x30, 0x10]
    # mxfp4: low nibble first
    y = np.zeros(32, np.float32)
    y[0], y[1], y[2] = 0.5, 6.0, -1.0
    codes, scales = oracle.quantize(y.reshape(1, 32), "mxfp4")
    assert scales[0, 0] == 127 and list(codes[0, :2]) == [0x71, 0x0A]


# ---- dequantize / fake-quantize -------------------------------------------------------

def test_round_binary_matches_numpy_and_ml_dtypes():
    rng = np.random.default_rng(8)
    v = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-45, 38, 20000),
                        np.ldexp(1.0, np.arange(-160, 130)).astype(np.float64)])
    v = v.astype(np.float64)
    f32 = np.array([oracle.round_binary(t, 24, -126, 127) for t in v])
    with np.errstate(over="ignore"):
        assert np.array_equal(f32, v.astype(np.float32).astype(np.float64))
    bf = np.array([oracle.round_binary(t, 8, -126, 127) for t in v])
    with np.errstate(over="ignore"):
        x32 = v.astype(np.float32)  # bf16 rounding is checked on float32 inputs
    bf32 = np.array([oracle.round_binary(float(t), 8, -126, 127) for t in x32])
    with np.errstate(over="ignore"):
        assert np.array_equal(bf32, x32.astype(ml_dtypes.bfloat16).astype(np.float64))
    assert np.all(np.isfinite(bf) | (np.abs(v) > 3e38))


@pytest.mark.parametrize("fmt", ALL_FORMATS)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_dequantize_of_quantize_equals_fake_quantize(fmt, dtype):
    x = synthetic.gaussian((8, 96), 0.7, seed=6, sid=1, dtype=dtype)
    if dtype == "f32":
        x[2, 5] = np.float32(1e-41)  # subnormal input
        x[3, :32] = 0
        x[3, 7] = -0.0
    codes, scales = oracle.quantize(x, fmt)
    dq = oracle.dequantize(codes, scales, fmt, x.shape, dtype)
    fq = oracle.fake_quantize(x, fmt)
    assert np.array_equal(dq.view(np.uint8), fq.view(np.uint8))
    # and dequantize is the decoded table value times the scale, rounded once
    vals = (synthetic.bf16_bits_to_f32(fq) if dtype == "bf16" else fq).astype(np.float64)
    xs = (synthetic.bf16_bits_to_f32(x) if dtype == "bf16" else x).astype(np.float64)
    b0 = xs.reshape(-1)[:32]
    c, byte = oracle_block_bruteforce(fmt, b0)
    expect = library_table(fmt)[c] * 2.0 ** (byte - 127)
    assert np.array_equal(vals.reshape(-1)[:32], expect)


@pytest.mark.parametrize("fmt", ALL_FORMATS)
def test_fake_quantize_idempotent_and_error_bound(fmt):
    x = synthetic.gaussian((16, 128), 1.0, seed=12, sid=0, dtype="f32")
    fq = oracle.fake_quantize(x, fmt)
    assert np.array_equal(oracle.fake_quantize(fq, fmt), fq)
    xs = x.reshape(-1, 32).astype(np.float64)
    q = fq.reshape(-1, 32).astype(np.float64)
    t = library_table(fmt)
    mags = np.sort(np.abs(t[~np.isnan(t)]))
    for b in range(xs.shape[0]):
        c, byte = oracle_block_bruteforce(fmt, xs[b])
        s = 2.0 ** (byte - 127)
        y = np.abs(xs[b]) / s
        unsat = y <= oracle.maxval(fmt)
        # error <= half of the local grid step
        idx = np.clip(np.searchsorted(mags, y), 1, mags.size - 1)
        step = mags[idx] - mags[idx - 1]
        err = np.abs(q[b] - xs[b]) / s
        assert np.all(err[unsat] <= step[unsat] / 2 + 1e-12)


def test_dequantize_nan_rules():
    codes = np.zeros((1, 32), np.uint8)
    scales = np.array([[0xFF]], np.uint8)
    out = oracle.dequantize(codes, scales, "mxfp8", (1, 32), "f32")
    assert np.all(out.view(np.uint32) == 0x7FC00000)
    codes[0, 3] = 0x7F  # E4M3 NaN code with a normal scale
    scales[0, 0] = 127
    out = oracle.dequantize(codes, scales, "mxfp8", (1, 32), "bf16")
    assert out[0, 3] == 0x7FC0 and out[0, 0] == 0
    # AXS-6 header: the config bits are not read
    c6 = np.zeros((1, 24), np.uint8)
    c6[0, 0] = 16  # code 16 = 1.0
    h = np.array([[127 | (3 << 8)]], np.uint16)
    out = oracle.dequantize(c6, h, "axs6", (1, 32), "f32")
    assert out[0, 0] == 1.0


def test_rejects_bad_shapes():
    with pytest.raises(ValueError):
        oracle.quantize(np.zeros((2, 48), np.float32), "mxfp8")


# ---- fp32 exponential -------------------------------------------------------------

def nearest_f32(dec):
    """Nearest float32 to an exact Decimal (no double rounding)."""
    getcontext().prec = 80
    f = np.float32(float(dec))
    cands = [np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))]
    return min(cands, key=lambda c: abs(Decimal(float(c)) - dec))


def test_exp_constants_derive_from_ln2():
    """The hex literals in oracle.c are the roundings of ln 2 and 1/k! they claim to be."""
    getcontext().prec = 80
    ln2 = Decimal(2).ln()
    src = open(os.path.join(os.path.dirname(oracle.__file__), "oracle.c")).read()
    L2E = np.float32(float.fromhex("0x1.715476p+0"))
    HI = np.float32(float.fromhex("0x1.62e4p-1"))
    LO = np.float32(float.fromhex("0x1.7f7d1cp-20"))
    for lit in ["0x1.715476p+0f", "0x1.62e4p-1f", "0x1.7f7d1cp-20f"]:
        assert lit in src
    assert L2E == nearest_f32(1 / ln2)
    scale = Decimal(2) ** 16  # ln 2 in [0.5, 1): 16 significant bits
    assert Decimal(float(HI)) == Decimal(int(ln2 * scale)) / scale
    assert LO == nearest_f32(ln2 - Decimal(float(HI)))
    lits = ["0x1p+0f", "0x1p+0f", "0x1p-1f", "0x1.555556p-3f", "0x1.555556p-5f",
            "0x1.111112p-7f", "0x1.6c16c2p-10f", "0x1.a01a02p-13f"]
    for k, lit in enumerate(lits):
        assert lit in src
        assert np.float32(float.fromhex(lit[:-1])) == nearest_f32(Decimal(1) / Decimal(math.factorial(k)))


def ulp_f32(x):
    x = np.float32(abs(x))
    return float(np.nextafter(x, np.float32(np.inf)) - x)


def test_expf_accuracy_and_specials():
    d = np.linspace(-87.0, 0.0, 60001, dtype=np.float32)
    d = np.concatenate([d, -np.abs(np.random.default_rng(1).standard_normal(20000).astype(np.float32)) * 6])
    got = oracle.expf(d).astype(np.float64)
    ref = np.exp(d.astype(np.float64))
    ulps = np.abs(got - ref) / np.array([ulp_f32(r) for r in ref])
    assert ulps.max() <= 2.0, ulps.max()
    assert oracle.expf(np.float32(0.0)) == 1.0
    assert oracle.expf(np.float32(-np.inf)) == 0.0
    assert np.isnan(oracle.expf(np.float32(np.nan)))
    # gradual underflow region: still the nearest subnormal within 2 of its ulps
    dd = np.linspace(-103.0, -88.0, 2001, dtype=np.float32)
    g = oracle.expf(dd).astype(np.float64)
    r = np.exp(dd.astype(np.float64))
    assert np.all(np.abs(g - r) <= 2 * 2.0 ** -149 + 2 * np.abs(r) * 2.0 ** -23)


def test_exp_quantize_worked_value_and_composition():
    s = synthetic.attention_scores(seed=4, heads=1, queries=4, keys=1024)
    codes, scales = oracle.exp_quantize(s, "mxfp4")
    m = s.max(axis=1)
    for r in range(s.shape[0]):
        j = int(np.argmax(s[r]))
        b = j // 32
        assert scales[r, b] == 125  # p = 1.0 -> floor(log2 1) - 2 + 127
        block = codes[r, 16 * b:16 * b + 16]
        code = (block[(j % 32) // 2] >> (4 * (j % 2))) & 0xF
        assert code == 0x6  # E2M1 4.0 = 1.0 / 2^-2
    # no code carries a sign bit
    assert not np.any(codes & 0x88)
    # composition: materialize p with numpy fp32 subtraction and the oracle's exp, then quantize
    d = (s - m[:, None]).astype(np.float32)
    p = oracle.expf(d)
    c2, s2 = oracle.quantize(p, "mxfp4")
    assert np.array_equal(codes, c2) and np.array_equal(scales, s2)


# ---- the input generator (shared by both sides; holds none of the method) ----------

def test_inputs_deterministic_and_distributed():
    a = synthetic.gaussian((64, 256), 0.02, seed=1, dtype="bf16")
    b = synthetic.gaussian((64, 256), 0.02, seed=1, dtype="bf16")
    assert np.array_equal(a, b)
    f = synthetic.bf16_bits_to_f32(a)
    assert abs(f.std() - 0.02) < 0.002 and abs(f.mean()) < 0.002
    w, pos = synthetic.weight_with_outliers(seed=1, shape=(256, 256))
    assert pos.size == round(0.001 * 256 * 256) and np.unique(pos).size == pos.size
    ch = synthetic.outlier_channels()
    assert len(set(ch)) == 16 and all(0 <= c < 8192 for c in ch)
    x = synthetic.student_t_activations(shape=(64, 8192))
    xs = synthetic.student_t_activations(shape=(64, 8192), row_start=10, rows=5)
    assert np.array_equal(x[10:15], xs)
    s = synthetic.attention_scores(heads=1, queries=8, keys=4096)
    s2 = synthetic.attention_scores(heads=1, queries=8, keys=4096, row_start=3, rows=2)
    assert np.array_equal(s[3:5], s2)


# ---- the fp32 exponential, re-evaluated step by step in exact rational arithmetic ----

from fractions import Fraction


def f32_round(q):
    """Exact rational -> nearest binary32 (ties to even, gradual underflow, overflow to inf)."""
    q = Fraction(q)
    if q == 0:
        return 0.0
    sign = -1.0 if q < 0 else 1.0
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, -126)
    ulp = Fraction(2) ** (e - 23)
    n = a / ulp
    lo = n.numerator // n.denominator
    rem = n - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    r = lo * ulp
    if r >= Fraction(2) ** 128:
        return sign * math.inf
    return sign * float(r)


def expf_by_definition(d):
    L2E = float.fromhex("0x1.715476p+0")
    HI = float.fromhex("0x1.62e4p-1")
    LO = float.fromhex("0x1.7f7d1cp-20")
    C = [Fraction(float.fromhex(s)) for s in ["0x1p+0", "0x1p+0", "0x1p-1", "0x1.555556p-3", "0x1.555556p-5",
                                              "0x1.111112p-7", "0x1.6c16c2p-10", "0x1.a01a02p-13"]]
    D = Fraction(d)
    t = f32_round(D * Fraction(L2E))
    if t < -160:
        return 0.0
    n = round(t)  # ties to even
    r = f32_round(D - n * Fraction(HI))
    r = f32_round(Fraction(r) - n * Fraction(LO))
    p = float(C[7])
    for k in range(6, -1, -1):
        p = f32_round(Fraction(p) * Fraction(r) + C[k])
    if n < -126:
        return f32_round(Fraction(f32_round(Fraction(p) * Fraction(2) ** (n + 64))) * Fraction(2) ** -64)
    return f32_round(Fraction(p) * Fraction(2) ** n)


def test_expf_is_the_stated_algorithm_bit_for_bit():
    rng = np.random.default_rng(21)
    d = np.concatenate([-np.abs(rng.standard_normal(1500)).astype(np.float32) * 8,
                        -rng.uniform(0, 104, 500).astype(np.float32),
                        np.float32([-0.0, -1e-30, -0.34657359, -0.3465736, -88.0, -87.33655, -103.2])])
    got = oracle.expf(d)
    for di, g in zip(d, got):
        want = expf_by_definition(float(di))
        assert np.float32(want).view(np.uint32) == np.float32(g).view(np.uint32), (di, g, want)
