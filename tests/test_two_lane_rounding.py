"""CPU check, exhaustive over bf16 magnitudes, of the rounding recipe the library's eXmY quantize
uses for bf16 values with M <= 5: two values per 32-bit word, bf16x2 arithmetic for the scaling
and the rounding, 16-bit-lane integer arithmetic for the codes. The recipe is emulated step by
step on words that hold two bf16 lanes (products and sums rounded to bf16 to nearest even with
ml_dtypes, integer steps in uint32 words, so a carry between the lanes would show):
    y    = RN_bf16(x * 2^(127 - byte)) & 0x7FFF7FFF
    e    = max_u16x2(y & 0x7F807F80, (128 - b) << 7)      (exponent field, at least 1 - b)
    c    = e + (((7 - M) << 7) | 0x40)                     (bits of 1.5 * 2^(e + 7 - M))
    q    = RN_bf16(y + c) - c                              (steps of 2^(e - M), ties to even)
    code = min_u16x2((e >> (7 - M)) + q - ((128 - b) << M), 2^(E + M) - 1)
and compared, lane by lane, with the oracle's nearest-code rounding of the exact |x| / 2^(byte -
127), for every finite bf16 magnitude, every split with M <= 5 and scale bytes across the range,
restricted to what a block can hold (|x| / 2^(byte - 127) < 2^(emax + 1): the block maximum
fixes the byte). Also the fused eXmY fake-quantize's grid value, r = RN(RN(y + C) - C) in fp32
with C = 1.5 * 2^(e + 23 - M), clamped: equal to the decoded nearest code for every split. CPU
checks of the recipes' exactness; the GPU tests check the kernels that implement them."""
import ml_dtypes
import numpy as np
import pytest

import oracle

SPLITS = [(E, M) for W in range(3, 10) for E in range(0, 6) for M in [W - 1 - E]
          if oracle.exmy_valid(E, M) and M <= 5]
BYTES = [0, 1, 2, 3, 10, 60, 100, 118, 124, 125, 126, 127, 128, 129, 130, 134, 140, 170, 200, 250, 253]


def bf16_bits_to_f64(h):
    return h.astype(np.uint16).view(ml_dtypes.bfloat16).astype(np.float64)


def f64_to_bf16_bits(v):
    # float64 -> float32 is exact for these values (8-bit significands, or far below any grid
    # step, where only code 0 matters), then round to bf16, nearest even
    return v.astype(np.float32).astype(ml_dtypes.bfloat16).view(np.uint16).astype(np.uint32)


def lanes(w):
    return w & np.uint32(0xFFFF), w >> np.uint32(16)


def join(lo, hi):
    return (hi << np.uint32(16)) | lo


def max_u16x2(a, b):
    al, ah = lanes(a)
    bl, bh = lanes(b)
    return join(np.maximum(al, bl), np.maximum(ah, bh))


def min_u16x2(a, b):
    al, ah = lanes(a)
    bl, bh = lanes(b)
    return join(np.minimum(al, bl), np.minimum(ah, bh))


def bf16x2_mul_pow2(w, k):
    lo, hi = lanes(w)
    s = 2.0 ** k
    return join(f64_to_bf16_bits(bf16_bits_to_f64(lo) * s), f64_to_bf16_bits(bf16_bits_to_f64(hi) * s))


def bf16x2_add(a, b):
    al, ah = lanes(a)
    bl, bh = lanes(b)
    return join(f64_to_bf16_bits(bf16_bits_to_f64(al) + bf16_bits_to_f64(bl)),
                f64_to_bf16_bits(bf16_bits_to_f64(ah) + bf16_bits_to_f64(bh)))


def two_lane_codes(w, byte, E, M):
    b = (1 << (E - 1)) - 1 if E >= 1 else 0
    emin2 = np.uint32(((128 - b) << 7) * 0x10001)
    cadd2 = np.uint32((((7 - M) << 7) | 0x40) * 0x10001)
    kneg2 = np.uint32((-((((128 - b) << M) * 0x10001))) & 0xFFFFFFFF)
    max2 = np.uint32(((1 << (E + M)) - 1) * 0x10001)
    y = bf16x2_mul_pow2(w, 127 - byte) & np.uint32(0x7FFF7FFF)
    e = max_u16x2(y & np.uint32(0x7F807F80), emin2)
    c = e + cadd2
    q = bf16x2_add(y, c) - c
    return min_u16x2((e >> np.uint32(7 - M)) + q + kneg2, max2)


@pytest.mark.parametrize("E,M", SPLITS)
def test_two_lane_rounding_equals_the_oracle_for_every_bf16_magnitude(E, M):
    emax = oracle.exmy_emax(E, M)
    mags = np.arange(0x7F80, dtype=np.uint32)  # every finite bf16 magnitude, +0 included
    rng = np.random.default_rng(E * 10 + M)
    for byte in BYTES:
        y_exact = bf16_bits_to_f64(mags) * 2.0 ** (127 - byte)
        ok = y_exact < 2.0 ** (emax + 1)  # what a block with this scale byte can hold
        lo = np.where(ok, mags, 0).astype(np.uint32)
        hi = lo[rng.permutation(lo.size)]
        signs = rng.integers(0, 2, (2, lo.size)).astype(np.uint32)
        w = join(lo | (signs[0] << np.uint32(15)), hi | (signs[1] << np.uint32(15)))
        got_lo, got_hi = lanes(two_lane_codes(w, byte, E, M))
        want_lo = oracle.exmy_round_mags(E, M, bf16_bits_to_f64(lo) * 2.0 ** (127 - byte))
        want_hi = oracle.exmy_round_mags(E, M, bf16_bits_to_f64(hi) * 2.0 ** (127 - byte))
        assert np.array_equal(got_lo, want_lo), (E, M, byte, np.flatnonzero(got_lo != want_lo)[:5])
        assert np.array_equal(got_hi, want_hi), (E, M, byte)


def test_the_recipe_needs_m_at_most_5():
    # with M = 6 the sum y + c can leave c's binade: the recipe is not used there
    E, M = 2, 6
    mags = np.arange(0x3F80, 0x4100, dtype=np.uint32)  # around 1.0 .. 8.0
    byte = 127
    got_lo, _ = lanes(two_lane_codes(join(mags, np.zeros_like(mags)), byte, E, M))
    want = oracle.exmy_round_mags(E, M, bf16_bits_to_f64(mags))
    assert not np.array_equal(got_lo, want)


ALL_SPLITS = [(E, M) for W in range(3, 10) for E in range(0, 6) for M in [W - 1 - E] if oracle.exmy_valid(E, M)]


def round_value_recipe(y, E, M):
    """The fused fake-quantize's grid value, emulated in fp32 (numpy float32 arithmetic rounds to
    nearest even): C = 1.5 * 2^(e + 23 - M) with e = max(exponent of y, 1 - b), r = (y + C) - C,
    clamped to the largest value."""
    b = (1 << (E - 1)) - 1 if E >= 1 else 0
    emin_b = np.uint32(128 - b)
    cadd = np.uint32(((23 - M) << 23) | 0x400000)
    eb = np.maximum(y.view(np.uint32) >> np.uint32(23), emin_b)
    c = (eb * np.uint32(0x800000) + cadd).view(np.float32)
    r = (y + c) - c
    return np.minimum(r, np.float32(oracle.exmy_maxval(E, M)))


@pytest.mark.parametrize("E,M", ALL_SPLITS)
def test_fused_fake_quantize_value_equals_decoded_nearest_code(E, M):
    emax = oracle.exmy_emax(E, M)
    table = oracle.exmy_decode_table(E, M)
    x = bf16_bits_to_f64(np.arange(0x7F80, dtype=np.uint32))
    for byte in BYTES:
        y64 = x * 2.0 ** (127 - byte)
        y64 = y64[y64 < 2.0 ** (emax + 1)]
        y = y64.astype(np.float32)
        got = round_value_recipe(y, E, M).astype(np.float64)
        want = table[oracle.exmy_round_mags(E, M, y64)]
        assert np.array_equal(got, want), (E, M, byte)
