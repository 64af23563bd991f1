"""Pins for the oracle's eXmY formats ("eXmY" abstract: any width, any split of
exponent and mantissa bits, dense packing).

- where a split coincides with a named format, the results coincide: e2m1 /
  e2m3 / e3m2 with MXFP4 / MXFP6, e0m5 with AXS-6 (codes and scale values);
- e4m3 / e5m2 / e3m4 decode tables equal ml_dtypes' float8 tables on every code
  those types do not reserve for Inf/NaN;
- structure of every supported split: 2^(E+M) increasing magnitudes, the
  largest (2 - 2^-M) 2^emax (E >= 1) or (2^M - 1) / 2^(M-1) (E = 0), the
  smallest 2^(1-b-M);
- rounding = brute-force nearest magnitude (ties to the even code), all splits.
"""
import ml_dtypes
import numpy as np
import pytest

import oracle
import synthetic

SPLITS = [(E, M) for W in range(3, 10) for E in range(0, 6) for M in [W - 1 - E] if oracle.exmy_valid(E, M)]


def test_split_list_covers_the_abstract_examples():
    ws = {1 + E + M for E, M in SPLITS}
    assert {3, 5, 6, 7, 9} <= ws
    seven = sorted(E for E, M in SPLITS if 1 + E + M == 7)
    assert seven == [0, 1, 2, 3, 4, 5]  # e0m6 .. e5m1 (e6m0 has no mantissa: not supported)


@pytest.mark.parametrize("E,M", SPLITS)
def test_structure(E, M):
    t = oracle.exmy_decode_table(E, M)
    half = t.size // 2
    mags = t[:half]
    assert half == 2 ** (E + M)
    assert np.all(np.diff(mags) > 0)
    assert np.array_equal(t[half:], -mags) and np.signbit(t[half])
    if E >= 1:
        b = 2 ** (E - 1) - 1
        emax = 2 ** (E - 1)
        assert mags[-1] == (2 - 2.0 ** -M) * 2.0 ** emax
        assert mags[1] == 2.0 ** (1 - b - M)
    else:
        emax = 0
        assert mags[-1] == (2 ** M - 1) / 2 ** (M - 1)
        assert mags[1] == 2.0 ** (1 - M)
    assert oracle.exmy_emax(E, M) == emax == int(np.floor(np.log2(mags[-1])))
    assert oracle.exmy_maxval(E, M) == mags[-1]


@pytest.mark.parametrize("E,M,lib", [(4, 3, ml_dtypes.float8_e4m3fn), (5, 2, ml_dtypes.float8_e5m2),
                                     (3, 4, getattr(ml_dtypes, "float8_e3m4", None))])
def test_float8_tables_match_ml_dtypes(E, M, lib):
    if lib is None:
        pytest.skip("ml_dtypes has no such type")
    ref = np.arange(256, dtype=np.uint8).view(lib).astype(np.float64)
    ours = oracle.exmy_decode_table(E, M)
    ok = np.isfinite(ref)
    assert np.array_equal(ours[ok], ref[ok])
    assert np.all(np.isfinite(ours))  # eXmY reserves no code


@pytest.mark.parametrize("E,M,fmt", [(2, 1, "mxfp4"), (2, 3, "mxfp6_e2m3"), (3, 2, "mxfp6_e3m2"), (0, 5, "axs6")])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_named_formats_coincide(E, M, fmt, dtype):
    x = synthetic.gaussian((33, 96), 1.0, seed=31, dtype=dtype)
    c1, s1 = oracle.quantize_exmy(x, E, M)
    c2, s2 = oracle.quantize(x, fmt)
    assert np.array_equal(c1, c2)
    assert np.array_equal(s1.astype(np.uint16), s2.astype(np.uint16) & 0xFF)
    assert np.array_equal(oracle.dequantize_exmy(c1, s1, E, M, x.shape, dtype).view(np.uint8),
                          oracle.dequantize(c2, s2, fmt, x.shape, dtype).view(np.uint8))
    assert np.array_equal(oracle.decode_table(fmt), oracle.exmy_decode_table(E, M))


def brute(E, M, y):
    t = oracle.exmy_decode_table(E, M)
    mags = t[: t.size // 2]
    codes = np.arange(mags.size)
    d = np.abs(y[:, None] - mags[None, :])
    tie = d == d.min(axis=1, keepdims=True)
    score = np.where(tie, codes[None, :] % 2, 2)
    return codes[np.argmin(score, axis=1)].astype(np.uint32)


@pytest.mark.parametrize("E,M", SPLITS)
def test_rounding_bruteforce(E, M):
    mx = oracle.exmy_maxval(E, M)
    t = oracle.exmy_decode_table(E, M)
    mags = t[: t.size // 2]
    mids = (mags[:-1] + mags[1:]) / 2
    rng = np.random.default_rng(E * 16 + M)
    y = np.concatenate([mids, np.nextafter(mids, 0), np.nextafter(mids, 9), mags, [mx * 1.5, 0.0],
                        rng.uniform(0, mx * 1.2, 20000)])
    assert np.array_equal(oracle.exmy_round_mags(E, M, y), brute(E, M, y))


@pytest.mark.parametrize("E,M", [(0, 2), (1, 3), (2, 4), (3, 3), (4, 4), (5, 3), (1, 1)])
def test_payload_is_w_words(E, M):
    x = synthetic.gaussian((2, 64), 1.0, seed=3, dtype="f32")
    c, s = oracle.quantize_exmy(x, E, M)
    assert c.shape[1] == 2 * 4 * (1 + E + M)
    fq = oracle.fake_quantize_exmy(x, E, M)
    assert np.array_equal(fq.view(np.uint32), oracle.dequantize_exmy(c, s, E, M, x.shape, "f32").view(np.uint32))


def test_rejects_unsupported_splits():
    with pytest.raises(ValueError):
        oracle.quantize_exmy(np.zeros((1, 32), np.float32), 6, 2)
    with pytest.raises(ValueError):
        oracle.quantize_exmy(np.zeros((1, 32), np.float32), 1, 8)
