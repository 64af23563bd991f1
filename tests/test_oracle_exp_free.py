"""Pins for the oracle's exp-free E2M1 rule ("EFQ-Softmax: exp-free E2M1 probabilities",
opening paragraph and the paragraph on the per-block rule: exponent-only scale from the
block's local maximum, then one affine rule from shifted scores to nonnegative E2M1 codes).

The page gives no constants, so the rule is a reading (code = clamp(rint(2u - 2Es) + 2, 0, 7)
with u = (s - rowmax)/ln 2 and Es = floor(max u) - 2) and its parity against the paper is
unpinned. What the tests below pin is that reading against things other than itself:
- the exp-then-quantize oracle (pinned separately, through its own exponential): same scale
  bytes on special rows, same codes wherever the probability is a power of two (even codes),
  and never more than one code apart, a property of the two roundings on the E2M1 grid
  (linear nearest vs nearest on the log line) that a wrong slope or offset breaks;
- closed forms: the row-maximum key is probability 1 = E2M1 4.0 x 2^-2 (byte 125, code 6);
- invariants: codes nondecreasing in the score within a block, sign bits 0, invariance under
  an exactly representable shift of a whole row.
"""
import math

import numpy as np
import pytest

import oracle
import synthetic

L2E = np.float32(1.0 / math.log(2.0))


def nibbles(codes):
    """[rows, bytes] packed E2M1 codes -> [rows, 2 * bytes] codes (low nibble first)."""
    lo = codes & 0xF
    hi = codes >> 4
    return np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)


def e2m1_grid():
    return np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)


def test_row_maximum_key_is_probability_one():
    s = synthetic.attention_scores(seed=4, heads=1, queries=16, keys=1024)
    codes, scales = oracle.exp_free_quantize(s)
    c = nibbles(codes)
    for r in range(s.shape[0]):
        j = int(np.argmax(s[r]))
        assert scales[r, j // 32] == 125          # floor(log2 1) - 2 + 127
        assert c[r, j] == 6                       # E2M1 4.0 = 1.0 / 2^-2
    assert np.all(c < 8)                          # sign bits are 0: probabilities are nonnegative


def key_with_power_of_two_probability(k, at_least=False):
    """An fp32 shifted score d with RN(d * L2E) == k (k <= 0 integer), searched near k ln 2; with
    at_least, also the exp-then-quantize oracle's exponential of d >= 2^k (so both rules see the
    same block scale). None if there is no such d."""
    d0 = np.float32(k * math.log(2.0))
    cands = [d0]
    up, dn = d0, d0
    for _ in range(256):
        up = np.nextafter(up, np.float32(np.inf), dtype=np.float32)
        dn = np.nextafter(dn, np.float32(-np.inf), dtype=np.float32)
        cands += [up, dn]
    for d in cands:
        if np.float32(d * L2E) == k and (not at_least or oracle.expf(np.array([d], np.float32))[0] >= np.float32(2.0 ** k)):
            return np.float32(d)
    return None


def test_even_codes_are_exact_powers_of_two_and_match_exp_then_quantize():
    # key 0 of each row holds the row maximum (d = 0); block 1's maximum has log2 p = k exactly,
    # its second key log2 p = k - lead, i.e. v = 2 - lead above the block scale: code 2v + 2
    cases = []
    for k in range(0, -126, -1):
        d = key_with_power_of_two_probability(k, at_least=True)
        if d is None:
            continue
        for lead in (0, 1, 2):
            d2 = key_with_power_of_two_probability(k - lead) if k - lead >= -125 else None
            if d2 is not None:
                cases.append((k, lead, d, d2))
    assert len(cases) > 100
    s = np.full((len(cases), 64), -1e4, dtype=np.float32)
    for i, (k, lead, d, d2) in enumerate(cases):
        s[i, 0], s[i, 32], s[i, 33] = 0.0, d, d2
    codes, scales = oracle.exp_free_quantize(s)
    c = nibbles(codes)
    ec, es = oracle.exp_quantize(s, "mxfp4")
    e = nibbles(ec)
    for i, (k, lead, _, _) in enumerate(cases):
        assert scales[i, 1] == max(k - 2, -127) + 127 == es[i, 1]
        assert c[i, 32] == 6 == e[i, 32]
        want = 2 * (2 - lead) + 2 if k - 2 >= -127 else None  # value 2^(2 - lead) exactly
        if want is not None:
            assert c[i, 33] == want == e[i, 33], (k, lead, c[i, 33], e[i, 33])


@pytest.mark.parametrize("seed,sigma", [(4, 3.0), (7, 1.0), (9, 8.0)])
def test_within_one_code_of_exp_then_quantize(seed, sigma):
    s = synthetic.attention_scores(seed=seed, heads=1, queries=32, keys=2048) * np.float32(sigma / 3.0)
    s = s.astype(np.float32)
    codes, scales = oracle.exp_free_quantize(s)
    ec, es = oracle.exp_quantize(s, "mxfp4")
    same = scales == es
    assert same.mean() > 0.999           # the two block scales differ only where exp(d_max) rounds across 2^k
    c, e = nibbles(codes).astype(int), nibbles(ec).astype(int)
    blk = np.repeat(same, 32, axis=1)
    assert np.abs(c - e)[blk].max() <= 1
    assert (c == e)[blk].mean() > 0.6    # most keys agree; the rest sit between two grid points


def test_within_one_code_over_the_whole_normalized_range():
    # brute force over y = p / 2^Es in [2^-12, 8): linear nearest E2M1 (ties to the even code)
    # vs the affine rule on the log line
    g = e2m1_grid()
    ys = np.exp2(np.linspace(-12, 3, 200001)[:-1])
    lin = np.array([int(np.argmin(np.abs(g - y) + 1e-12 * np.arange(8))) for y in ys[::50]])
    log = np.clip(np.rint(2 * np.log2(ys[::50])) + 2, 0, 7).astype(int)
    assert np.abs(lin - log).max() <= 1
    # and a slope or offset off by one breaks it
    assert np.abs(lin - np.clip(np.rint(np.log2(ys[::50])) + 2, 0, 7)).max() > 1
    assert np.abs(lin - np.clip(np.rint(2 * np.log2(ys[::50])) + 4, 0, 7)).max() > 1


def test_codes_nondecreasing_in_the_score_within_a_block():
    s = synthetic.attention_scores(seed=11, heads=1, queries=8, keys=4096)
    codes, _ = oracle.exp_free_quantize(s)
    c = nibbles(codes)
    for r in range(s.shape[0]):
        for b in range(s.shape[1] // 32):
            o = np.argsort(s[r, 32 * b:32 * b + 32], kind="stable")
            assert np.all(np.diff(c[r, 32 * b + o].astype(int)) >= 0)


def test_invariant_under_an_exact_shift_of_the_row():
    rng = np.random.default_rng(3)
    s = (np.round(rng.normal(0, 3, size=(8, 512)) * 64) / 64).astype(np.float32)
    c0, s0 = oracle.exp_free_quantize(s)
    c1, s1 = oracle.exp_free_quantize(s + np.float32(37.0))
    assert np.array_equal(c0, c1) and np.array_equal(s0, s1)


def test_special_rows_match_exp_then_quantize_scales():
    s = synthetic.attention_scores(seed=5, heads=1, queries=6, keys=256)
    s[0, 5] = np.nan            # NaN row maximum: every block NaN
    s[1, :] = -np.inf           # no finite key: s - m is NaN everywhere
    s[2, 32:64] = -np.inf       # one block of zero probabilities
    s[3, 7] = np.inf            # +inf maximum: its block NaN, the others zero
    s[4, :] = 0.0               # all probabilities 1
    codes, scales = oracle.exp_free_quantize(s)
    ec, es = oracle.exp_quantize(s, "mxfp4")
    assert np.array_equal(scales[:5], es[:5])
    assert np.all(scales[0] == 0xFF) and np.all(codes[0] == 0)
    assert np.all(scales[1] == 0xFF)
    assert scales[2, 1] == 0 and np.all(codes[2, 16:32] == 0)
    assert scales[3, 0] == 0xFF and np.all(scales[3, 1:] == 0)
    assert np.all(scales[4] == 125) and np.all(nibbles(codes)[4] == 6)
