"""Seeded synthetic inputs for block-scaled quantization workloads.

This module holds no arithmetic of the method: it only draws the input
tensors that both the CUDA path and the CPU oracle are fed, on the host, so
both sides see identical bits.

Generator (stated once, used everywhere):
  * SplitMix64 (Steele, Lea & Flood, 2014) run in counter mode: the i-th
    64-bit word of stream (seed, sid) is mix64(key + (i+1)*GOLDEN) with
    key = mix64(mix64(seed) + sid*GOLDEN).
  * uniforms: u = (word >> 11) * 2^-53; the first Box-Muller operand uses
    (word >> 11) + 1 so it lies in (0, 1].
  * normals: Box-Muller (1958) in float64, words 2j and 2j+1 giving
    elements 2j (cosine branch) and 2j+1 (sine branch).
  * values are built in float64, rounded to float32 (nearest even) and, for
    bf16 tensors, from float32 to bf16 (nearest even).
bf16 tensors are returned as numpy uint16 bit patterns.
"""
from concurrent.futures import ThreadPoolExecutor
import os

import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 21
_THREADS = max(1, min(16, os.cpu_count() or 1))


def _mix64(z):
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _key(seed, sid):
    with np.errstate(over="ignore"):
        k0 = _mix64(np.array([seed], dtype=np.uint64))
        return _mix64(k0 + np.uint64(sid) * GOLDEN)[0]


def words(seed, sid, start, count):
    """count 64-bit words of stream (seed, sid) starting at counter `start`."""
    key = _key(seed, sid)
    i = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(key + i * GOLDEN)


def _normals_chunk(seed, sid, start, count):
    # start and count are even: pairs (2j, 2j+1) stay together
    w = words(seed, sid, start, count)
    a = w[0::2]
    b = w[1::2]
    u1 = ((a >> np.uint64(11)) + np.uint64(1)).astype(np.float64) * 2.0 ** -53
    u2 = (b >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
    rad = np.sqrt(-2.0 * np.log(u1))
    ang = 2.0 * np.pi * u2
    out = np.empty(count, dtype=np.float64)
    out[0::2] = rad * np.cos(ang)
    out[1::2] = rad * np.sin(ang)
    return out


def normals(seed, sid, n, start=0):
    """n standard normals (float64) of stream (seed, sid), from element `start` (even)."""
    assert start % 2 == 0
    m = n + (n & 1)
    out = np.empty(m, dtype=np.float64)
    spans = [(s, min(_CHUNK, m - s)) for s in range(0, m, _CHUNK)]

    def work(span):
        s, c = span
        out[s:s + c] = _normals_chunk(seed, sid, start + s, c)

    if len(spans) > 1:
        with ThreadPoolExecutor(_THREADS) as ex:
            list(ex.map(work, spans))
    else:
        for sp in spans:
            work(sp)
    return out[:n]


def uniform_ints(seed, sid, count, bound):
    """count draws of uniform integers in [0, bound) (multiply-shift on 53 bits)."""
    w = words(seed, sid, 0, count)
    return [int((int(x) >> 11) * bound >> 53) for x in w]


def to_f32(v):
    return np.asarray(v, dtype=np.float64).astype(np.float32)


def f32_to_bf16_bits(f):
    """float32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(f, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(h):
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def floyd_sample(seed, sid, n, k):
    """k distinct positions in [0, n), uniformly without replacement (Floyd)."""
    draws = words(seed, sid, 0, k)
    chosen = set()
    for t, j in enumerate(range(n - k, n)):
        r = (int(draws[t]) >> 11) * (j + 1) >> 53
        chosen.add(j if r in chosen else r)
    return np.array(sorted(chosen), dtype=np.int64)


# ---- the five workloads --------------------------------------------------------

def gaussian(shape, std, seed, sid=0, dtype="f32"):
    n = int(np.prod(shape))
    v = normals(seed, sid, n) * std
    f = to_f32(v).reshape(shape)
    return f if dtype == "f32" else f32_to_bf16_bits(f)


def quickstart_fp32(seed=0, shape=(128, 256)):
    """fp32 N(0, 1) tensor (AXS-6 quick-start shape 128 x 256)."""
    return gaussian(shape, 1.0, seed, 0, "f32")


def weight_with_outliers(seed=1, shape=(4096, 4096), std=0.02, frac=0.001, mult=50.0):
    """bf16 weight N(0, std) with round(frac*N) distinct uniform positions times `mult`."""
    n = int(np.prod(shape))
    v = normals(seed, 0, n) * std
    k = int(round(frac * n))
    pos = floyd_sample(seed, 1, n, k)
    v[pos] *= mult
    return f32_to_bf16_bits(to_f32(v)).reshape(shape), pos


DECODER_LAYER = (  # nn.Linear storage [out, in]; the input dim is contiguous
    ("q", 4096, 2560), ("k", 1024, 2560), ("v", 1024, 2560), ("o", 2560, 4096),
    ("gate", 9728, 2560), ("up", 9728, 2560), ("down", 2560, 9728))
N_LAYERS = 36


def decoder_weight(layer, k, seed=2, std=0.02):
    """bf16 N(0, std) weight k of a decoder layer; stream id = layer*7 + k."""
    _, rows, cols = DECODER_LAYER[k]
    return gaussian((rows, cols), std, seed, layer * 7 + k, "bf16")


def outlier_channels(seed=3, hidden=8192, count=16):
    """The first `count` distinct draws of uniform[0, hidden) from stream (seed, 9)."""
    out = []
    t = 0
    while len(out) < count:
        for c in uniform_ints_from(seed, 9, t, 64, hidden):
            if c not in out:
                out.append(c)
                if len(out) == count:
                    break
        t += 64
    return out


def uniform_ints_from(seed, sid, start, count, bound):
    w = words(seed, sid, start, count)
    return [int((int(x) >> 11) * bound >> 53) for x in w]


def student_t_activations(seed=3, shape=(16384, 8192), nu=3, scale=0.5, out_mult=100.0,
                          row_start=0, rows=None):
    """bf16 activations scale * t(nu=3) with 16 fixed outlier channels x out_mult.

    t = Z0 / sqrt((Z1^2 + Z2^2 + Z3^2) / 3), Z_k from streams (seed, 10 + k).
    `row_start`/`rows` draw a row slice of the same tensor.
    """
    assert nu == 3
    R, H = shape
    rows = R if rows is None else rows
    start = row_start * H
    n = rows * H
    z = [normals(seed, 10 + k, n + (start & 1), start - (start & 1))[(start & 1):] for k in range(4)]
    t = z[0] / np.sqrt((z[1] ** 2 + z[2] ** 2 + z[3] ** 2) / 3.0)
    v = (t * scale).reshape(rows, H)
    ch = outlier_channels(seed, H)
    v[:, ch] *= out_mult
    return f32_to_bf16_bits(to_f32(v))


def gradients_fp32(seed=3, shape=(16384, 8192), std=1e-3, row_start=0, rows=None):
    """fp32 gradients N(0, std), stream (seed, 20)."""
    R, H = shape
    rows = R if rows is None else rows
    start = row_start * H
    n = rows * H
    v = normals(seed, 20, n + (start & 1), start - (start & 1))[(start & 1):] * std
    return to_f32(v).reshape(rows, H)


def attention_scores(seed=4, heads=32, queries=128, keys=32768, std=3.0, row_start=0, rows=None):
    """fp32 scores N(0, std) viewed as [heads*queries, keys], stream (seed, 0)."""
    R = heads * queries
    rows = R if rows is None else rows
    start = row_start * keys
    v = normals(seed, 0, rows * keys, start) * std
    return to_f32(v).reshape(rows, keys)
