"""CPU oracle for block-scaled shared-exponent quantization (numpy front end).

TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and the CPU legs of
bench.py (cpu_baseline and --impl reference) may import this package. It wraps
the scalar C oracle in oracle.c (fp64 arithmetic, one block at a time); it
shares no code with the CUDA library and never calls it.

Arrays are numpy: fp32 values as float32, bf16 values as their uint16 bit
patterns. Formats are named "axs6", "mxfp6_e2m3", "mxfp6_e3m2", "mxfp8",
"mxfp4"; value types "f32", "bf16".
"""
import ctypes
import os

import numpy as np

from . import build as _build

FORMATS = {"axs6": 0, "mxfp6_e2m3": 1, "mxfp6_e3m2": 2, "mxfp8": 3, "mxfp4": 4}
DTYPES = {"f32": 0, "bf16": 1}

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        i64, i32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
        L.orc_decode.restype = ctypes.c_double
        L.orc_decode.argtypes = [i32, ctypes.c_uint32]
        L.orc_maxval.restype = ctypes.c_double
        L.orc_maxval.argtypes = [i32]
        L.orc_bits.argtypes = [i32]
        L.orc_emax.argtypes = [i32]
        L.orc_round_mag.restype = ctypes.c_uint32
        L.orc_round_mag.argtypes = [i32, ctypes.c_double]
        L.orc_round_mags.argtypes = [i32, vp, i64, vp]
        L.orc_round_binary.restype = ctypes.c_double
        L.orc_round_binary.argtypes = [ctypes.c_double, i32, i32, i32]
        L.orc_quantize_block.argtypes = [i32, vp, vp]
        L.orc_quantize.argtypes = [i32, vp, i32, i64, i64, vp, vp]
        L.orc_dequantize.argtypes = [i32, vp, vp, i64, i64, vp, i32]
        L.orc_fake_quantize.argtypes = [i32, vp, i32, i64, i64, vp]
        L.orc_exp_quantize.argtypes = [i32, vp, i64, i64, vp, vp]
        L.orc_expf.restype = ctypes.c_float
        L.orc_expf.argtypes = [ctypes.c_float]
        L.orc_exp_free_quantize.argtypes = [vp, i64, i64, vp, vp]
        L.orc_codes_bytes.restype = i64
        L.orc_codes_bytes.argtypes = [i32, i64, i64]
        L.orc_scales_bytes.restype = i64
        L.orc_scales_bytes.argtypes = [i32, i64, i64]
        _lib = L
    return _lib


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _dtype_of(x):
    if x.dtype == np.float32:
        return "f32"
    if x.dtype == np.uint16:
        return "bf16"
    raise TypeError(f"values must be float32 or uint16 (bf16 bits), got {x.dtype}")


def payload_bytes(fmt):
    return 32 * lib().orc_bits(FORMATS[fmt]) // 8


def scale_dtype(fmt):
    return np.uint16 if fmt == "axs6" else np.uint8


def decode(fmt, code):
    """Value of one code (closed form of the element format)."""
    return lib().orc_decode(FORMATS[fmt], int(code))


def decode_table(fmt):
    n = 1 << lib().orc_bits(FORMATS[fmt])
    return np.array([decode(fmt, c) for c in range(n)], dtype=np.float64)


def maxval(fmt):
    return lib().orc_maxval(FORMATS[fmt])


def emax(fmt):
    return lib().orc_emax(FORMATS[fmt])


def bits(fmt):
    return lib().orc_bits(FORMATS[fmt])


def round_mag(fmt, y):
    """Magnitude code of y >= 0 (already divided by the block scale)."""
    return lib().orc_round_mag(FORMATS[fmt], float(y))


def round_mags(fmt, y):
    """Vectorised round_mag over a float64 array."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    out = np.zeros(y.shape, dtype=np.uint32)
    lib().orc_round_mags(FORMATS[fmt], _ptr(y), y.size, _ptr(out))
    return out


def round_binary(v, p, emin, emax_):
    return lib().orc_round_binary(float(v), p, emin, emax_)


def quantize_block(fmt, x):
    """One block of 32 values (any float array) -> (unpacked codes uint32[32], scale byte)."""
    xd = np.ascontiguousarray(np.asarray(x, dtype=np.float64).reshape(32))
    codes = np.zeros(32, dtype=np.uint32)
    byte = lib().orc_quantize_block(FORMATS[fmt], _ptr(xd), _ptr(codes))
    return codes, byte


def quantize(x, fmt):
    """x: [rows, cols] float32 or uint16(bf16 bits) -> (codes uint8[rows, cols/32*payload], scales)."""
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    f = FORMATS[fmt]
    codes = np.zeros((rows, cols // 32 * payload_bytes(fmt)), dtype=np.uint8)
    scales = np.zeros((rows, cols // 32), dtype=scale_dtype(fmt))
    rc = lib().orc_quantize(f, _ptr(x), DTYPES[_dtype_of(x)], rows, cols, _ptr(codes), _ptr(scales))
    if rc:
        raise ValueError(f"oracle quantize rejected the arguments (rc={rc})")
    return codes, scales


def dequantize(codes, scales, fmt, shape, dtype="bf16"):
    rows, cols = shape
    codes = np.ascontiguousarray(codes)
    scales = np.ascontiguousarray(scales)
    out = np.zeros((rows, cols), dtype=np.float32 if dtype == "f32" else np.uint16)
    rc = lib().orc_dequantize(FORMATS[fmt], _ptr(codes), _ptr(scales), rows, cols, _ptr(out), DTYPES[dtype])
    if rc:
        raise ValueError(f"oracle dequantize rejected the arguments (rc={rc})")
    return out


def fake_quantize(x, fmt):
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    out = np.zeros_like(x)
    rc = lib().orc_fake_quantize(FORMATS[fmt], _ptr(x), DTYPES[_dtype_of(x)], rows, cols, _ptr(out))
    if rc:
        raise ValueError(f"oracle fake_quantize rejected the arguments (rc={rc})")
    return out


def expf(d):
    """The method's own fp32 exponential, elementwise over a float32 array."""
    d = np.asarray(d, dtype=np.float32)
    f = lib().orc_expf
    out = np.array([f(float(v)) for v in d.reshape(-1)], dtype=np.float32)
    return out.reshape(d.shape)


def exp_quantize(scores, fmt="mxfp4"):
    """scores: [rows, cols] float32 -> (codes, scales) of exp(s - rowmax) block-quantized."""
    s = np.ascontiguousarray(scores, dtype=np.float32)
    rows, cols = s.shape
    codes = np.zeros((rows, cols // 32 * payload_bytes(fmt)), dtype=np.uint8)
    scales = np.zeros((rows, cols // 32), dtype=scale_dtype(fmt))
    rc = lib().orc_exp_quantize(FORMATS[fmt], _ptr(s), rows, cols, _ptr(codes), _ptr(scales))
    if rc:
        raise ValueError(f"oracle exp_quantize rejected the arguments (rc={rc})")
    return codes, scales


def exp_free_quantize(scores):
    """scores: [rows, cols] float32 -> (codes, scales) of the exp-free E2M1 rule: per block of 32
    shifted scores an exponent-only scale from the block's maximum of u = (s - rowmax)/ln 2 and
    code = clamp(rint(2u - 2Es) + 2, 0, 7) (see oracle.c; constants are a reading of the page)."""
    s = np.ascontiguousarray(scores, dtype=np.float32)
    rows, cols = s.shape
    codes = np.zeros((rows, cols // 32 * payload_bytes("mxfp4")), dtype=np.uint8)
    scales = np.zeros((rows, cols // 32), dtype=np.uint8)
    rc = lib().orc_exp_free_quantize(_ptr(s), rows, cols, _ptr(codes), _ptr(scales))
    if rc:
        raise ValueError(f"oracle exp_free_quantize rejected the arguments (rc={rc})")
    return codes, scales


def unpack_codes(codes_block_bytes, fmt):
    """Unpack one block's payload (LSB-first bit string) into 32 codes (test helper)."""
    w = bits(fmt)
    b = np.asarray(codes_block_bytes, dtype=np.uint8)
    bitstr = np.unpackbits(b, bitorder="little")
    out = np.zeros(32, dtype=np.uint32)
    for j in range(32):
        for t in range(w):
            out[j] |= np.uint32(bitstr[w * j + t]) << np.uint32(t)
    return out


# ---- eXmY formats (E exponent bits, M mantissa bits; see oracle.c) ---------------------

def _exmy_lib():
    L = lib()
    if not getattr(L, "_exmy", False):
        i32, i64, vp = ctypes.c_int, ctypes.c_int64, ctypes.c_void_p
        L.orc_exmy_decode.restype = ctypes.c_double
        L.orc_exmy_decode.argtypes = [i32, i32, ctypes.c_uint32]
        L.orc_exmy_maxval.restype = ctypes.c_double
        L.orc_exmy_maxval.argtypes = [i32, i32]
        L.orc_exmy_emax.argtypes = [i32, i32]
        L.orc_exmy_round_mags.argtypes = [i32, i32, vp, i64, vp]
        L.orc_quantize_exmy.argtypes = [i32, i32, vp, i32, i64, i64, vp, vp]
        L.orc_dequantize_exmy.argtypes = [i32, i32, vp, vp, i64, i64, vp, i32]
        L.orc_fake_quantize_exmy.argtypes = [i32, i32, vp, i32, i64, i64, vp]
        L._exmy = True
    return L


def exmy_valid(E, M):
    return 0 <= E <= 5 and M >= 1 and 3 <= 1 + E + M <= 9


def exmy_decode_table(E, M):
    L = _exmy_lib()
    return np.array([L.orc_exmy_decode(E, M, c) for c in range(1 << (1 + E + M))], dtype=np.float64)


def exmy_maxval(E, M):
    return _exmy_lib().orc_exmy_maxval(E, M)


def exmy_emax(E, M):
    return _exmy_lib().orc_exmy_emax(E, M)


def exmy_round_mags(E, M, y):
    y = np.ascontiguousarray(y, dtype=np.float64)
    out = np.zeros(y.shape, dtype=np.uint32)
    _exmy_lib().orc_exmy_round_mags(E, M, _ptr(y), y.size, _ptr(out))
    return out


def quantize_exmy(x, E, M):
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    W = 1 + E + M
    codes = np.zeros((rows, cols // 32 * 4 * W), dtype=np.uint8)
    scales = np.zeros((rows, cols // 32), dtype=np.uint8)
    rc = _exmy_lib().orc_quantize_exmy(E, M, _ptr(x), DTYPES[_dtype_of(x)], rows, cols, _ptr(codes), _ptr(scales))
    if rc:
        raise ValueError(f"oracle quantize_exmy rejected the arguments (rc={rc})")
    return codes, scales


def dequantize_exmy(codes, scales, E, M, shape, dtype="bf16"):
    rows, cols = shape
    codes = np.ascontiguousarray(codes)
    scales = np.ascontiguousarray(scales)
    out = np.zeros((rows, cols), dtype=np.float32 if dtype == "f32" else np.uint16)
    rc = _exmy_lib().orc_dequantize_exmy(E, M, _ptr(codes), _ptr(scales), rows, cols, _ptr(out), DTYPES[dtype])
    if rc:
        raise ValueError(f"oracle dequantize_exmy rejected the arguments (rc={rc})")
    return out


def fake_quantize_exmy(x, E, M):
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    out = np.zeros_like(x)
    rc = _exmy_lib().orc_fake_quantize_exmy(E, M, _ptr(x), DTYPES[_dtype_of(x)], rows, cols, _ptr(out))
    if rc:
        raise ValueError(f"oracle fake_quantize_exmy rejected the arguments (rc={rc})")
    return out


# ---- scale-factor layout of the block-scaled MMA (see oracle.c) -------------------------

def _mma_lib():
    L = lib()
    if not getattr(L, "_mma", False):
        i64, vp = ctypes.c_int64, ctypes.c_void_p
        L.orc_mma_scales_bytes.restype = i64
        L.orc_mma_scales_bytes.argtypes = [i64, i64]
        L.orc_mma_scale_index.restype = i64
        L.orc_mma_scale_index.argtypes = [i64, i64, i64]
        L.orc_swizzle_scales.argtypes = [vp, i64, i64, vp]
        L._mma = True
    return L


def mma_scales_bytes(rows, kb):
    return _mma_lib().orc_mma_scales_bytes(rows, kb)


def mma_scale_index(r, k, kb):
    return _mma_lib().orc_mma_scale_index(r, k, kb)


def swizzle_scales(scales):
    """[rows, kb] uint8 E8M0 scales -> 1-D uint8 array in the block-scaled MMA layout."""
    s = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, kb = s.shape
    out = np.zeros(mma_scales_bytes(rows, kb), dtype=np.uint8)
    if _mma_lib().orc_swizzle_scales(_ptr(s), rows, kb, _ptr(out)):
        raise ValueError("oracle swizzle_scales rejected the arguments")
    return out
