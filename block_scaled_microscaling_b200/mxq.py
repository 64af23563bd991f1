"""Python binding of libmxq (include/mxq.h), argument marshalling only.

The functions named like the C entry points (mxq_quantize, ...) take raw
integers (device pointers, sizes, a cudaStream_t handle) and return the
mxq_status code. The torch-facing helpers below them (quantize, dequantize,
fake_quantize, exp_quantize, exp_free_quantize, quantize_grouped, batch, ...)
only allocate outputs with torch, refuse host tensors and caller-supplied
buffers that are non-contiguous or smaller than the shape needs (the C calls
take bare pointers, so a short buffer would be read or written past its end),
read pointers and the current stream, call the C entry point and raise MXQError
on a non-zero status. Every step of the method runs in the
CUDA kernels of libmxq; there is no CPU path: if libmxq.so is missing, every
call raises.
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmxq.so")

FORMATS = {"axs6": 0, "mxfp6_e2m3": 1, "mxfp6_e3m2": 2, "mxfp8": 3, "mxfp4": 4}
DTYPES = {"f32": 0, "bf16": 1}
STATUS = {0: "MXQ_OK", 1: "MXQ_ERR_INVALID_ARG", 2: "MXQ_ERR_SHAPE", 3: "MXQ_ERR_ALIGN",
          4: "MXQ_ERR_UNSUPPORTED", 5: "MXQ_ERR_CUDA", 6: "MXQ_ERR_TIMEOUT"}
MAX_GROUP = 64
ELEM_BITS = {"axs6": 6, "mxfp6_e2m3": 6, "mxfp6_e3m2": 6, "mxfp8": 8, "mxfp4": 4}

EXPORTS = ["mxq_quantize", "mxq_dequantize", "mxq_fake_quantize", "mxq_exp_quantize", "mxq_exp_free_quantize",
           "mxq_quantize_grouped",
           "mxq_quantize_cols", "mxq_dequantize_cols", "mxq_quantize_exmy", "mxq_dequantize_exmy",
           "mxq_fake_quantize_exmy", "mxq_quantize_mma", "mxq_swizzle_scales", "mxq_mma_scales_bytes", "mxq_run_batch", "mxq_check_device", "mxq_selftest_timeout",
           "mxq_codes_bytes", "mxq_scales_bytes", "mxq_block_bits", "mxq_status_string",
           "mxq_version"]


class MXQError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)} ({mxq_status_string(status)})")


class _Tensor(ctypes.Structure):
    _fields_ = [("src", ctypes.c_void_p), ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64)]


class _Op(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("fmt", ctypes.c_int), ("src", ctypes.c_void_p),
                ("src_scales", ctypes.c_void_p), ("dst", ctypes.c_void_p), ("dst_scales", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64)]


_lib = None


def lib():
    """The loaded libmxq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m block_scaled_microscaling_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        i32, i64, vp, sz = ctypes.c_int, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t
        for name, args in [
            ("mxq_quantize", [i32, vp, i32, i64, i64, vp, vp, vp]),
            ("mxq_dequantize", [i32, vp, vp, i64, i64, vp, i32, vp]),
            ("mxq_fake_quantize", [i32, vp, i32, i64, i64, vp, vp]),
            ("mxq_exp_quantize", [i32, vp, i64, i64, vp, vp, vp]),
            ("mxq_exp_free_quantize", [vp, i64, i64, vp, vp, vp]),
            ("mxq_quantize_grouped", [i32, i32, ctypes.POINTER(_Tensor), i32, vp]),
            ("mxq_quantize_cols", [i32, vp, i32, i64, i64, vp, vp, vp]),
            ("mxq_dequantize_cols", [i32, vp, vp, i64, i64, vp, i32, vp]),
            ("mxq_quantize_exmy", [i32, i32, vp, i32, i64, i64, vp, vp, vp]),
            ("mxq_dequantize_exmy", [i32, i32, vp, vp, i64, i64, vp, i32, vp]),
            ("mxq_fake_quantize_exmy", [i32, i32, vp, i32, i64, i64, vp, vp]),
            ("mxq_quantize_mma", [i32, vp, i32, i64, i64, vp, vp, vp]),
            ("mxq_run_batch", [i32, ctypes.POINTER(_Op), i32, vp]),
            ("mxq_swizzle_scales", [vp, i64, i64, vp, vp]),
        ]:
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = i32
        L.mxq_codes_bytes.argtypes = [i32, i64, i64]
        L.mxq_codes_bytes.restype = sz
        L.mxq_scales_bytes.argtypes = [i32, i64, i64]
        L.mxq_scales_bytes.restype = sz
        L.mxq_selftest_timeout.argtypes = [i32]
        L.mxq_selftest_timeout.restype = i32
        L.mxq_check_device.argtypes = []
        L.mxq_check_device.restype = i32
        L.mxq_mma_scales_bytes.argtypes = [i64, i64]
        L.mxq_mma_scales_bytes.restype = sz
        L.mxq_block_bits.argtypes = [i32]
        L.mxq_block_bits.restype = i32
        L.mxq_status_string.argtypes = [i32]
        L.mxq_status_string.restype = ctypes.c_char_p
        L.mxq_version.argtypes = []
        L.mxq_version.restype = ctypes.c_char_p
        _lib = L
    return _lib


# ---- the C entry points, same names and arguments --------------------------------

def mxq_quantize(fmt, src, dtype, rows, cols, codes, scales, stream):
    return lib().mxq_quantize(fmt, src, dtype, rows, cols, codes, scales, stream)


def mxq_dequantize(fmt, codes, scales, rows, cols, dst, dtype, stream):
    return lib().mxq_dequantize(fmt, codes, scales, rows, cols, dst, dtype, stream)


def mxq_fake_quantize(fmt, src, dtype, rows, cols, dst, stream):
    return lib().mxq_fake_quantize(fmt, src, dtype, rows, cols, dst, stream)


def mxq_exp_quantize(fmt, scores, rows, cols, codes, scales, stream):
    return lib().mxq_exp_quantize(fmt, scores, rows, cols, codes, scales, stream)


def mxq_exp_free_quantize(scores, rows, cols, codes, scales, stream):
    return lib().mxq_exp_free_quantize(scores, rows, cols, codes, scales, stream)


def mxq_quantize_grouped(fmt, dtype, tensors, stream):
    """tensors: sequence of (src, codes, scales, rows, cols) integer tuples."""
    arr = (_Tensor * max(1, len(tensors)))()
    for i, (s, c, sc, r, k) in enumerate(tensors):
        arr[i] = _Tensor(s, c, sc, r, k)
    return lib().mxq_quantize_grouped(fmt, dtype, arr, len(tensors), stream)


def mxq_quantize_cols(fmt, src, dtype, rows, cols, codes, scales, stream):
    return lib().mxq_quantize_cols(fmt, src, dtype, rows, cols, codes, scales, stream)


def mxq_dequantize_cols(fmt, codes, scales, rows, cols, dst, dtype, stream):
    return lib().mxq_dequantize_cols(fmt, codes, scales, rows, cols, dst, dtype, stream)


def mxq_quantize_exmy(ebits, mbits, src, dtype, rows, cols, codes, scales, stream):
    return lib().mxq_quantize_exmy(ebits, mbits, src, dtype, rows, cols, codes, scales, stream)


def mxq_dequantize_exmy(ebits, mbits, codes, scales, rows, cols, dst, dtype, stream):
    return lib().mxq_dequantize_exmy(ebits, mbits, codes, scales, rows, cols, dst, dtype, stream)


def mxq_fake_quantize_exmy(ebits, mbits, src, dtype, rows, cols, dst, stream):
    return lib().mxq_fake_quantize_exmy(ebits, mbits, src, dtype, rows, cols, dst, stream)


def mxq_quantize_mma(fmt, src, dtype, rows, cols, codes, scales, stream):
    return lib().mxq_quantize_mma(fmt, src, dtype, rows, cols, codes, scales, stream)


def mxq_swizzle_scales(scales, rows, kblocks, out, stream):
    return lib().mxq_swizzle_scales(scales, rows, kblocks, out, stream)


def mxq_mma_scales_bytes(rows, cols):
    return lib().mxq_mma_scales_bytes(rows, cols)


def mxq_run_batch(dtype, ops, stream):
    """ops: sequence of (kind, fmt, src, src_scales, dst, dst_scales, rows, cols) integer tuples."""
    arr = (_Op * max(1, len(ops)))()
    for i, o in enumerate(ops):
        arr[i] = _Op(*o)
    return lib().mxq_run_batch(dtype, arr, len(ops), stream)


def mxq_check_device():
    return lib().mxq_check_device()


def mxq_selftest_timeout(limit_ms):
    return lib().mxq_selftest_timeout(limit_ms)


def check_device():
    """Synchronize and raise MXQError(MXQ_ERR_TIMEOUT) if a bounded wait in a kernel ran out."""
    _check(mxq_check_device(), "mxq_check_device")


def mxq_codes_bytes(fmt, rows, cols):
    return lib().mxq_codes_bytes(fmt, rows, cols)


def mxq_scales_bytes(fmt, rows, cols):
    return lib().mxq_scales_bytes(fmt, rows, cols)


def mxq_block_bits(fmt):
    return lib().mxq_block_bits(fmt)


def mxq_status_string(status):
    return lib().mxq_status_string(status).decode()


def mxq_version():
    return lib().mxq_version().decode()


# ---- torch helpers ---------------------------------------------------------------

def _torch():
    import torch
    return torch


def _fmt(fmt):
    if fmt not in FORMATS:
        raise ValueError(f"unknown format {fmt!r}; one of {sorted(FORMATS)}")
    return FORMATS[fmt]


def _dt(t):
    torch = _torch()
    if t.dtype == torch.float32:
        return DTYPES["f32"]
    if t.dtype == torch.bfloat16:
        return DTYPES["bf16"]
    raise TypeError(f"values must be float32 or bfloat16, got {t.dtype}")


def _stream(stream):
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _as2d(t):
    if t.dim() == 0:
        raise ValueError("need at least one dimension")
    cols = t.shape[-1]
    rows = t.numel() // cols if cols else 0
    return rows, cols


def _check(status, what):
    if status != 0:
        raise MXQError(status, what)


def _finish(check):
    """check=True: synchronize and raise MXQError(MXQ_ERR_TIMEOUT) if a bounded wait of a kernel
    ran out (its outputs are then incomplete). The bulk-copy kernels (exp_quantize,
    exp_free_quantize, quantize_cols, fake_quantize of 2^19 blocks or more) bound their waits;
    without check=True a caller learns of such a timeout only from a later check_device()."""
    if check:
        check_device()


def _on_gpu(t, what):
    """The library computes on the GPU only: a host tensor is refused here, before any call."""
    if not t.is_cuda:
        raise ValueError(f"{what} must be a CUDA tensor (libmxq has no CPU path)")


def _fits(t, nbytes, what):
    """A buffer handed to the library as a bare pointer must be contiguous and hold at least
    nbytes, or a kernel would read or write past the tensor's end."""
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    have = t.numel() * t.element_size()
    if have < nbytes:
        raise ValueError(f"{what} holds {have} bytes, the call needs {nbytes}")


def _nblocks(rows, cols):
    return rows * (cols // 32) if rows >= 0 and cols > 0 else 0


def _codes_scales_bytes(fmt, rows, cols):
    """Bytes of the code and scale arrays (0 for a shape the library rejects)."""
    f = _fmt(fmt)
    return mxq_codes_bytes(f, rows, cols), mxq_scales_bytes(f, rows, cols)


def scale_dtype(fmt):
    torch = _torch()
    return torch.int16 if fmt == "axs6" else torch.uint8


def empty_codes(fmt, rows, cols, device):
    torch = _torch()
    return torch.empty((rows, (cols // 32) * 4 * ELEM_BITS[fmt]), dtype=torch.uint8, device=device)


def empty_scales(fmt, rows, cols, device):
    torch = _torch()
    return torch.empty((rows, cols // 32), dtype=scale_dtype(fmt), device=device)


def quantize(x, fmt, codes=None, scales=None, stream=None):
    """x [..., cols] (bf16/fp32, contiguous, CUDA) -> (codes uint8 [rows, cols/32*P], scales)."""
    if not x.is_contiguous():
        raise ValueError("x must be contiguous")
    _on_gpu(x, "x")
    rows, cols = _as2d(x)
    nc, ns = _codes_scales_bytes(fmt, rows, cols)
    if codes is None:
        codes = empty_codes(fmt, rows, cols, x.device)
    if scales is None:
        scales = empty_scales(fmt, rows, cols, x.device)
    _fits(codes, nc, "codes")
    _fits(scales, ns, "scales")
    _check(mxq_quantize(_fmt(fmt), x.data_ptr(), _dt(x), rows, cols, codes.data_ptr(), scales.data_ptr(),
                        _stream(stream)), "mxq_quantize")
    return codes, scales


def dequantize(codes, scales, fmt, shape, dtype=None, out=None, stream=None):
    """codes + scales -> values of `shape` (last dim = cols) and `dtype` (default bf16)."""
    torch = _torch()
    _on_gpu(codes, "codes")
    if out is None:
        out = torch.empty(tuple(shape), dtype=dtype or torch.bfloat16, device=codes.device)
    rows, cols = _as2d(out)
    nc, ns = _codes_scales_bytes(fmt, rows, cols)
    _fits(codes, nc, "codes")
    _fits(scales, ns, "scales")
    _fits(out, 0, "out")
    _check(mxq_dequantize(_fmt(fmt), codes.data_ptr(), scales.data_ptr(), rows, cols, out.data_ptr(), _dt(out),
                          _stream(stream)), "mxq_dequantize")
    return out


def _same_values(x, out):
    """out of a fake-quantize: x's type and element count, contiguous."""
    if out.dtype != x.dtype or out.numel() != x.numel():
        raise ValueError(f"out must have x's dtype and size ({x.dtype}, {x.numel()}), got ({out.dtype}, {out.numel()})")
    _fits(out, 0, "out")


def fake_quantize(x, fmt="axs6", block_size=32, out=None, stream=None, check=False):
    """Quantize then dequantize in one pass; out=x runs in place. Tensors of 2^19 blocks or more
    go through a bulk-copy kernel with bounded waits: check=True synchronizes and raises if one
    ran out (else call check_device() before trusting `out`)."""
    if block_size != 32:
        raise MXQError(4, f"block_size={block_size}")
    torch = _torch()
    if not x.is_contiguous():
        raise ValueError("x must be contiguous")
    _on_gpu(x, "x")
    if out is None:
        out = torch.empty_like(x)
    _same_values(x, out)
    rows, cols = _as2d(x)
    _check(mxq_fake_quantize(_fmt(fmt), x.data_ptr(), _dt(x), rows, cols, out.data_ptr(), _stream(stream)),
           "mxq_fake_quantize")
    _finish(check)
    return out


def exp_quantize(scores, fmt="mxfp4", codes=None, scales=None, stream=None, check=False):
    """fp32 scores [..., keys] -> codes + scales of exp(s - rowmax), block-quantized per 32 keys.
    The kernel's waits are bounded: check=True synchronizes and raises if one ran out (else
    call check_device() before trusting the outputs)."""
    torch = _torch()
    if scores.dtype != torch.float32 or not scores.is_contiguous():
        raise ValueError("scores must be contiguous float32")
    _on_gpu(scores, "scores")
    rows, cols = _as2d(scores)
    nc, ns = _codes_scales_bytes(fmt, rows, cols)
    if codes is None:
        codes = empty_codes(fmt, rows, cols, scores.device)
    if scales is None:
        scales = empty_scales(fmt, rows, cols, scores.device)
    _fits(codes, nc, "codes")
    _fits(scales, ns, "scales")
    _check(mxq_exp_quantize(_fmt(fmt), scores.data_ptr(), rows, cols, codes.data_ptr(), scales.data_ptr(),
                            _stream(stream)), "mxq_exp_quantize")
    _finish(check)
    return codes, scales


def exp_free_quantize(scores, codes=None, scales=None, stream=None, check=False):
    """fp32 scores [..., keys] -> MXFP4 codes + E8M0 scales by the exp-free rule (no exponential):
    per 32 keys an exponent-only scale from the block's maximum, one affine map to E2M1 codes.
    The kernel's waits are bounded: check=True synchronizes and raises if one ran out (else
    call check_device() before trusting the outputs)."""
    torch = _torch()
    if scores.dtype != torch.float32 or not scores.is_contiguous():
        raise ValueError("scores must be contiguous float32")
    _on_gpu(scores, "scores")
    rows, cols = _as2d(scores)
    nc, ns = _codes_scales_bytes("mxfp4", rows, cols)
    if codes is None:
        codes = empty_codes("mxfp4", rows, cols, scores.device)
    if scales is None:
        scales = empty_scales("mxfp4", rows, cols, scores.device)
    _fits(codes, nc, "codes")
    _fits(scales, ns, "scales")
    _check(mxq_exp_free_quantize(scores.data_ptr(), rows, cols, codes.data_ptr(), scales.data_ptr(), _stream(stream)),
           "mxq_exp_free_quantize")
    _finish(check)
    return codes, scales


def quantize_mma(x, fmt, codes=None, scales=None, stream=None):
    """As quantize, with the scales as a 1-D uint8 tensor in the block-scaled MMA tile layout
    (mxq_mma_scales_bytes(rows, cols) bytes, zero padding)."""
    torch = _torch()
    if not x.is_contiguous():
        raise ValueError("x must be contiguous")
    _on_gpu(x, "x")
    rows, cols = _as2d(x)
    nc, _ = _codes_scales_bytes(fmt, rows, cols)
    if codes is None:
        codes = empty_codes(fmt, rows, cols, x.device)
    if scales is None:
        scales = torch.empty(mxq_mma_scales_bytes(rows, cols), dtype=torch.uint8, device=x.device)
    _fits(codes, nc, "codes")
    _fits(scales, mxq_mma_scales_bytes(rows, cols), "scales")
    _check(mxq_quantize_mma(_fmt(fmt), x.data_ptr(), _dt(x), rows, cols, codes.data_ptr(), scales.data_ptr(),
                            _stream(stream)), "mxq_quantize_mma")
    return codes, scales


def swizzle_scales(scales, out=None, stream=None):
    """uint8 scales [rows, kblocks] (contiguous, CUDA) -> 1-D uint8 tensor in the MMA tile layout."""
    torch = _torch()
    if scales.dtype != torch.uint8 or scales.dim() != 2 or not scales.is_contiguous():
        raise ValueError("scales must be a contiguous 2-D uint8 tensor")
    _on_gpu(scales, "scales")
    rows, kb = scales.shape
    if out is None:
        out = torch.empty(mxq_mma_scales_bytes(rows, 32 * kb), dtype=torch.uint8, device=scales.device)
    _fits(out, mxq_mma_scales_bytes(rows, 32 * kb), "out")
    _check(mxq_swizzle_scales(scales.data_ptr(), rows, kb, out.data_ptr(), _stream(stream)), "mxq_swizzle_scales")
    return out


OP_KINDS = {"quantize": 0, "dequantize": 1, "fake_quantize": 2}


def batch(ops, stream=None):
    """Several independent conversions in one launch (all values of one dtype):
      ("quantize", fmt, x, codes, scales)
      ("dequantize", fmt, codes, scales, out)      -- out's shape gives rows, cols
      ("fake_quantize", fmt, x, out)
    Outputs must be preallocated; no output may overlap another op's buffers."""
    descs, dtype = [], None
    for op in ops:
        kind = op[0]
        if kind == "quantize":
            _, fmt, x, codes, scales = op
            vals, d = x, (x.data_ptr(), 0, codes.data_ptr(), scales.data_ptr())
        elif kind == "dequantize":
            _, fmt, codes, scales, out = op
            vals, d = out, (codes.data_ptr(), scales.data_ptr(), out.data_ptr(), 0)
        elif kind == "fake_quantize":
            _, fmt, x, out = op
            vals, d = x, (x.data_ptr(), 0, out.data_ptr(), 0)
        else:
            raise ValueError(f"unknown batch op {kind!r}")
        if not vals.is_contiguous():
            raise ValueError("value tensors must be contiguous")
        _on_gpu(vals, "batch values")
        if dtype is None:
            dtype = _dt(vals)
        elif _dt(vals) != dtype:
            raise TypeError("all values of a batch must have one dtype")
        rows, cols = _as2d(vals)
        if kind == "fake_quantize":
            _same_values(x, out)
        else:
            nc, ns = _codes_scales_bytes(fmt, rows, cols)
            _fits(codes, nc, "codes")
            _fits(scales, ns, "scales")
        descs.append((OP_KINDS[kind], _fmt(fmt), *d, rows, cols))
    if not descs:
        raise ValueError("empty batch")
    _check(mxq_run_batch(dtype, descs, _stream(stream)), "mxq_run_batch")


def quantize_grouped(xs, fmt, outs=None, stream=None):
    """Quantize several tensors of one dtype in one launch; returns [(codes, scales), ...]."""
    if not xs:
        return []
    if len(xs) > MAX_GROUP:
        raise ValueError(f"at most {MAX_GROUP} tensors per grouped launch")
    dt = _dt(xs[0])
    if outs is None:
        outs = []
        for x in xs:
            r, c = _as2d(x)
            outs.append((empty_codes(fmt, r, c, x.device), empty_scales(fmt, r, c, x.device)))
    if len(outs) != len(xs):
        raise ValueError("one (codes, scales) pair per tensor")
    descs = []
    for x, (c, s) in zip(xs, outs):
        if _dt(x) != dt or not x.is_contiguous():
            raise ValueError("grouped tensors must be contiguous and share one dtype")
        _on_gpu(x, "grouped tensors")
        r, k = _as2d(x)
        nc, ns = _codes_scales_bytes(fmt, r, k)
        _fits(c, nc, "codes")
        _fits(s, ns, "scales")
        descs.append((x.data_ptr(), c.data_ptr(), s.data_ptr(), r, k))
    _check(mxq_quantize_grouped(_fmt(fmt), dt, descs, _stream(stream)), "mxq_quantize_grouped")
    return outs


def quantize_cols(x, fmt, codes=None, scales=None, stream=None, check=False):
    """x [rows, cols] -> blocks of 32 rows per column, laid out as quantize(x.T):
    codes [cols, rows/32*P], scales [cols, rows/32]. The kernel's waits are bounded:
    check=True synchronizes and raises if one ran out (else call check_device() before
    trusting the outputs)."""
    if not x.is_contiguous() or x.dim() != 2:
        raise ValueError("x must be a contiguous 2-D tensor")
    _on_gpu(x, "x")
    rows, cols = x.shape
    nc, ns = _codes_scales_bytes(fmt, cols, rows)
    if codes is None:
        codes = empty_codes(fmt, cols, rows, x.device)
    if scales is None:
        scales = empty_scales(fmt, cols, rows, x.device)
    _fits(codes, nc, "codes")
    _fits(scales, ns, "scales")
    _check(mxq_quantize_cols(_fmt(fmt), x.data_ptr(), _dt(x), rows, cols, codes.data_ptr(), scales.data_ptr(),
                             _stream(stream)), "mxq_quantize_cols")
    _finish(check)
    return codes, scales


def dequantize_cols(codes, scales, fmt, shape, dtype=None, out=None, stream=None):
    """Inverse of quantize_cols: values of `shape` = (rows, cols)."""
    torch = _torch()
    _on_gpu(codes, "codes")
    if out is None:
        out = torch.empty(tuple(shape), dtype=dtype or torch.bfloat16, device=codes.device)
    if out.dim() != 2:
        raise ValueError("out must be 2-D (rows, cols)")
    rows, cols = out.shape
    nc, ns = _codes_scales_bytes(fmt, cols, rows)
    _fits(codes, nc, "codes")
    _fits(scales, ns, "scales")
    _fits(out, 0, "out")
    _check(mxq_dequantize_cols(_fmt(fmt), codes.data_ptr(), scales.data_ptr(), rows, cols, out.data_ptr(), _dt(out),
                               _stream(stream)), "mxq_dequantize_cols")
    return out


def quantize_exmy(x, ebits, mbits, codes=None, scales=None, stream=None):
    """eXmY codes (W = 1 + ebits + mbits bits, W words per block) + E8M0 scales."""
    torch = _torch()
    if not x.is_contiguous():
        raise ValueError("x must be contiguous")
    _on_gpu(x, "x")
    rows, cols = _as2d(x)
    W = 1 + ebits + mbits
    if codes is None:
        codes = torch.empty((rows, (cols // 32) * 4 * W), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((rows, cols // 32), dtype=torch.uint8, device=x.device)
    _fits(codes, _nblocks(rows, cols) * 4 * max(W, 0), "codes")
    _fits(scales, _nblocks(rows, cols), "scales")
    _check(mxq_quantize_exmy(ebits, mbits, x.data_ptr(), _dt(x), rows, cols, codes.data_ptr(), scales.data_ptr(),
                             _stream(stream)), "mxq_quantize_exmy")
    return codes, scales


def dequantize_exmy(codes, scales, ebits, mbits, shape, dtype=None, out=None, stream=None):
    torch = _torch()
    _on_gpu(codes, "codes")
    if out is None:
        out = torch.empty(tuple(shape), dtype=dtype or torch.bfloat16, device=codes.device)
    rows, cols = _as2d(out)
    _fits(codes, _nblocks(rows, cols) * 4 * max(1 + ebits + mbits, 0), "codes")
    _fits(scales, _nblocks(rows, cols), "scales")
    _fits(out, 0, "out")
    _check(mxq_dequantize_exmy(ebits, mbits, codes.data_ptr(), scales.data_ptr(), rows, cols, out.data_ptr(),
                               _dt(out), _stream(stream)), "mxq_dequantize_exmy")
    return out


def fake_quantize_exmy(x, ebits, mbits, out=None, stream=None):
    torch = _torch()
    if not x.is_contiguous():
        raise ValueError("x must be contiguous")
    _on_gpu(x, "x")
    if out is None:
        out = torch.empty_like(x)
    _same_values(x, out)
    rows, cols = _as2d(x)
    _check(mxq_fake_quantize_exmy(ebits, mbits, x.data_ptr(), _dt(x), rows, cols, out.data_ptr(), _stream(stream)),
           "mxq_fake_quantize_exmy")
    return out
