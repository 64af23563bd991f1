"""GPU: mxq_run_batch -- several independent conversions in one launch -- gives, op for op, the
bits of the single-operation entry points and of the oracle ("Sonar: Online MXFP6", Start a
model: a layer's tensors converted together; Select the FP6 encoding: per-tensor formats)."""
import numpy as np
import pytest

import oracle
import synthetic

torch = pytest.importorskip("torch")
from block_scaled_microscaling_b200 import mxq  # noqa: E402

pytestmark = pytest.mark.gpu

FMTS = ["axs6", "mxfp6_e2m3", "mxfp6_e3m2", "mxfp8", "mxfp4"]


def values(rows, cols, seed, dtype):
    x = synthetic.gaussian((rows, cols), 1.0, seed, 0, "f32").reshape(-1, 32)
    e = np.asarray(synthetic.uniform_ints(seed, 5, x.shape[0], 41), dtype=np.int64) - 20
    x = (x * np.ldexp(1.0, e)[:, None].astype(np.float32)).astype(np.float32).reshape(rows, cols)
    return x if dtype == "f32" else synthetic.f32_to_bf16_bits(x)


def dev(x):
    if x.dtype == np.float32:
        return torch.from_numpy(np.ascontiguousarray(x)).cuda()
    return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()


def host(t):
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    if t.dtype == torch.int16:
        return t.cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def bits(a):
    a = np.ascontiguousarray(a)
    return a.view(np.uint32 if a.dtype == np.float32 else np.uint16)


SHAPES = [(1, 32), (3, 96), (7, 160), (129, 416), (33, 8192), (1000, 64)]


def mixed_batch(dtype, seed0):
    """One op per (kind, format), shapes cycling through SHAPES (ragged last warp tiles)."""
    ops, want, k = [], [], 0
    for kind in ("quantize", "dequantize", "fake_quantize"):
        for fmt in FMTS:
            rows, cols = SHAPES[k % len(SHAPES)]
            x = values(rows, cols, seed0 + k, dtype)
            if kind == "quantize":
                c = torch.full((rows, mxq.mxq_codes_bytes(mxq.FORMATS[fmt], rows, cols) // rows), 0xAB,
                               dtype=torch.uint8, device="cuda")
                s = mxq.empty_scales(fmt, rows, cols, "cuda")
                ops.append(("quantize", fmt, dev(x), c, s))
                want.append(("q", fmt, x, c, s))
            elif kind == "dequantize":
                oc, os_ = oracle.quantize(x, fmt)
                out = torch.empty((rows, cols), dtype=torch.bfloat16 if dtype == "bf16" else torch.float32,
                                  device="cuda")
                sc = torch.from_numpy(os_.view(np.int16) if fmt == "axs6" else os_).cuda()
                ops.append(("dequantize", fmt, torch.from_numpy(oc).cuda(), sc, out))
                want.append(("dq", fmt, (oc, os_, (rows, cols)), out, None))
            else:
                xd = dev(x)
                out = torch.empty_like(xd)
                ops.append(("fake_quantize", fmt, xd, out))
                want.append(("fq", fmt, x, out, None))
            k += 1
    return ops, want


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_mixed_batch_matches_oracle(dtype):
    ops, want = mixed_batch(dtype, 300 if dtype == "bf16" else 400)
    mxq.batch(ops)
    torch.cuda.synchronize()
    for kind, fmt, x, a, b in want:
        if kind == "q":
            oc, os_ = oracle.quantize(x, fmt)
            assert np.array_equal(host(a), oc), (kind, fmt, x.shape)
            assert np.array_equal(host(b), os_), (kind, fmt, x.shape)
        elif kind == "dq":
            oc, os_, shape = x
            ref = oracle.dequantize(oc, os_, fmt, shape, dtype)
            assert np.array_equal(bits(host(a)), bits(ref)), (kind, fmt, shape)
        else:
            ref = oracle.fake_quantize(x, fmt)
            assert np.array_equal(bits(host(a)), bits(ref)), (kind, fmt, x.shape)


def test_batch_equals_single_ops_on_the_weight_workload():
    """The four conversions of the MXFP6 weight workload (bf16 4096x4096, 0.1% outliers x50),
    batched, against the single-operation kernels on the same buffers."""
    w_host, _ = synthetic.weight_with_outliers(seed=1)
    w = dev(w_host)
    ca, sa = mxq.quantize(w, "mxfp6_e2m3")
    cb, sb = mxq.quantize(w, "mxfp6_e3m2")
    ya, yb = mxq.dequantize(ca, sa, "mxfp6_e2m3", w.shape), mxq.dequantize(cb, sb, "mxfp6_e3m2", w.shape)
    ca2, sa2, cb2, sb2 = (torch.empty_like(t) for t in (ca, sa, cb, sb))
    ya2, yb2 = torch.empty_like(ya), torch.empty_like(yb)
    mxq.batch([("quantize", "mxfp6_e2m3", w, ca2, sa2), ("quantize", "mxfp6_e3m2", w, cb2, sb2),
               ("dequantize", "mxfp6_e2m3", ca, sa, ya2), ("dequantize", "mxfp6_e3m2", cb, sb, yb2)])
    torch.cuda.synchronize()
    for a, b in [(ca, ca2), (sa, sa2), (cb, cb2), (sb, sb2), (ya.view(torch.int16), ya2.view(torch.int16)),
                 (yb.view(torch.int16), yb2.view(torch.int16))]:
        assert torch.equal(a, b)


def test_batch_rejects_overlap_and_mixed_dtypes():
    x = torch.zeros((64, 256), dtype=torch.bfloat16, device="cuda")
    c, s = mxq.quantize(x, "mxfp8")
    y = torch.empty_like(x)
    # the second op writes the first op's input
    with pytest.raises(mxq.MXQError) as e:
        mxq.batch([("quantize", "mxfp8", x, c, s), ("dequantize", "mxfp8", c, s, x)])
    assert e.value.status == 1
    # two ops write the same output
    with pytest.raises(mxq.MXQError):
        mxq.batch([("fake_quantize", "axs6", x, y), ("dequantize", "mxfp8", c, s, y)])
    # in-place fake-quantize inside one op is allowed
    mxq.batch([("fake_quantize", "axs6", y, y), ("quantize", "mxfp8", x, c, s)])
    with pytest.raises(TypeError):
        mxq.batch([("fake_quantize", "axs6", x.float(), torch.empty_like(x.float())), ("fake_quantize", "axs6", x, y)])
    torch.cuda.synchronize()


def test_batch_of_64_small_ops():
    xs = [dev(values(r, 64, 900 + r, "bf16")) for r in range(1, 65)]
    outs = [torch.empty_like(x) for x in xs]
    mxq.batch([("fake_quantize", FMTS[i % 5], x, o) for i, (x, o) in enumerate(zip(xs, outs))])
    torch.cuda.synchronize()
    for i, (x, o) in enumerate(zip(xs, outs)):
        assert np.array_equal(bits(host(o)), bits(oracle.fake_quantize(host(x), FMTS[i % 5])))
