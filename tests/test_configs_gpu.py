"""Parity at the five workloads' full sizes, launched exactly as bench.py launches
them, checked bit for bit against the oracle: in full where the oracle takes
seconds, on sampled blocks / rows (each computed by the oracle on its own)
otherwise. Inputs come from the seeded generators in synthetic/.

 1. AXS-6 fake-quantize of fp32 128x256 N(0,1), plus quantize/dequantize round trip
 2. MXFP6 E2M3 and E3M2 quantize + dequantize of a bf16 4096x4096 N(0,0.02)
    weight with 0.1% outliers x50
 3. online conversion of a 36-layer decoder stack (7 bf16 weights per layer,
    one grouped launch per layer) to MXFP6 E2M3 and to AXS-6
 4. MXFP8 E4M3 and MXFP6 E2M3 quantize + dequantize of bf16 16384x8192
    Student-t activations with 16 outlier channels, AXS-6 fake-quantize of
    fp32 16384x8192 N(0,1e-3) gradients
 5. exp-then-quantize of fp32 attention scores 32x128 rows x 32768 keys N(0,3) to MXFP4
"""
import numpy as np
import pytest

import oracle
import synthetic

torch = pytest.importorskip("torch")
from block_scaled_microscaling_b200 import mxq  # noqa: E402

from test_parity_gpu import bits, dev, host  # noqa: E402

pytestmark = pytest.mark.gpu


def sample(n, k, seed):
    rng = np.random.default_rng(seed)
    idx = rng.choice(n, size=min(k, n), replace=False)
    return np.unique(np.concatenate([idx, [0, n - 1]]))


def check_quantize_sampled(x, codes, scales, fmt, k=20000, seed=0):
    nb = x.size // 32
    idx = sample(nb, k, seed)
    xs = x.reshape(nb, 32)[idx]
    oc, os_ = oracle.quantize(xs, fmt)
    pb = oracle.payload_bytes(fmt)
    assert np.array_equal(host(scales).reshape(nb)[idx], os_.reshape(-1))
    assert np.array_equal(host(codes).reshape(nb, pb)[idx], oc)
    return idx, xs


def check_values_sampled(out, ref_fn, xs_idx, nb):
    idx, xs = xs_idx
    got = bits(host(out).reshape(nb, 32)[idx])
    assert np.array_equal(got, bits(ref_fn(xs)))


def test_config1_axs6_quickstart():
    x = synthetic.quickstart_fp32(seed=0)
    t = dev(x)
    fq = mxq.fake_quantize(t, "axs6", block_size=32)
    assert np.array_equal(bits(host(fq)), bits(oracle.fake_quantize(x, "axs6")))
    codes, scales = mxq.quantize(t, "axs6")
    oc, os_ = oracle.quantize(x, "axs6")
    assert np.array_equal(host(codes), oc) and np.array_equal(host(scales), os_)
    assert np.all((host(scales) >> 8) == 0)  # config field = 0
    rt = mxq.dequantize(codes, scales, "axs6", x.shape, torch.float32)
    assert np.array_equal(bits(host(rt)), bits(host(fq)))


@pytest.mark.parametrize("fmt", ["mxfp6_e2m3", "mxfp6_e3m2"])
def test_config2_mxfp6_weight(fmt):
    w, pos = synthetic.weight_with_outliers(seed=1)
    t = dev(w)
    codes, scales = mxq.quantize(t, fmt)
    oc, os_ = oracle.quantize(w, fmt)
    assert np.array_equal(host(scales), os_)
    assert np.array_equal(host(codes), oc)
    out = mxq.dequantize(codes, scales, fmt, w.shape, torch.bfloat16)
    assert np.array_equal(bits(host(out)), bits(oracle.dequantize(oc, os_, fmt, w.shape, "bf16")))


@pytest.mark.parametrize("fmt", ["mxfp6_e2m3", "axs6"])
@pytest.mark.parametrize("layer", [0, 35])
def test_config3_decoder_stack_layer(fmt, layer):
    ws = [synthetic.decoder_weight(layer, k) for k in range(7)]
    outs = mxq.quantize_grouped([dev(w) for w in ws], fmt)
    for k, (w, (c, s)) in enumerate(zip(ws, outs)):
        idx_xs = check_quantize_sampled(w, c, s, fmt, k=4000, seed=k)
        if k in (0, 6):
            out = mxq.dequantize(c, s, fmt, w.shape, torch.bfloat16)
            check_values_sampled(out, lambda xs: oracle.fake_quantize(xs, fmt), idx_xs, w.size // 32)


def sampled_rows(rows, k, rng):
    return np.unique(np.concatenate([rng.choice(rows, k, replace=False), [0, rows - 1]]))


@pytest.mark.parametrize("fmt", ["mxfp6_e2m3", "axs6"])
def test_config3_every_layer_sampled_rows(fmt):
    """All 36 layers, each converted by one grouped launch of its 7 full-size tensors exactly as
    the bench launches them. 18 rows of every tensor (its first and last among them) hold the
    workload's own bits, drawn from the seeded counter-based generator at those rows' element
    offsets; the other rows are seeded N(0, 0.02) filler drawn on the device. The codes and
    scales of the sampled rows equal the oracle's, and a dequantize of each layer's first and
    last tensor gives the oracle's values on those rows."""
    dev_ = torch.device("cuda")
    gen = torch.Generator(device=dev_)
    rng = np.random.default_rng(36)
    for layer in range(synthetic.N_LAYERS):
        gen.manual_seed(7000 + layer)
        ts, picks = [], []
        for k, (_, rows, cols) in enumerate(synthetic.DECODER_LAYER):
            t = (torch.randn(rows, cols, device=dev_, generator=gen) * 0.02).to(torch.bfloat16)
            sel = sampled_rows(rows, 16, rng)
            xs = np.stack([synthetic.f32_to_bf16_bits(synthetic.to_f32(
                synthetic.normals(2, layer * 7 + k, cols, start=int(r) * cols) * 0.02)) for r in sel])
            t[torch.from_numpy(sel).to(dev_)] = dev(xs)
            ts.append(t)
            picks.append((sel, xs))
        outs = mxq.quantize_grouped(ts, fmt)
        for k, ((sel, xs), (c, s)) in enumerate(zip(picks, outs)):
            oc, os_ = oracle.quantize(xs, fmt)
            assert np.array_equal(host(s[torch.from_numpy(sel).to(dev_)]), os_), (layer, k)
            assert np.array_equal(host(c[torch.from_numpy(sel).to(dev_)]), oc), (layer, k)
            if k in (0, 6):
                y = mxq.dequantize(c, s, fmt, ts[k].shape, torch.bfloat16)
                got = bits(host(y[torch.from_numpy(sel).to(dev_)]))
                assert np.array_equal(got, bits(oracle.dequantize(oc, os_, fmt, xs.shape, "bf16"))), (layer, k)
        del ts, outs


@pytest.mark.parametrize("fmt", ["mxfp8", "mxfp6_e2m3"])
def test_config4_activations(fmt):
    a = synthetic.student_t_activations(seed=3)
    t = dev(a)
    codes, scales = mxq.quantize(t, fmt)
    idx_xs = check_quantize_sampled(a, codes, scales, fmt, seed=1)
    out = mxq.dequantize(codes, scales, fmt, a.shape, torch.bfloat16)
    check_values_sampled(out, lambda xs: oracle.fake_quantize(xs, fmt), idx_xs, a.size // 32)
    # the outlier channels get their own large scales
    ch = synthetic.outlier_channels()
    blocks = sorted({c // 32 for c in ch})
    sc = host(scales)[:64]
    other = [b for b in range(256) if b not in blocks]
    assert sc[:, blocks].mean() > sc[:, other].mean() + 3


def test_config4_gradients_fake_quantize():
    g = synthetic.gradients_fp32(seed=3)
    t = dev(g)
    out = mxq.fake_quantize(t, "axs6")
    nb = g.size // 32
    idx = sample(nb, 20000, 2)
    xs = g.reshape(nb, 32)[idx]
    assert np.array_equal(bits(host(out).reshape(nb, 32)[idx]), bits(oracle.fake_quantize(xs, "axs6")))
    mxq.fake_quantize(t, "axs6", out=t)  # in place, same launch shape
    assert np.array_equal(bits(host(t)), bits(host(out)))


def test_config5_exp_quantize_mxfp4():
    """All 4096 rows (134M scores, each through the method's own fp32 exponential) against
    the oracle, bit for bit: about ten seconds of oracle time."""
    s = synthetic.attention_scores(seed=4)
    codes, scales = mxq.exp_quantize(dev(s), "mxfp4")
    oc, os_ = oracle.exp_quantize(s, "mxfp4")
    assert np.array_equal(host(scales), os_)
    assert np.array_equal(host(codes), oc)
    # every row's maximum key: p = 1 -> scale byte 125, E2M1 code 0x6; no sign bits
    hc, hs = host(codes), host(scales)
    j = np.argmax(s, axis=1)
    r = np.arange(s.shape[0])
    assert np.all(hs[r, j // 32] == 125)
    nib = (hc[r, j // 2] >> (4 * (j % 2))) & 0xF
    assert np.all(nib == 0x6)
    assert not np.any(hc & 0x88)
