"""GPU parity of the exp-free E2M1 rule ("EFQ-Softmax: exp-free E2M1 probabilities": per block
of 32 shifted scores an exponent-only scale from the block's local maximum, one affine rule to
nonnegative E2M1 codes) against the CPU oracle, bit for bit (0 ULP: codes and scale bytes
compared as raw bytes). Calls go through the C ABI (mxq_exp_free_quantize)."""
import numpy as np
import pytest

import oracle
import synthetic

torch = pytest.importorskip("torch")
from block_scaled_microscaling_b200 import mxq  # noqa: E402

pytestmark = pytest.mark.gpu


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def host(t):
    return t.cpu().numpy()


def with_specials(s):
    if s.shape[0] >= 6:
        s[1, 5] = np.nan
        s[2, 7] = np.inf
        s[3, :] = -np.inf
        s[4, ::3] = -np.inf
        s[5, :] = 0.0
    return s


@pytest.mark.parametrize("cols", [32, 96, 1024, 4096, 4992, 32768, 65536, 131072])
def test_exp_free_matches_oracle(cols):
    rows = max(2, min(64, 2 ** 21 // cols))
    s = with_specials(synthetic.attention_scores(seed=4, heads=1, queries=rows, keys=cols))
    codes, scales = mxq.exp_free_quantize(dev(s))
    oc, os_ = oracle.exp_free_quantize(s)
    assert np.array_equal(host(scales), os_)
    assert np.array_equal(host(codes), oc)


@pytest.mark.parametrize("rows,cols", [(3000, 640), (700, 8192), (5, 131072), (3, 262144 + 32), (149, 4128)])
def test_exp_free_many_rows_per_cta(rows, cols):
    """More rows than resident CTAs (the row stream runs ahead of the consumers and the row-slot
    rings wrap), rows of one full stage plus a partial one, rows shorter than one stage."""
    s = synthetic.attention_scores(seed=6, heads=1, queries=rows, keys=cols)
    s[::97, 3] = np.nan
    s[1::89, :] = -np.inf
    s[2::83, 5] = np.inf
    codes, scales = mxq.exp_free_quantize(dev(s))
    oc, os_ = oracle.exp_free_quantize(s)
    assert np.array_equal(host(scales), os_)
    assert np.array_equal(host(codes), oc)


def test_exp_free_scores_at_every_scale():
    # scores spread over many binades, and rows where the block scales hit the -127 clamp
    rng = np.random.default_rng(12)
    s = (rng.normal(0, 1, size=(64, 2048)) * np.exp2(rng.integers(-8, 9, size=(64, 1)))).astype(np.float32)
    s[10, 64:] -= np.float32(500.0)
    s[11, 32:] = np.float32(-1e30)
    codes, scales = mxq.exp_free_quantize(dev(s))
    oc, os_ = oracle.exp_free_quantize(s)
    assert np.array_equal(host(scales), os_)
    assert np.array_equal(host(codes), oc)


def test_exp_free_attention_scores_all_rows():
    """Attention scores of 32 heads x 128 queries x 32768 keys, N(0, 3) (the softmax-stage
    workload), launched whole; all 4096 rows checked against the oracle, every row's maximum
    key decoded to probability 1 (byte 125, code 6), and the codes decode through
    mxq_dequantize like any MXFP4 operand."""
    s = synthetic.attention_scores(seed=4)
    t = dev(s)
    codes, scales = mxq.exp_free_quantize(t)
    oc, os_ = oracle.exp_free_quantize(s)
    hc, hs = host(codes), host(scales)
    assert np.array_equal(hs, os_)
    assert np.array_equal(hc, oc)
    j = np.argmax(s, axis=1)
    r = np.arange(s.shape[0])
    assert np.all(hs[r, j // 32] == 125)
    assert np.all(((hc[r, j // 2] >> (4 * (j % 2))) & 0xF) == 0x6)
    assert not np.any(hc & 0x88)
    p = mxq.dequantize(codes[:8], scales[:8], "mxfp4", (8, s.shape[1]), torch.float32)
    ref = oracle.dequantize(hc[:8], hs[:8], "mxfp4", (8, s.shape[1]), "f32")
    assert np.array_equal(host(p).view(np.uint32), ref.view(np.uint32))
    assert mxq.mxq_check_device() == 0


def test_exp_free_errors():
    s = torch.zeros(4, 64, device="cuda")
    c = torch.empty(4, 32, dtype=torch.uint8, device="cuda")
    sc = torch.empty(4, 2, dtype=torch.uint8, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert mxq.mxq_exp_free_quantize(s.data_ptr(), 4, 64, c.data_ptr(), sc.data_ptr(), st) == 0
    assert mxq.mxq_exp_free_quantize(s.data_ptr(), 4, 48, c.data_ptr(), sc.data_ptr(), st) == 2   # cols % 32
    assert mxq.mxq_exp_free_quantize(s.data_ptr() + 4, 3, 32, c.data_ptr(), sc.data_ptr(), st) == 3  # misaligned
    assert mxq.mxq_exp_free_quantize(s.data_ptr(), 0, 64, c.data_ptr(), sc.data_ptr(), st) == 0   # empty
    torch.cuda.synchronize()
