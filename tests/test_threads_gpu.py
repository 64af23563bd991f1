"""GPU: calls from several host threads at once. The library keeps no per-call state (its only
caches, the resident-CTA counts, the tensor-map encoder and the device error word's address,
are guarded), so threads that each convert their own tensors on their own stream get, bit for
bit, the results of one thread calling alone. The calls cover a one-pass quantize, the
bulk-copy fake-quantize stream (2^19 blocks), the exp-then-quantize pipeline and the
column-direction quantize through tensor maps."""
import threading

import pytest

torch = pytest.importorskip("torch")
from block_scaled_microscaling_b200 import mxq  # noqa: E402

pytestmark = pytest.mark.gpu

THREADS = 4
ROUNDS = 10


def convert(x, s):
    c, sc = mxq.quantize(x, "mxfp6_e2m3")
    fq = mxq.fake_quantize(x, "axs6")
    ec, es = mxq.exp_quantize(s, "mxfp4")
    cc, cs = mxq.quantize_cols(x, "mxfp8")
    return [c, sc, fq, ec, es, cc, cs]


def test_concurrent_calls_from_host_threads():
    xs, ss = [], []
    for i in range(THREADS):
        g = torch.Generator(device="cuda").manual_seed(100 + i)
        xs.append(torch.randn((2048, 8192), generator=g, device="cuda"))  # 2^19 blocks, fp32
        ss.append(torch.randn((64, 8192), generator=g, device="cuda") * 3)
    want = [[t.clone() for t in convert(x, s)] for x, s in zip(xs, ss)]
    torch.cuda.synchronize()
    assert mxq.mxq_check_device() == 0

    got = [None] * THREADS
    errors = []

    def work(i):
        try:
            st = torch.cuda.Stream()
            with torch.cuda.stream(st):
                for _ in range(ROUNDS):
                    res = convert(xs[i], ss[i])
            st.synchronize()
            got[i] = res
        except Exception as e:  # reported below, in the test's own thread
            errors.append((i, repr(e)))

    ts = [threading.Thread(target=work, args=(i,)) for i in range(THREADS)]
    for t in ts:
        t.start()
    for t in ts:
        t.join(120)
    assert not any(t.is_alive() for t in ts)
    assert not errors, errors
    torch.cuda.synchronize()
    assert mxq.mxq_check_device() == 0
    for i in range(THREADS):
        for k, (a, b) in enumerate(zip(got[i], want[i])):
            assert a.dtype == b.dtype and a.shape == b.shape, (i, k)
            assert torch.equal(a, b), (i, k)
