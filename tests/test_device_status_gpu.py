"""GPU: the bounded waits of the bulk-copy pipeline and their host-side report.

A wait that runs out is made to happen on purpose only in the library's self-test (one warp
waits on an mbarrier nothing arrives at, for 20 ms): the status must come back as
MXQ_ERR_TIMEOUT and the device must stay usable. No GPU fault, trap or unbounded wait is
involved."""
import numpy as np
import pytest

import oracle
import synthetic

torch = pytest.importorskip("torch")
from block_scaled_microscaling_b200 import mxq  # noqa: E402

pytestmark = pytest.mark.gpu


def test_selftest_wait_gives_up_and_is_reported():
    assert mxq.mxq_check_device() == 0
    assert mxq.mxq_selftest_timeout(20) == 6       # MXQ_ERR_TIMEOUT
    assert mxq.mxq_check_device() == 0             # the report clears the word
    # the context is intact: a pipeline run afterwards is correct and reports no timeout
    s = synthetic.attention_scores(seed=9, heads=1, queries=300, keys=4096)
    codes, scales = mxq.exp_quantize(torch.from_numpy(s).cuda(), "mxfp4")
    mxq.check_device()
    oc, os_ = oracle.exp_quantize(s, "mxfp4")
    assert np.array_equal(scales.cpu().numpy(), os_) and np.array_equal(codes.cpu().numpy(), oc)


def test_pipeline_full_size_reports_ok():
    s = torch.randn(4096, 32768, device="cuda") * 3
    for fmt in ("mxfp4", "mxfp8"):
        mxq.exp_quantize(s, fmt)
    assert mxq.mxq_check_device() == 0


def test_helpers_check_on_request():
    """check=True on the bulk-copy helpers synchronizes and reads the status word: a clean run
    returns normally (a timed-out one would raise MXQError with MXQ_ERR_TIMEOUT)."""
    s = torch.randn(64, 4096, device="cuda") * 3
    mxq.exp_quantize(s, "mxfp4", check=True)
    mxq.exp_free_quantize(s, check=True)
    x = torch.randn(512, 256, device="cuda")
    mxq.quantize_cols(x, "mxfp6_e2m3", check=True)
    g = torch.randn(1 << 19, 32, device="cuda")  # 2^19 blocks: the bulk-copy fake-quantize
    mxq.fake_quantize(g, "axs6", check=True)
    assert mxq.mxq_check_device() == 0
