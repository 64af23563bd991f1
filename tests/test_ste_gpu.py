"""Straight-through estimator around the fused fake-quantize (GPU)."""
import numpy as np
import pytest

import oracle
import synthetic

torch = pytest.importorskip("torch")
from block_scaled_microscaling_b200 import fake_quantize_ste, mxq  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt", ["axs6", "mxfp6_e2m3", "mxfp4"])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_forward_is_the_fused_kernel_and_backward_is_identity(fmt, dtype):
    x32 = synthetic.gaussian((64, 256), 1.0, seed=21, dtype="f32")
    x = torch.from_numpy(x32).to("cuda", dtype).requires_grad_(True)
    y = fake_quantize_ste(x, fmt)
    ref = mxq.fake_quantize(x.detach(), fmt)
    assert torch.equal(y.detach().view(torch.int16 if dtype == torch.bfloat16 else torch.int32),
                       ref.view(torch.int16 if dtype == torch.bfloat16 else torch.int32))
    g = torch.randn_like(x)
    y.backward(g)
    assert torch.equal(x.grad, g)
    if dtype == torch.float32:
        assert np.array_equal(y.detach().cpu().numpy().view(np.uint32),
                              oracle.fake_quantize(x32, fmt).view(np.uint32))


def test_ste_in_a_linear_layer_trains():
    """Least squares through an AXS-6 fake-quantized weight: with the straight-through
    gradient the loss falls to the quantization floor, like the unquantized fit."""
    torch.manual_seed(0)
    w_true = torch.randn(64, 128, device="cuda") * 0.5
    xs = torch.randn(512, 128, device="cuda")
    ys = xs @ w_true.T

    def fit(q):
        w = torch.zeros(64, 128, device="cuda", requires_grad=True)
        opt = torch.optim.SGD([w], lr=8.0)
        losses = []
        for _ in range(150):
            opt.zero_grad()
            wq = fake_quantize_ste(w, "axs6") if q else w
            loss = ((xs @ wq.T - ys) ** 2).mean()
            loss.backward()
            opt.step()
            losses.append(float(loss.detach()))
        return losses

    plain, ste = fit(False), fit(True)
    assert plain[-1] < 1e-4 * plain[0]
    # the floor: the loss of the best fit quantized to AXS-6
    floor = float(((xs @ mxq.fake_quantize(w_true.contiguous(), "axs6").T - ys) ** 2).mean())
    assert ste[-1] < 0.02 * ste[0]
    assert ste[-1] < 10 * floor + 1e-6
