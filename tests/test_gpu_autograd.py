"""The block inside autograd: gradients to the activations through both the experts and the
caller's router linear, against the fp64 oracle (dX_total = dX_experts + d_logits W_r^T)."""

import numpy as np
import pytest
import torch

from mxfp4_quantized_moe_b200 import inputs
from oracle import mxfp4_oracle as O

from test_gpu_parity import assert_close

pytestmark = pytest.mark.gpu


def test_autograd_gradient_through_experts_and_router():
    from mxfp4_quantized_moe_b200 import moe
    from mxfp4_quantized_moe_b200.autograd import MoeLayer, moe_block
    T, H, I, E, k = 48, 128, 192, 8, 2
    inp = inputs.make_layer(T, H, I, E, k, 21)
    layer = MoeLayer(moe.MoeShape(T, H, I, E, k), moe.weights_to(inp, "cuda"))
    x = inp["x"].cuda().requires_grad_(True)
    w_r, b_r = inp["w_r"].cuda().float(), inp["b_r"].cuda().float()
    logits = x.float() @ w_r + b_r
    y = moe_block(x, logits, layer)
    y.backward(inp["dy"].cuda())
    torch.cuda.synchronize()
    assert moe.device_check(layer.ws) == (0, 0)

    n = inputs.as_numpy(inp)
    lg = logits.detach().cpu().numpy().astype(np.float64)  # the logits the GPU routed on
    f = O.moe_forward(n["x"], lg, n["W"], k)
    dX, d_w, d_logits = O.moe_backward(n["dy"], f, n["W"])
    ref_dx = dX + d_logits @ inp["w_r"].double().numpy().T
    assert_close(y.detach().float().cpu().numpy(), f["out"], "y")
    assert_close(x.grad.float().cpu().numpy(), ref_dx, "dx_total")

    # the workspace holds one forward's state: a second backward of the same graph is refused
    y2 = moe_block(x, logits.detach(), layer)
    moe_block(x, logits.detach(), layer)  # a later forward overwrites the state
    with pytest.raises(RuntimeError):
        y2.backward(inp["dy"].cuda())
