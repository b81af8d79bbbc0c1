"""Failure detection on the GPU, without a fault.

The library bounds every device-side wait.  The self-test entry point runs a kernel whose
waits nothing ever completes: the first must run out after the one-second limit and report
DEVICE_TIMEOUT with its tag through the workspace error word, the second must leave through
the kernel's abort flag, the kernel must free its tensor memory and return, and the CUDA
context must stay usable (a later kernel still computes exact results).
"""

import time

import numpy as np
import pytest
import torch

from mxfp4_quantized_moe_b200 import _lib as L
from oracle import mxfp4_oracle as O

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_the_context_survives():
    from mxfp4_quantized_moe_b200 import moe
    ws = torch.zeros(64, dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    moe.selftest_wait_timeout(ws)
    rc, where = moe.device_check(ws)
    dt = time.perf_counter() - t0
    assert rc == L.ERR_DEVICE_TIMEOUT, L.strerror(rc)
    assert where == 0xF00
    assert int(ws.view(torch.int32)[2]) == 1, "the second wait did not leave through the abort flag"
    assert 0.9 < dt < 30.0
    # the check cleared the error word
    assert moe.device_check(ws) == (0, 0)
    # the context still runs kernels: an exact dequantization afterwards
    g = torch.Generator().manual_seed(5)
    blocks = torch.randint(0, 256, (64, 32), generator=g, dtype=torch.uint8)
    scales = torch.randint(119, 124, (64, 2), generator=g, dtype=torch.uint8)
    out = moe.dequantize(blocks.cuda(), scales.cuda())
    ref = O.f64_to_bf16_bits(O.dequantize(blocks.numpy(), scales.numpy()))
    got = out.view(torch.int16).cpu().numpy().astype(np.uint16)
    assert np.array_equal(got, ref.astype(np.uint16))


def test_selftest_rejects_a_short_workspace():
    from mxfp4_quantized_moe_b200 import moe
    ws = torch.zeros(8, dtype=torch.uint8, device="cuda")
    with pytest.raises(L.MoeError):
        moe.selftest_wait_timeout(ws)
