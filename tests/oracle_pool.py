"""Oracle work the GPU tests hand to worker processes (CPU only: numpy, the seeded input
generator and the fp64 oracle; nothing here touches CUDA)."""

import os

import numpy as np

from mxfp4_quantized_moe_b200 import inputs
from oracle import mxfp4_oracle as O


def block(job):
    """One block of a stack checked on recorded inputs: job = (workload, seed, layer, x,
    logits, g) with x, logits, g the sampled tokens' block input, router logits and upstream
    gradient as the GPU saw them.  Returns the oracle's (out, dX, d_w, d_logits, w) and
    sum_h |g_h| |y_{j,h}| per token and slot."""
    os.environ.setdefault("OMP_NUM_THREADS", "2")
    wl, seed, l, x, logits, g = job
    inp = inputs.make_workload(wl, seed, layer=l, with_dy=False)
    W = inputs.as_numpy(inp, [])["W"]
    del inp
    f = O.moe_forward(x, logits, W, wl.k)
    dX, d_w, d_logits = O.moe_backward(g, f, W)
    # sum_h |g_h y_{j,h}| per (token, slot): the scale of the rounding of y in d_w = <g, y_j>
    y_abs = np.einsum("th,tjh->tj", np.abs(g), np.abs(f["y"]))
    return np.asarray(f["out"]), dX, d_w, d_logits, f["w"], y_abs
