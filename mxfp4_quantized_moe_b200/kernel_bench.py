"""Achieved HBM bandwidth of the memory-bound stages on one GPU.

    python -m mxfp4_quantized_moe_b200.kernel_bench [--iters N]

* standalone dequantization (`mxfp4_moe_dequantize`) of a whole gpt-oss-20b gate_up weight
  set, E*2I rows of H elements: 0.5 B of codes + 1/32 B of scale read and 2 B of bf16 written
  per element;
* the memory-bound kernels of one gpt-oss-20b layer step at T=8192, from the library's
  per-kernel event timing: the forward gather (`gather_x`: A rows of H bf16 read and
  written), the combines
  (`combine_y`, `combine_dx`: A rows read, T rows written) and the dY gather with the
  routing-weight dot (`gather_dy_dw`: A rows of dY and of y read, A rows written).

Prints one JSON line per stage with its algorithmic bytes, time and GB/s against the HBM copy
bandwidth in MEASURED_PEAKS.json (or the fallback figure).
"""

from __future__ import annotations

import argparse
import json
import os

import torch

from . import inputs, moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--iters", type=int, default=20)
    args = ap.parse_args()
    peak, src = hbm_peak()
    wl = inputs.WORKLOADS["gpt-oss-20b-moe-T8192"]
    inp = inputs.make_workload(wl, 0)
    dev = torch.device("cuda", 0)

    # ---- standalone dequantization of the gate_up weights -------------------------------
    blocks = inp["gu_blocks"].to(dev).reshape(-1, wl.H // 2)
    scales = inp["gu_scales"].to(dev).reshape(-1, wl.H // 32)
    rows, K = blocks.shape[0], wl.H
    out = torch.empty(rows, K, dtype=torch.bfloat16, device=dev)
    for _ in range(3):
        moe.dequantize(blocks, scales, out=out)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.iters):
        moe.dequantize(blocks, scales, out=out)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.iters
    nbytes = rows * K * (0.5 + 1 / 32 + 2.0)
    print(json.dumps({"stage": "dequant", "rows": rows, "K": K, "bytes": nbytes, "ms": ms,
                      "gbs": nbytes / (ms / 1e3) / 1e9, "frac_of_hbm": nbytes / (ms / 1e3) / 1e9 / peak,
                      "peak_gbs": peak, "peak_source": src}), flush=True)
    del out, blocks, scales
    torch.cuda.empty_cache()

    # ---- gathers and combines of a layer step ------------------------------------------
    shape = moe.MoeShape(wl.T, wl.H, wl.I, wl.E, wl.k)
    w = moe.weights_to(inp, dev)
    wt = moe.transpose_weights(shape, w)
    x, lg, dy = inp["x"].to(dev), inp["logits"].to(dev), inp["dy"].to(dev)
    ws = moe.alloc_workspace(shape, dev)
    y = torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device=dev)
    for _ in range(3):
        moe.forward(shape, w, x, lg, ws, y=y)
        moe.backward_input(shape, w, wt, dy, ws)
    torch.cuda.synchronize()
    moe.profile_begin()
    for _ in range(args.iters):
        moe.forward(shape, w, x, lg, ws, y=y)
        moe.backward_input(shape, w, wt, dy, ws)
    kt = moe.profile_end()
    A, T, H = wl.T * wl.k, wl.T, wl.H
    stages = (("gather_x", A * H * 2.0 * 2),
              ("combine_y", (A + T) * H * 2.0),
              ("gather_dy_dw", A * H * 2.0 * 3 + A * 4.0),
              ("combine_dx", (A + T) * H * 2.0))
    for name, nbytes in stages:
        launches, tot = kt[name]
        ms = tot / launches
        print(json.dumps({"stage": name, "bytes": nbytes, "ms": ms,
                          "gbs": nbytes / (ms / 1e3) / 1e9,
                          "frac_of_hbm": nbytes / (ms / 1e3) / 1e9 / peak,
                          "peak_gbs": peak, "peak_source": src}), flush=True)


if __name__ == "__main__":
    main()
