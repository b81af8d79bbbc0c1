"""A residual stack of MXFP4 MoE blocks with a recompute-per-block backward.

    x_{l+1} = x_l + MoE_l(x_l, logits_l),   logits_l = x_l W_r^l + b_r^l   (fp32)

The blocks are the library's entry points (mxfp4_moe_forward / mxfp4_moe_backward_input);
the caller's side of the block boundary is two more of its kernels: mxfp4_moe_residual_router
forms x_{l+1} = bf16(x_l + y_l) and the next block's logits from one read of x_l and y_l, and
mxfp4_moe_grad_chain forms g_l below.  The backward is activation checkpointing at block
granularity: the forward keeps only each block's input x_l (bf16); the backward re-runs
block l's forward from x_l to refill the one shared workspace, then runs its input-gradient
backward, so at most one block's transients are alive at any time.

Chain rule per block (g_{l+1} = dL/dx_{l+1}):
    g_l = g_{l+1} + dX_moe_l + d_logits_l (W_r^l)^T
with dX_moe_l and d_logits_l returned by the block's backward for upstream gradient g_{l+1}.
Sums are taken in fp32 and rounded to bf16 once per block, like the residual stream.

The forward checkpoints each block's input x_l together with its logits_l (T x E fp32, a
few MB a block), so the recompute needs no router call.  The block functions and the two
caller-side steps are injectable, so that the chaining itself can be checked on the CPU
against an fp64 reference without a GPU.

Source: "Add MXFP4 training support via a dequantize-on-the-fly fallback" (the MoE block of
a decoder layer trained with gradient checkpointing over packed frozen weights).
"""

from __future__ import annotations

import argparse
import json
from dataclasses import dataclass
from typing import Callable

import torch


@dataclass
class StackBlock:
    """One block's operands on the device: packed weights (dict as `moe.weights_to` returns),
    the transposed copy for the backward, and the router linear W_r [H,E], b_r [E]."""
    w: dict
    wt: torch.Tensor | None
    w_r: torch.Tensor
    b_r: torch.Tensor


class MoeStack:
    """Forward and recompute-per-block backward over a list of blocks.

    `block_forward(l, x, logits) -> y` and `block_backward(l, g) -> (dx, d_logits)` default to
    the library's entry points on one shared workspace; `block_backward` sees the workspace
    that the immediately preceding `block_forward(l, ...)` left.
    `residual_router(x, y, w_r, b_r) -> (x + y or None, logits or None)` (y None: logits of
    x; w_r None: no logits) and `grad_chain(g, dx, d_logits, w_r)` default to the library's
    mxfp4_moe_residual_router and mxfp4_moe_grad_chain."""

    def __init__(self, shape, blocks: list[StackBlock], device=None,
                 block_forward: Callable | None = None, block_backward: Callable | None = None,
                 residual_router: Callable | None = None, grad_chain: Callable | None = None):
        self.shape = shape
        self.blocks = blocks
        if residual_router is None or grad_chain is None:
            from . import moe
            self._moe = moe
        self.residual_router = residual_router or self._lib_residual_router
        self.grad_chain = grad_chain or self._lib_grad_chain
        if block_forward is None or block_backward is None:
            from . import moe
            self._moe = moe
            dev = blocks[0].w_r.device if device is None else torch.device(device)
            self.ws = moe.alloc_workspace(shape, dev)
            T, H = shape.T, shape.H
            self._y = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
            self._dx = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
            self._dtw = torch.empty(T, shape.k, dtype=torch.float32, device=dev)
            self._dl = torch.empty(T, shape.E, dtype=torch.float32, device=dev)
        self.block_forward = block_forward or self._lib_forward
        self.block_backward = block_backward or self._lib_backward

    # ---- the library's entry points ------------------------------------------------------
    def _lib_forward(self, l, x, logits):
        return self._moe.forward(self.shape, self.blocks[l].w, x, logits, self.ws, y=self._y)

    def _lib_backward(self, l, g):
        b = self.blocks[l]
        dx, dtw, dl = self._moe.backward_input(self.shape, b.w, b.wt, g, self.ws, dx=self._dx,
                                               d_topk_w=self._dtw, d_logits=self._dl)
        return dx, dl, dtw

    def _lib_residual_router(self, x, y, w_r, b_r):
        return self._moe.residual_router(x, y, w_r, b_r)

    def _lib_grad_chain(self, g, dx, d_logits, w_r):
        return self._moe.grad_chain(g, dx, d_logits, w_r)

    # ---- the stack -----------------------------------------------------------------------
    def forward(self, x: torch.Tensor, tap: Callable | None = None):
        """Returns (x_L, saved), saved[l] = (x_l, logits_l) for the recompute.  `tap(l, dict)`
        sees each block's x, logits, y."""
        saved = []
        first = self.blocks[0]
        logits = self.residual_router(x, None, first.w_r, first.b_r)[1]
        for l in range(len(self.blocks)):
            saved.append((x, logits))
            y = self.block_forward(l, x, logits)
            if tap is not None:
                tap(l, {"x": x, "logits": logits, "y": y})
            nxt = self.blocks[l + 1] if l + 1 < len(self.blocks) else None
            # x_{l+1} and, for the next block, its router logits, from one read of x_l and y_l
            x, logits = self.residual_router(x, y, nxt.w_r if nxt else None,
                                             nxt.b_r if nxt else None)
        return x, saved

    def backward(self, dy: torch.Tensor, saved: list, tap: Callable | None = None):
        """dL/dx_0 from dL/dx_L, re-running each block's forward from its saved input."""
        g = dy
        for l in reversed(range(len(self.blocks))):
            b = self.blocks[l]
            x, logits = saved[l]
            self.block_forward(l, x, logits)  # recompute: refills the block's saved state
            out = self.block_backward(l, g)
            dx_moe, d_logits = out[0], out[1]
            if tap is not None:
                tap(l, {"g": g, "dx": dx_moe, "d_logits": d_logits,
                        "d_w": out[2] if len(out) > 2 else None})
            g = self.grad_chain(g, dx_moe, d_logits, b.w_r)
        return g


def build_stack(wl, seed: int = 0, device="cuda", layers: int | None = None):
    """Device blocks of a stacked workload (layer l drawn from seed + l), the stack input x
    (layer 0's x draw) and the upstream gradient dY (layer 0's dY draw)."""
    from . import inputs, moe
    n_layers = wl.layers if layers is None else layers
    shape = moe.MoeShape(wl.T, wl.H, wl.I, wl.E, wl.k)
    blocks, x, dy = [], None, None
    for l in range(n_layers):
        inp = inputs.make_workload(wl, seed, layer=l, with_dy=(l == 0))
        if l == 0:
            x, dy = inp["x"].to(device), inp["dy"].to(device)
        w = moe.weights_to(inp, device)
        wt = moe.transpose_weights(shape, w)
        blocks.append(StackBlock(w, wt, inp["w_r"].to(device), inp["b_r"].to(device)))
        del inp
    return shape, blocks, x, dy


def main():
    """Times the stack's forward + recompute backward on one GPU and reports peak memory."""
    from . import inputs
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="gpt-oss-20b-moe-stack24-T32768")
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=1)
    args = ap.parse_args()
    wl = inputs.WORKLOADS[args.workload]
    shape, blocks, x, dy = build_stack(wl)
    st = MoeStack(shape, blocks)
    for _ in range(args.warmup):
        out, saved = st.forward(x)
        st.backward(dy, saved)
        del out, saved
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        out, saved = st.forward(x)
        st.backward(dy, saved)
        del out, saved
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    A = wl.T * wl.k
    model_flop = 12.0 * A * wl.H * wl.I * wl.layers
    exec_flop = model_flop * 1.5  # the recompute repeats every block's forward (half the work)
    print(json.dumps({
        "workload": wl.name, "layers": wl.layers, "ms_per_step": ms,
        "tokens_per_s": wl.T / (ms / 1e3),
        "model_tflops": model_flop / (ms / 1e3) / 1e12,
        "executed_tflops": exec_flop / (ms / 1e3) / 1e12,
        "peak_memory_gb": torch.cuda.max_memory_allocated() / 1e9,
        "resident_weights_gb": sum(
            sum(int(t.numel()) * t.element_size() for t in b.w.values()) +
            int(b.wt.numel()) * b.wt.element_size() for b in blocks) / 1e9,
    }), flush=True)


if __name__ == "__main__":
    main()
