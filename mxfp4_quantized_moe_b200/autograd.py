"""The expert block as a torch.autograd.Function, for adapter training over frozen MXFP4 experts.

    layer = MoeLayer(shape, weights)              # packed weights on the GPU, prepared once
    y = moe_block(x, logits, layer)               # x bf16 [T,H], logits fp32 [T,E] (may need grad)
    y.backward(dy)                                # x.grad and logits.grad; no weight gradient

The forward and backward are the library's entry points; this module only wires them into
autograd.  The forward leaves the state the backward needs (routing, permutation, GLU output
and derivative factors) in the layer's workspace, so a layer's backward must follow its own
forward before that layer runs forward again: one MoeLayer per block in the graph, or
recompute the forward before the backward (see stack.py).

Source: "Add MXFP4 training support via a dequantize-on-the-fly fallback" (sections "What this
does" and "Relation to the backward triton kernels": gradients reach the inputs through the
expert math; the frozen quantized base gets no weight gradient).
"""

from __future__ import annotations

import torch

from . import moe


class MoeLayer:
    """One block's frozen packed weights with its transposed backward copy and workspace."""

    def __init__(self, shape: moe.MoeShape, weights: dict, device=None):
        self.shape = shape
        self.w = weights
        dev = weights["gu_blocks"].device if device is None else torch.device(device)
        self.wt = moe.transpose_weights(shape, weights)
        self.ws = moe.alloc_workspace(shape, dev)
        self.forwards = 0       # forwards run on this workspace
        self.consumed = True    # the latest forward's state was used by a backward


class _MoeBlock(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x: torch.Tensor, logits: torch.Tensor, layer: MoeLayer):
        y = moe.forward(layer.shape, layer.w, x.contiguous(), logits.contiguous(), layer.ws)
        layer.forwards += 1
        layer.consumed = False
        ctx.layer = layer
        ctx.forward_id = layer.forwards
        return y

    @staticmethod
    def backward(ctx, dy: torch.Tensor):
        layer = ctx.layer
        if layer.forwards != ctx.forward_id or layer.consumed:
            raise RuntimeError("MoeLayer: the workspace no longer holds this forward's state "
                               "(another forward or backward of the layer ran in between)")
        dx, _, d_logits = moe.backward_input(layer.shape, layer.w, layer.wt,
                                             dy.to(torch.bfloat16).contiguous(), layer.ws)
        layer.consumed = True
        return dx, d_logits, None


def moe_block(x: torch.Tensor, logits: torch.Tensor, layer: MoeLayer) -> torch.Tensor:
    """y = MoE(x, logits) with gradients to x and logits (bf16 x, fp32 logits, bf16 y)."""
    return _MoeBlock.apply(x, logits, layer)
