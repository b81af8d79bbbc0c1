"""Seeded synthetic inputs for the MXFP4 MoE expert block (shared by tests, bench and smoke).

This module only draws random numbers and lays them out; it holds none of the
expert block's arithmetic.  The one computation here is the caller-side router
linear (logits = x @ W_r + b_r in fp32), which sits outside the block: the
block's entry points take the logits as an input.

Recipe (per layer, one CPU ``torch.Generator`` seeded with ``seed``, in this
fixed draw order): x ~ N(0,1) bf16 [T,H]; W_r ~ N(0,0.02) bf16 [H,E];
b_r ~ N(0,0.01) bf16 [E]; gate_up packed bytes uniform 0..255 [E,2I,H/2]
(so both nibbles are uniform over the 16 E2M1 codes); gate_up UE8M0 scales
uniform integers in [scale_lo, scale_hi] [E,2I,H/32]; gate_up bias ~ N(0,0.01)
bf16 [E,2I] (interleaved rows: gate j at 2j, up j at 2j+1); down packed bytes
[E,H,I/2]; down scales [E,H,I/32]; down bias ~ N(0,0.01) bf16 [E,H];
dY ~ N(0,1) bf16 [T,H].  For the skewed-routing workload the router bias is
replaced by b_e = -1.5 * s * ln(e + 1) (s = 1.2), which makes expert
popularity fall off like a Zipf law.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    I: int
    E: int
    k: int
    layers: int = 1
    zipf_s: float | None = None
    scale_lo: int = 119
    scale_hi: int = 123
    extra: dict = field(default_factory=dict)


WORKLOADS = {
    "tiny-moe-T64-H256-E8-k2": Workload("tiny-moe-T64-H256-E8-k2", 64, 256, 256, 8, 2),
    "gpt-oss-20b-moe-T8192": Workload("gpt-oss-20b-moe-T8192", 8192, 2880, 2880, 32, 4),
    # smaller batch of the same layer, for profiler captures that must stay a few GB
    "gpt-oss-20b-moe-T4096": Workload("gpt-oss-20b-moe-T4096", 4096, 2880, 2880, 32, 4),
    # small-token case: ~32 rows per expert, bound by streaming the packed weights
    "gpt-oss-20b-moe-T256": Workload("gpt-oss-20b-moe-T256", 256, 2880, 2880, 32, 4),
    "gpt-oss-120b-moe-T16384": Workload("gpt-oss-120b-moe-T16384", 16384, 2880, 2880, 128, 4),
    "gpt-oss-20b-moe-zipf-T16384": Workload("gpt-oss-20b-moe-zipf-T16384", 16384, 2880, 2880, 32, 4,
                                            zipf_s=1.2),
    "gpt-oss-20b-moe-stack24-T32768": Workload("gpt-oss-20b-moe-stack24-T32768", 32768, 2880, 2880,
                                               32, 4, layers=24),
}


def make_layer(T, H, I, E, k, seed, *, zipf_s=None, scale_lo=119, scale_hi=123, with_dy=True):
    """Draw one layer's inputs on the CPU.  Returns a dict of CPU torch tensors."""
    if H % 32 or I % 32:
        raise ValueError("H and I must be multiples of the 32-element MX block")
    g = torch.Generator().manual_seed(int(seed))
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    w_r = (torch.randn(H, E, generator=g) * 0.02).to(torch.bfloat16)
    b_r = (torch.randn(E, generator=g) * 0.01).to(torch.bfloat16)
    gu_blocks = torch.randint(0, 256, (E, 2 * I, H // 2), generator=g, dtype=torch.uint8)
    gu_scales = torch.randint(scale_lo, scale_hi + 1, (E, 2 * I, H // 32), generator=g,
                              dtype=torch.uint8)
    gu_bias = (torch.randn(E, 2 * I, generator=g) * 0.01).to(torch.bfloat16)
    dn_blocks = torch.randint(0, 256, (E, H, I // 2), generator=g, dtype=torch.uint8)
    dn_scales = torch.randint(scale_lo, scale_hi + 1, (E, H, I // 32), generator=g,
                              dtype=torch.uint8)
    dn_bias = (torch.randn(E, H, generator=g) * 0.01).to(torch.bfloat16)
    dy = torch.randn(T, H, generator=g).to(torch.bfloat16) if with_dy else None
    if zipf_s is not None:
        b_r = torch.tensor([-1.5 * zipf_s * math.log(e + 1) for e in range(E)]).to(torch.bfloat16)
    logits = x.float() @ w_r.float() + b_r.float()
    return {
        "T": T, "H": H, "I": I, "E": E, "k": k,
        "x": x, "w_r": w_r, "b_r": b_r, "logits": logits.contiguous(),
        "gu_blocks": gu_blocks, "gu_scales": gu_scales, "gu_bias": gu_bias,
        "dn_blocks": dn_blocks, "dn_scales": dn_scales, "dn_bias": dn_bias,
        "dy": dy,
    }


def make_workload(wl: Workload | str, seed: int = 0, layer: int = 0, **kw):
    """Inputs of one layer of a named workload (layer l of a stack uses seed + l)."""
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    return make_layer(wl.T, wl.H, wl.I, wl.E, wl.k, seed + layer, zipf_s=wl.zipf_s,
                      scale_lo=wl.scale_lo, scale_hi=wl.scale_hi, **kw)


def as_numpy(inp, tokens=None):
    """Values of a layer's tensors as float64/uint8 numpy arrays (optionally a token subset)."""
    sel = slice(None) if tokens is None else torch.as_tensor(tokens, dtype=torch.long)
    out = {
        "x": inp["x"][sel].double().numpy(),
        "logits": inp["logits"][sel].numpy(),
        "W": {
            "gu_blocks": inp["gu_blocks"].numpy(), "gu_scales": inp["gu_scales"].numpy(),
            "gu_bias": inp["gu_bias"].double().numpy(),
            "dn_blocks": inp["dn_blocks"].numpy(), "dn_scales": inp["dn_scales"].numpy(),
            "dn_bias": inp["dn_bias"].double().numpy(),
        },
    }
    if inp.get("dy") is not None:
        out["dy"] = inp["dy"][sel].double().numpy()
    return out
