"""Test helpers: torch tensors <-> NumPy views and Workload -> oracle Layer.

Only conversions live here (exact bf16 -> float64, uint8 passthrough). No
arithmetic of the method.
"""

from __future__ import annotations

import numpy as np
import torch

from oracle import moe as omoe
from oracle import rawint4 as orq
from workloads import LORA_NAMES, Workload


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def f64(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return orq.bf16_bits_to_f64(bf16_bits(t))
    return t.detach().cpu().to(torch.float64).numpy()


def u8(t: torch.Tensor) -> np.ndarray:
    assert t.dtype == torch.uint8
    return t.detach().cpu().contiguous().numpy()


def oracle_layer(wl: Workload, lazy_scales: bool = False) -> omoe.Layer:
    """``lazy_scales`` keeps scales as bf16 bit patterns (widened per expert)."""
    c = wl.cfg
    if c.weight_format == "mxfp4":
        sc = u8  # UE8M0 scale bytes, as stored
    else:
        sc = bf16_bits if lazy_scales else f64
    return omoe.Layer(
        gate_q=u8(wl.gate_q), gate_s=sc(wl.gate_s),
        up_q=u8(wl.up_q), up_s=sc(wl.up_s),
        down_q=u8(wl.down_q), down_s=sc(wl.down_s),
        lora={n: f64(wl.lora[n]) for n in LORA_NAMES},
        alpha=c.alpha, swiglu_limit=c.swiglu_limit, weight_format=c.weight_format,
    )


def oracle_run(wl: Workload, experts=None):
    layer = oracle_layer(wl)
    out, ctx = omoe.forward(layer, f64(wl.x), wl.expert_ids.cpu().numpy(), f64(wl.route_weights), experts=experts)
    gin, groute, grads = omoe.backward(layer, ctx, f64(wl.grad_out))
    return layer, out, gin, groute, grads
