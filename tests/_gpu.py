"""GPU-side helpers for the parity tests: run the C-ABI layer on a Workload."""

from __future__ import annotations

from typing import Dict, Optional

import torch

from workloads import LORA_NAMES, Workload, lora_shapes

try:
    from int4_quantised_moe_b200 import binding as B
except ImportError:  # library not built: GPU tests are skipped by their marker guard
    B = None

DEV = "cuda"

# Tolerances of the method's target (forward output and grad_input: rel-L2
# <= 5e-3 and cosine >= 0.9999; LoRA gradients: rel-L2 <= 1e-2). dRoute has
# no stated bound; it takes the LoRA-gradient one with the forward cosine.
TOL_OUT = (5e-3, 0.9999)
TOL_DX = (5e-3, 0.9999)
TOL_ROUTE = (1e-2, 0.9999)
TOL_LORA = (1e-2, 0.999)


def make_layer(wl: Workload, max_tokens: Optional[int] = None) -> "B.Layer":
    c = wl.cfg
    return B.Layer.create(c.experts, c.top_k, c.hidden, c.inter, c.rank, c.alpha, c.swiglu_limit,
                          max_tokens or max(c.qlen, 1), wl.gate_q, wl.gate_s, wl.up_q, wl.up_s, wl.down_q, wl.down_s,
                          wl.lora, weight_format=c.weight_format)


def grad_buffers(wl: Workload, fill: float = 7.0) -> Dict[str, torch.Tensor]:
    return {n: torch.full(s, fill, dtype=torch.bfloat16, device=DEV) for n, s in lora_shapes(wl.cfg).items()}


def run_fwd_bwd(layer, wl: Workload, grads, accumulate=False, grad_scale=1.0, save=True):
    out = layer.forward(wl.expert_ids, wl.route_weights, wl.x, save_for_backward=save)
    gin = torch.full_like(wl.x, float("nan"))
    groute = torch.full(wl.expert_ids.shape, float("nan"), dtype=torch.float32, device=DEV)
    layer.backward(wl.grad_out, grads, accumulate=accumulate, grad_scale=grad_scale, grad_in=gin, grad_route=groute)
    return out, gin, groute
