"""Per-expert oracle work for the full-size parity tests, run in a spawned
process pool (each task is one expert; the layer's output and every gradient
are sums of independent per-expert terms).

A task treats every routed row of its expert as a token of its own with one
slot, so the oracle's outputs come back per row: w y (the row's share of
out), the row's share of grad_in, its route gradient, and the LoRA gradients
of the expert over the rows it was given. Where the layer clamps, the task
also compares the GPU's fp32 pre-activations of those rows with the oracle's
and recomputes the backward with the GPU's clamp decisions wherever the two
lie within `delta` of a bound (both decisions are then correct within fp32
accumulation error). Only data moves here; the arithmetic is the oracle's.
"""

from __future__ import annotations

import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _init() -> None:
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)


def expert_task(args):
    _init()
    from oracle import moe as omoe

    (e, base, lora, alpha, limit, x, dy, w, g_gpu, u_gpu, delta) = args
    layer = omoe.Layer(base["gate_q"], base["gate_s"], base["up_q"], base["up_s"], base["down_q"], base["down_s"],
                       lora, alpha=alpha, swiglu_limit=limit)
    m = x.shape[0]
    ids = np.zeros((m, 1), dtype=np.int64)
    out, ctx = omoe.forward(layer, x, ids, w[:, None])
    ec = ctx.experts[0]
    stats = {"max_dg": float(np.max(np.abs(g_gpu - ec.G))), "max_du": float(np.max(np.abs(u_gpu - ec.U))),
             "ambiguous": 0, "flipped": 0, "decided_apart": 0}
    masks = None
    if limit > 0:
        L = limit
        own_g = ec.G <= L
        own_u = (ec.U >= -L) & (ec.U <= L)
        gpu_g = g_gpu <= L
        gpu_u = (u_gpu >= -L) & (u_gpu <= L)
        amb_g = np.abs(ec.G - L) <= delta
        amb_u = (np.abs(ec.U - L) <= delta) | (np.abs(ec.U + L) <= delta)
        stats["ambiguous"] = int(amb_g.sum() + amb_u.sum())
        stats["flipped"] = int(((gpu_g != own_g) & amb_g).sum() + ((gpu_u != own_u) & amb_u).sum())
        # outside the band the two decisions must agree
        stats["decided_apart"] = int(((gpu_g != own_g) & ~amb_g).sum() + ((gpu_u != own_u) & ~amb_u).sum())
        masks = {0: (np.where(amb_g, gpu_g, own_g), np.where(amb_u, gpu_u, own_u))}
    gin, groute, grads = omoe.backward(layer, ctx, dy, masks=masks)
    return e, out, gin, groute[:, 0], {n: v[0] for n, v in grads.items()}, stats
