"""Parity report: rel-L2 and cosine of every GPU output against the oracle.

Run on a GPU machine (``python -m tests.report_parity``); prints one JSON line
per config. Configs 0 and 1 are compared in full; for the large configs the
forward output, grad_input and dRoute are compared on sampled tokens (the
oracle runs on exactly those tokens' experts) and the LoRA gradients on the
most and the median loaded expert, as in ``test_gpu_fullsize.py``.
"""

from __future__ import annotations

import json

import numpy as np
import torch

from oracle import metrics
from oracle import moe as omoe
from oracle import rawint4 as orq
from tests._gpu import grad_buffers, make_layer, run_fwd_bwd
from tests._util import f64, oracle_run
from tests.test_gpu_fullsize import bits, sub_layer
from workloads import CONFIGS, LORA_NAMES, expert_counts, make_workload


def rel(a, e):
    r, c = metrics.relative_l2_and_cosine(np.asarray(a, np.float64), np.asarray(e, np.float64))
    return {"rel_l2": float(r), "cos": float(c)}


def full(cfg_id):
    cfg = CONFIGS[cfg_id]
    wl = make_workload(cfg, device="cuda")
    layer = make_layer(wl)
    grads = grad_buffers(wl)
    out, gin, groute = run_fwd_bwd(layer, wl, grads)
    _, o_out, o_gin, o_groute, o_grads = oracle_run(wl)
    rep = {"out": rel(f64(out), o_out), "grad_in": rel(f64(gin), o_gin), "grad_route": rel(f64(groute), o_groute)}
    for n in LORA_NAMES:
        rep[n] = rel(f64(grads[n]), o_grads[n])
    return rep


def sampled(cfg_id):
    cfg = CONFIGS[cfg_id]
    wl = make_workload(cfg, device="cuda")
    layer = make_layer(wl)
    grads = grad_buffers(wl)
    out, gin, groute = run_fwd_bwd(layer, wl, grads)
    Q = cfg.qlen
    toks = sorted({0, Q // 3, Q // 2, Q - 1})
    ids = wl.expert_ids.cpu().numpy()
    experts = sorted({int(e) for e in ids[toks].reshape(-1)})
    remap = {e: i for i, e in enumerate(experts)}
    o_layer = sub_layer(wl, experts)
    t = torch.as_tensor(toks, device="cuda")
    x = orq.bf16_bits_to_f64(bits(wl.x.index_select(0, t)))
    dy = orq.bf16_bits_to_f64(bits(wl.grad_out.index_select(0, t)))
    rw = wl.route_weights.cpu().numpy()[toks].astype(np.float64)
    o_out, ctx = omoe.forward(o_layer, x, np.vectorize(remap.get)(ids[toks]), rw)
    o_gin, o_groute, _ = omoe.backward(o_layer, ctx, dy)
    rep = {"tokens": toks, "out": rel(out.float().cpu().numpy()[toks], o_out),
           "grad_in": rel(gin.float().cpu().numpy()[toks], o_gin),
           "grad_route": rel(groute.cpu().numpy()[toks], o_groute)}
    counts = expert_counts(wl.expert_ids, cfg.experts).numpy()
    e = int(np.argsort(-counts, kind="stable")[0])
    sel = np.nonzero((ids == e).any(axis=1))[0]
    sub_ids = np.where(ids[sel] == e, 0, -1)
    o_layer = sub_layer(wl, [e])
    t = torch.as_tensor(sel, device="cuda")
    x = orq.bf16_bits_to_f64(bits(wl.x.index_select(0, t)))
    dy = orq.bf16_bits_to_f64(bits(wl.grad_out.index_select(0, t)))
    rw = wl.route_weights.cpu().numpy()[sel].astype(np.float64)
    _, ctx = omoe.forward(o_layer, x, sub_ids, rw)
    _, _, o_grads = omoe.backward(o_layer, ctx, dy)
    rep["lora_expert"] = e
    for n in LORA_NAMES:
        rep[n] = rel(grads[n][e].float().cpu().numpy(), o_grads[n][0])
    return rep


def main():
    for cfg_id in (0, 1):
        print(json.dumps({"config": cfg_id, "compare": "full", **full(cfg_id)}), flush=True)
    for cfg_id in (2, 3, 4):
        print(json.dumps({"config": cfg_id, "compare": "sampled", **sampled(cfg_id)}), flush=True)


if __name__ == "__main__":
    main()
