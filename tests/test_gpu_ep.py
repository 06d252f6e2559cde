"""Expert parallelism through the library on one B200: a one-process NCCL
group, so every slot stays on the process, but the step runs the whole
expert-parallel path with the library's kernels: the slot plan
(rawint4_moe_permute on the owning process), the row dispatch, the local
layer with top_k = 1 over the received slots, the NCCL all-to-alls, the
combine of the returned rows and the dRoute gather. The results must match
the float64 oracle of the whole layer. The multi-process exchanges are
covered on CPU by tests/test_ep_gloo.py (this pool runs one GPU per job).
"""

from __future__ import annotations

import dataclasses
import socket

import pytest
import torch

from oracle import metrics, moe as omoe
from tests._gpu import TOL_DX, TOL_LORA, TOL_OUT, TOL_ROUTE, grad_buffers
from tests._util import f64, oracle_layer
from workloads import CONFIGS, LORA_NAMES, make_workload

pytestmark = pytest.mark.gpu


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _close(name, got, ref, tol):
    rel, cos = metrics.relative_l2_and_cosine(f64(got), ref)
    assert rel <= tol[0] and cos >= tol[1], f"{name}: rel-L2 {rel:.3e}, cos {cos:.6f}"


@pytest.mark.parametrize("fmt", ["rawint4", "mxfp4"])
def test_expert_parallel_one_process(fmt):
    import torch.distributed as dist

    from int4_quantised_moe_b200 import binding as B
    from int4_quantised_moe_b200 import ep

    cfg = dataclasses.replace(CONFIGS[1], swiglu_limit=0.0, weight_format=fmt)
    wl = make_workload(cfg)
    g = wl.to("cuda")
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1)
    try:
        cap = cfg.qlen * cfg.top_k
        local = B.Layer.create(cfg.experts, 1, cfg.hidden, cfg.inter, cfg.rank, cfg.alpha, cfg.swiglu_limit, cap,
                               g.gate_q, g.gate_s, g.up_q, g.up_s, g.down_q, g.down_s, g.lora,
                               weight_format=cfg.weight_format)
        layer = ep.ExpertParallelLayer(dist, cfg.experts, cfg.top_k, local, capacity=cap)
        out = layer.forward(g.expert_ids, g.route_weights, g.x)
        grads = grad_buffers(g)
        groute = torch.full(g.expert_ids.shape, float("nan"), dtype=torch.float32, device="cuda")
        gin = layer.backward(g.grad_out, grads, grad_route=groute)
        torch.cuda.synchronize()
        assert local.status() == 0
    finally:
        dist.destroy_process_group()
    olayer = oracle_layer(wl)
    o_out, ctx = omoe.forward(olayer, f64(wl.x), wl.expert_ids.numpy(), f64(wl.route_weights))
    o_gin, o_groute, o_grads = omoe.backward(olayer, ctx, f64(wl.grad_out))
    _close("out", out, o_out, TOL_OUT)
    _close("grad_in", gin, o_gin, TOL_DX)
    _close("grad_route", groute, o_groute, TOL_ROUTE)
    for n in LORA_NAMES:
        _close(n, grads[n], o_grads[n], TOL_LORA)


def test_row_moves_are_exact():
    """The three row-movement exports against their definitions, bit for bit."""
    from int4_quantised_moe_b200 import binding as B

    gen = torch.Generator().manual_seed(7)
    q, k, h = 37, 3, 264
    src = torch.randn((q, h), generator=gen).to(torch.bfloat16).cuda()
    owner = torch.randint(-1, 4, (q, k), generator=gen).cuda()
    offsets = torch.empty(5, dtype=torch.int32, device="cuda")
    perm = torch.empty(q * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(q * k, dtype=torch.int32, device="cuda")
    B.rawint4_moe_permute(owner, 4, offsets, perm, inv)
    n = int(offsets[4])
    dst = torch.empty((n, h), dtype=torch.bfloat16, device="cuda")
    B.rawint4_moe_dispatch_rows(src, perm, n, k, dst)
    assert torch.equal(dst, src[perm[:n].long() // k])
    rows = torch.randn((n, h), generator=gen).to(torch.bfloat16).cuda()
    out = torch.empty((q, h), dtype=torch.bfloat16, device="cuda")
    B.rawint4_moe_combine_slots(rows, inv, q, k, out)
    inv2 = inv.view(q, k).long()
    ref = torch.zeros((q, h), dtype=torch.float32, device="cuda")
    for s in range(k):
        ok = inv2[:, s] >= 0
        ref[ok] += rows[inv2[ok, s]].float()
    assert torch.equal(out, ref.to(torch.bfloat16))
    vals = torch.randn(n, generator=gen).cuda()
    got = torch.empty(q * k, dtype=torch.float32, device="cuda")
    B.rawint4_moe_gather_slots(vals, inv, got)
    want = torch.where(inv >= 0, vals[inv.clamp(min=0).long()] if n else torch.zeros_like(got), torch.zeros_like(got))
    assert torch.equal(got, want)
