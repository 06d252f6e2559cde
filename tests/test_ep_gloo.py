"""Expert-parallel host logic on CPU: two gloo ranks, world size 2.

Each rank owns half of config 1's experts and half of its tokens. The
expert-parallel layer (``int4_quantised_moe_b200.ep``) plans the slot moves,
exchanges counts, token rows, local expert ids, route weights, results and
gradients with all-to-alls, and combines the returned rows. Here the four
row-movement calls are torch restatements of the library's and the per-rank
layer is the float64 oracle over the rank's experts with top_k = 1 (results
rounded to bf16, gradients stored in bf16 buffers as the library stores
them), so the test checks the plumbing: the output, grad_in, dRoute and each
rank's LoRA gradients must match the oracle of the whole layer over all
tokens.
"""

from __future__ import annotations

import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from int4_quantised_moe_b200 import ep
from oracle import metrics
from oracle import moe as omoe
from tests._util import f64, oracle_layer
from workloads import CONFIGS, LORA_NAMES, make_workload

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16)


# --- torch restatements of the library's row-movement calls (test doubles) ---

def _permute(owner: torch.Tensor, world: int, offsets, perm, inv) -> None:
    flat = owner.reshape(-1)
    valid = (flat >= 0) & (flat < world)
    slots = torch.nonzero(valid).reshape(-1)
    order = torch.sort(flat[slots], stable=True).indices
    chosen = slots[order]
    n = chosen.numel()
    counts = torch.bincount(flat[slots], minlength=world)
    offsets[0] = 0
    offsets[1:] = torch.cumsum(counts, 0).to(torch.int32)
    perm.fill_(-1)
    perm[:n] = chosen.to(torch.int32)
    inv.fill_(-1)
    inv[chosen] = torch.arange(n, dtype=torch.int32)


def _dispatch_rows(src, perm, n, k, dst) -> None:
    dst[:n] = src[perm[:n].to(torch.int64) // k]


def _combine_slots(src, inv, q, k, out) -> None:
    acc = torch.zeros((q, out.shape[1]), dtype=torch.float32)
    inv2 = inv[: q * k].reshape(q, k).to(torch.int64)
    for s in range(k):
        p = inv2[:, s]
        ok = p >= 0
        acc[ok] += src[p[ok]].float()
    out.copy_(acc.to(torch.bfloat16))


def _gather_slots(src, inv, out) -> None:
    p = inv[: out.numel()].to(torch.int64)
    ok = p >= 0
    out.zero_()
    out[ok] = src[p[ok]]


class _OracleLocalLayer:
    """The per-rank layer: the float64 oracle over this rank's experts with
    top_k = 1, with the library's bf16 outputs and gradient buffers."""

    def __init__(self, wl, lo: int, hi: int):
        full = oracle_layer(wl)
        self.layer = omoe.Layer(full.gate_q[lo:hi], full.gate_s[lo:hi], full.up_q[lo:hi], full.up_s[lo:hi],
                                full.down_q[lo:hi], full.down_s[lo:hi], {n: full.lora[n][lo:hi] for n in LORA_NAMES},
                                full.alpha, full.swiglu_limit)
        self.ctx = None

    def forward(self, ids, w, x, save_for_backward=True):
        out, ctx = omoe.forward(self.layer, f64(x), ids.numpy(), f64(w))
        self.ctx = ctx if save_for_backward else None
        return _bf16(out)

    def backward(self, g, grads, accumulate=False, grad_scale=1.0, grad_in=None, grad_route=None):
        gin, groute, lgrads = omoe.backward(self.layer, self.ctx, f64(g))
        self.ctx = None
        for n in LORA_NAMES:
            base = grads[n].double().numpy() if accumulate else 0.0
            grads[n].copy_(_bf16(base + grad_scale * lgrads[n]))
        grad_in.copy_(_bf16(gin))
        grad_route.copy_(torch.from_numpy(np.ascontiguousarray(groute)).float().reshape(grad_route.shape))


def _worker(rank: int, world: int, port: int, out_dir: str) -> None:
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = CONFIGS[1]
        wl = make_workload(cfg, device="cpu")
        per = cfg.experts // world
        q0, q1 = rank * cfg.qlen // world, (rank + 1) * cfg.qlen // world
        local = _OracleLocalLayer(wl, rank * per, (rank + 1) * per)
        ops = ep.KernelOps(permute=_permute, dispatch_rows=_dispatch_rows, combine_slots=_combine_slots,
                           gather_slots=_gather_slots)
        layer = ep.ExpertParallelLayer(dist, cfg.experts, cfg.top_k, local, capacity=cfg.qlen * cfg.top_k, ops=ops)
        ids = wl.expert_ids[q0:q1].contiguous()
        out = layer.forward(ids, wl.route_weights[q0:q1].contiguous(), wl.x[q0:q1].contiguous())
        grads = {n: torch.full(wl.lora[n][rank * per:(rank + 1) * per].shape, float("nan"), dtype=torch.bfloat16)
                 for n in LORA_NAMES}
        groute = torch.empty(ids.shape, dtype=torch.float32)
        gin = layer.backward(wl.grad_out[q0:q1].contiguous(), grads, accumulate=False, grad_scale=1.0,
                             grad_route=groute)
        torch.save({"out": out, "gin": gin, "groute": groute, "grads": grads},
                   os.path.join(out_dir, f"ep_rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


def test_expert_parallel_matches_whole_layer(tmp_path):
    mp.spawn(_worker, args=(WORLD, _free_port(), str(tmp_path)), nprocs=WORLD, join=True)
    parts = [torch.load(os.path.join(tmp_path, f"ep_rank{r}.pt")) for r in range(WORLD)]
    cfg = CONFIGS[1]
    wl = make_workload(cfg, device="cpu")
    layer = oracle_layer(wl)
    o_out, ctx = omoe.forward(layer, f64(wl.x), wl.expert_ids.numpy(), f64(wl.route_weights))
    o_gin, o_groute, o_grads = omoe.backward(layer, ctx, f64(wl.grad_out))

    def close(name, got, ref, tol):
        rel, cos = metrics.relative_l2_and_cosine(got.double().numpy() if isinstance(got, torch.Tensor) else got, ref)
        assert rel <= tol, f"{name}: rel-L2 {rel:.3e} > {tol}"

    close("out", torch.cat([p["out"] for p in parts]), o_out, 5e-3)
    close("grad_in", torch.cat([p["gin"] for p in parts]), o_gin, 5e-3)
    close("grad_route", torch.cat([p["groute"] for p in parts]), o_groute, 1e-6)
    per = cfg.experts // WORLD
    for n in LORA_NAMES:
        got = torch.cat([p["grads"][n] for p in parts])
        close(n, got, o_grads[n], 1e-2)
    # each rank holds gradients of its own experts only, all of them written
    for r, p in enumerate(parts):
        for n in LORA_NAMES:
            assert p["grads"][n].shape[0] == per
            assert torch.isfinite(p["grads"][n]).all()


def _edge_worker(rank: int, world: int, port: int, out_dir: str) -> None:
    """Rank 1 has no tokens; rank 0's tokens include slots with an expert id
    outside [0, E) (dropped) and every slot of rank 0 goes to rank 1's
    experts or nowhere, so rank 0 receives nothing and rank 1 sends nothing."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = CONFIGS[1]
        wl = make_workload(cfg, device="cpu")
        per = cfg.experts // world
        local = _OracleLocalLayer(wl, rank * per, (rank + 1) * per)
        ops = ep.KernelOps(permute=_permute, dispatch_rows=_dispatch_rows, combine_slots=_combine_slots,
                           gather_slots=_gather_slots)
        layer = ep.ExpertParallelLayer(dist, cfg.experts, cfg.top_k, local, capacity=cfg.qlen * cfg.top_k, ops=ops)
        q = 16 if rank == 0 else 0
        ids = torch.remainder(wl.expert_ids[:q], per) + per  # rank 1's experts
        if q:
            ids[::3, 1] = -1
            ids[1::5, 0] = cfg.experts + 2
        w = wl.route_weights[:q].contiguous()
        x = wl.x[:q].contiguous()
        out = layer.forward(ids.contiguous(), w, x)
        grads = {n: torch.full(wl.lora[n][rank * per:(rank + 1) * per].shape, float("nan"), dtype=torch.bfloat16)
                 for n in LORA_NAMES}
        groute = torch.full(ids.shape, float("nan"), dtype=torch.float32)
        gin = layer.backward(wl.grad_out[:q].contiguous(), grads, grad_route=groute)
        torch.save({"out": out, "gin": gin, "groute": groute, "grads": grads, "ids": ids},
                   os.path.join(out_dir, f"edge_rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


def test_expert_parallel_empty_and_dropped_slots(tmp_path):
    mp.spawn(_edge_worker, args=(WORLD, _free_port(), str(tmp_path)), nprocs=WORLD, join=True)
    p0, p1 = (torch.load(os.path.join(tmp_path, f"edge_rank{r}.pt")) for r in range(WORLD))
    cfg = CONFIGS[1]
    wl = make_workload(cfg, device="cpu")
    ids = p0["ids"].numpy()
    valid = np.where((ids >= 0) & (ids < cfg.experts), ids, -1)
    layer = oracle_layer(wl)
    o_out, ctx = omoe.forward(layer, f64(wl.x[:16]), valid, f64(wl.route_weights[:16]))
    o_gin, o_groute, o_grads = omoe.backward(layer, ctx, f64(wl.grad_out[:16]))
    for name, got, ref, tol in (("out", p0["out"], o_out, 5e-3), ("grad_in", p0["gin"], o_gin, 5e-3)):
        rel, _ = metrics.relative_l2_and_cosine(got.double().numpy(), ref)
        assert rel <= tol, f"{name}: rel-L2 {rel:.3e}"
    # dropped slots: no route gradient; the others match
    dropped = valid < 0
    assert torch.all(p0["groute"][torch.from_numpy(dropped)] == 0)
    np.testing.assert_allclose(p0["groute"].double().numpy()[~dropped], o_groute[~dropped], rtol=1e-5, atol=1e-7)
    # rank 0 received nothing: its experts' gradients are zero; rank 1 had no tokens
    per = cfg.experts // WORLD
    for n in LORA_NAMES:
        assert torch.count_nonzero(p0["grads"][n]) == 0
        rel, _ = metrics.relative_l2_and_cosine(p1["grads"][n].double().numpy(), o_grads[n][per:])
        assert rel <= 1e-2, f"{n}: rel-L2 {rel:.3e}"
    assert p1["out"].shape == (0, cfg.hidden) and p1["gin"].shape == (0, cfg.hidden)


def test_owner_of_slots():
    ids = torch.tensor([[0, 3], [4, 7], [-1, 8]], dtype=torch.int64)
    assert ep.owner_of(ids, 4).tolist() == [[0, 0], [1, 1], [-1, 2]]
