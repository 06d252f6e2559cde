"""Data-parallel host logic on CPU: two gloo ranks, world size 2.

Each rank computes the oracle LoRA gradients of its own token batch (the
batch seed of ``dp.rank_batch_seed``), rounds them into bf16 buffers as the
library's gradient window stores them, and sums the buffers with
``dp.reduce_window_grads`` (fp32 sum, one rounding). The result must equal the oracle gradients of the
union of both batches (one layer, 2 Q tokens) within the LoRA-gradient
tolerance: the gradient of the layer over several token batches is the sum of
the per-batch gradients, which is what makes token sharding with one
all-reduce exact up to the bf16 rounding of the buffers.
"""

from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from int4_quantised_moe_b200 import dp
from oracle import metrics
from oracle import moe as omoe
from tests._util import f64, oracle_layer
from workloads import CONFIGS, LORA_NAMES, make_batch, make_workload

TOL = 1e-2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_grads(rank: int):
    cfg = CONFIGS[1]
    wl = make_workload(cfg, device="cpu")
    x, ids, w, g = make_batch(cfg, seed=dp.rank_batch_seed(rank))
    layer = oracle_layer(wl)
    _, ctx = omoe.forward(layer, f64(x), ids.numpy(), f64(w))
    _, _, grads = omoe.backward(layer, ctx, f64(g))
    return {n: torch.from_numpy(np.ascontiguousarray(grads[n])).to(torch.bfloat16) for n in LORA_NAMES}


def _worker(rank: int, world: int, port: int, out_dir: str) -> None:
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        grads = _rank_grads(rank)
        # the exact bf16 buffers the benchmark reduces after each one-step window
        dp.reduce_window_grads(grads)
        slowest = dp.max_over_ranks(float(rank + 1))
        if rank == 0:
            torch.save({"grads": grads, "slowest": slowest}, os.path.join(out_dir, "reduced.pt"))
    finally:
        dist.destroy_process_group()


def test_shard_tokens_cover():
    for q in (0, 1, 5, 17, 8192):
        for world in (1, 2, 3, 8):
            parts = [dp.shard_tokens(q, r, world) for r in range(world)]
            assert parts[0].start == 0 and parts[-1].stop == q
            for a, b in zip(parts, parts[1:]):
                assert a.stop == b.start
            sizes = [p.stop - p.start for p in parts]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        dp.shard_tokens(10, 2, 2)


def test_allreduce_matches_union_batch(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    got = torch.load(os.path.join(tmp_path, "reduced.pt"))
    assert got["slowest"] == float(world)

    # oracle over the union of both ranks' batches
    cfg = CONFIGS[1]
    wl = make_workload(cfg, device="cpu")
    batches = [make_batch(cfg, seed=dp.rank_batch_seed(r)) for r in range(world)]
    x = torch.cat([b[0] for b in batches])
    ids = torch.cat([b[1] for b in batches])
    w = torch.cat([b[2] for b in batches])
    g = torch.cat([b[3] for b in batches])
    layer = oracle_layer(wl)
    _, ctx = omoe.forward(layer, f64(x), ids.numpy(), f64(w))
    _, _, ref = omoe.backward(layer, ctx, f64(g))
    for n in LORA_NAMES:
        r, c = metrics.relative_l2_and_cosine(got["grads"][n].double().numpy(), ref[n])
        assert r <= TOL and c >= 0.9999, (n, r, c)


def _window_worker(rank: int, world: int, port: int, out_dir: str) -> None:
    """Two micro-steps on this rank's own batches, accumulated in bf16 as the
    library's window stores them (overwrite, then add), then one window-end
    reduction of the exact bf16 buffers."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = CONFIGS[1]
        wl = make_workload(cfg, device="cpu")
        layer = oracle_layer(wl)
        scale = 0.5
        buf = None
        for micro in range(2):
            x, ids, w, g = make_batch(cfg, seed=dp.rank_batch_seed(rank) + 101 * micro)
            _, ctx = omoe.forward(layer, f64(x), ids.numpy(), f64(w))
            _, _, gr = omoe.backward(layer, ctx, f64(g))
            prev = None if buf is None else {n: buf[n].double().numpy() for n in LORA_NAMES}
            win = omoe.grad_window(prev, gr, accumulate=micro > 0, grad_scale=scale)
            buf = {n: torch.from_numpy(np.ascontiguousarray(win[n])).to(torch.bfloat16) for n in LORA_NAMES}
        owner = {n: torch.full_like(t, 7.0) for n, t in buf.items()}
        dp.reduce_window_grads(buf, out=owner, dst=0)  # owner rank only
        dp.reduce_window_grads(buf)  # every rank, in place
        if rank == 0:
            torch.save({"all": buf, "owner": owner}, os.path.join(out_dir, "window.pt"))
        else:
            assert all(torch.all(owner[n] == 7.0) for n in LORA_NAMES)  # non-owners untouched
    finally:
        dist.destroy_process_group()


def test_window_reduction_matches_union_of_micro_batches(tmp_path):
    """World 2 x 2 accumulated micro-steps, reduced once at the window end in
    fp32 from the exact bf16 buffers: equals the oracle gradients of all four
    batches together times grad_scale (LoRA-gradient tolerance)."""
    world = 2
    mp.start_processes(_window_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    got = torch.load(os.path.join(tmp_path, "window.pt"))
    cfg = CONFIGS[1]
    wl = make_workload(cfg, device="cpu")
    batches = [make_batch(cfg, seed=dp.rank_batch_seed(r) + 101 * m) for r in range(world) for m in range(2)]
    x = torch.cat([b[0] for b in batches])
    ids = torch.cat([b[1] for b in batches])
    w = torch.cat([b[2] for b in batches])
    g = torch.cat([b[3] for b in batches])
    layer = oracle_layer(wl)
    _, ctx = omoe.forward(layer, f64(x), ids.numpy(), f64(w))
    _, _, ref = omoe.backward(layer, ctx, f64(g))
    for key in ("all", "owner"):
        for n in LORA_NAMES:
            r, c = metrics.relative_l2_and_cosine(got[key][n].double().numpy(), 0.5 * ref[n])
            assert r <= TOL and c >= 0.9999, (key, n, r, c)
