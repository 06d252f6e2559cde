"""Data-parallel host logic on CPU: two gloo ranks, world size 2.

Each rank computes the oracle LoRA gradients of its own token batch (the
batch seed of ``dp.rank_batch_seed``), rounds them into bf16 buffers as the
library's gradient window stores them, and sums the buffers with
``dp.allreduce_lora_grads``. The result must equal the oracle gradients of the
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
        # gloo sums in the buffer's dtype; widen so the test isolates the sharding logic
        g32 = {n: t.float() for n, t in grads.items()}
        dp.allreduce_lora_grads(g32)
        slowest = dp.max_over_ranks(float(rank + 1))
        if rank == 0:
            torch.save({"grads": g32, "slowest": slowest}, os.path.join(out_dir, "reduced.pt"))
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
