"""Data-parallel plumbing for the layer: one process per GPU, tokens sharded.

Every rank holds the whole frozen int4 base and the LoRA tensors and runs the
forward/backward on its own tokens; the only exchange is the sum of the six
LoRA-gradient buffers after each backward (the gradient of the layer over the
union of the ranks' tokens is the sum of the per-rank gradients, since every
token contributes independently). Process-group plumbing only: no arithmetic of
the method lives here, and nothing here touches another GPU's memory from a
kernel.
"""

from __future__ import annotations

from typing import Dict, Iterable, Optional

import torch

# fixed order of the six buffers: every rank issues the same collectives in the same order
GRAD_ORDER = ("gate_lora_a", "gate_lora_b", "up_lora_a", "up_lora_b", "down_lora_a", "down_lora_b")

BATCH_SEED = 20261001
RANK_SEED_STRIDE = 7919


def rank_batch_seed(rank: int, base_seed: int = BATCH_SEED) -> int:
    """Seed of the token batch of `rank` (rank 0 keeps the layer's own batch)."""
    return base_seed + RANK_SEED_STRIDE * rank


def shard_tokens(qlen: int, rank: int, world: int) -> slice:
    """Contiguous share of `qlen` tokens for `rank` (sizes differ by at most one)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside world of {world}")
    base, extra = divmod(qlen, world)
    start = rank * base + min(rank, extra)
    return slice(start, start + base + (1 if rank < extra else 0))


def allreduce_lora_grads(grads: Dict[str, torch.Tensor], group=None, names: Iterable[str] = GRAD_ORDER) -> None:
    """Sum each LoRA-gradient buffer over the ranks, in place, in a fixed order."""
    import torch.distributed as dist

    for n in names:
        dist.all_reduce(grads[n], op=dist.ReduceOp.SUM, group=group)


def max_over_ranks(value: float, device: Optional[torch.device] = None, group=None) -> float:
    """The largest of the ranks' values (timings are reported as the slowest rank)."""
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
