"""Data-parallel plumbing for the layer: one process per GPU, tokens sharded.

Every rank holds the whole frozen int4 base and the LoRA tensors and runs the
forward/backward on its own tokens; the only exchange is the sum of the six
LoRA-gradient buffers (the gradient of the layer over the union of the ranks'
tokens is the sum of the per-rank gradients, since every token contributes
independently). Process-group plumbing only: no arithmetic of the method lives
here, and nothing here touches another GPU's memory from a kernel.

Gradient window with data parallelism. The library keeps the contract test's
authoritative window per rank: the first backward of a window overwrites the
six buffers (accumulate = 0), later micro-steps add to them (accumulate = 1),
all on the rank's own tokens and without any collective. At the end of the
window, once, ``reduce_window_grads`` sums the ranks' buffers in fp32 and
rounds the sum once into bf16 (on every rank, or on one owner rank); the next
window then starts again with accumulate = 0. Reducing after every micro-step
instead would re-add the already reduced part of the window on each rank.
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


def reduce_window_grads(local: Dict[str, torch.Tensor], out: Optional[Dict[str, torch.Tensor]] = None, group=None,
                        dst: Optional[int] = None, names: Iterable[str] = GRAD_ORDER) -> Dict[str, torch.Tensor]:
    """End of a gradient window: sum the ranks' local window buffers.

    Each bf16 buffer is widened to fp32, summed over the ranks (all-reduce, or
    reduce to rank ``dst``, in a fixed order), and rounded once into ``out``
    (default: the local buffers themselves). With ``dst`` set, only that rank's
    output holds the sum (the owner of the authoritative gradients); the
    others are left untouched. Returns the output buffers.
    """
    import torch.distributed as dist

    target = local if out is None else out
    me = dist.get_rank(group) if dst is not None else None
    for n in names:
        t = local[n].to(torch.float32)
        if dst is None:
            dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
            target[n].copy_(t)
        else:
            dist.reduce(t, dst=dst, op=dist.ReduceOp.SUM, group=group)
            if me == dst:
                target[n].copy_(t)
    return target


def max_over_ranks(value: float, device: Optional[torch.device] = None, group=None) -> float:
    """The largest of the ranks' values (timings are reported as the slowest rank)."""
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
