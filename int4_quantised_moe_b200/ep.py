"""Expert parallelism for the routed RAWINT4 MoE-LoRA layer: one process per
GPU, each holding the base weights and LoRA adapters of experts
[rank * E / G, (rank + 1) * E / G) only, so the weight bytes per GPU drop by G.

A step moves routed slots, not tokens. Forward on each process, for its own
tokens:

1. the owning process of every slot (expert // (E / G)) is found and the
   slots are grouped by it, stably (``rawint4_moe_permute`` with the process
   index as the "expert"): ``perm``, ``inv`` and the per-process counts;
2. the counts are exchanged (an all-to-all of G integers), then the token
   row of every leaving slot (``rawint4_moe_dispatch_rows``), its local
   expert index and its route weight (all-to-all over NCCL);
3. each process runs its local layer on the slots it received, as a layer
   of E / G experts with top_k = 1 (one received slot per row): row n gives
   w_n * expert(x_n), with the LoRA, clamp and saved context of the method;
4. the result rows go back (all-to-all) and ``rawint4_moe_combine_slots``
   sums each token's slots in slot order (fp32 sums, one bf16 rounding).

Backward replays the same moves: grad_out rows go out with the plan of the
forward, the local layer's backward yields each slot's grad_in row and
dRoute value, which come back and are combined (``combine_slots``) or put in
slot order (``rawint4_moe_gather_slots``). The LoRA gradients of an expert
stay on the process that owns it: nothing is reduced.

Against the single-process layer the only numerical difference is that each
slot's result (and grad_in contribution) is rounded to bf16 once before the
slots of a token are summed, where the single-process layer sums fp32
partials; the route gradients are unchanged.

The host needs the per-process counts to size the exchanges, so a forward and
a backward each read G integers back from the device once. Every process
must call forward and backward the same number of times, in the same order
(they are collective).
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Dict, Optional

import torch

from . import binding as B


def owner_of(expert_ids: torch.Tensor, experts_per_rank: int) -> torch.Tensor:
    """Owning process of every slot: expert // (E / G); an id outside [0, E)
    maps outside [0, G) (negative ids stay negative)."""
    return torch.div(expert_ids, experts_per_rank, rounding_mode="floor")


@dataclass
class KernelOps:
    """The four row-movement calls of a step (the library's by default)."""

    permute: Callable  # (owner ids int64 [Q, k], G, offsets, perm, inv) -> None
    dispatch_rows: Callable  # (src [Q, H] bf16, perm, n, top_k, dst [n, H]) -> None
    combine_slots: Callable  # (src [n, H] bf16, inv, qlen, top_k, out [Q, H]) -> None
    gather_slots: Callable  # (src [n] fp32, inv, out [Q * k]) -> None


def library_ops() -> KernelOps:
    return KernelOps(permute=B.rawint4_moe_permute, dispatch_rows=B.rawint4_moe_dispatch_rows,
                     combine_slots=B.rawint4_moe_combine_slots, gather_slots=B.rawint4_moe_gather_slots)


def _exchange(dist, tensor: torch.Tensor, send_counts, recv_counts) -> torch.Tensor:
    """All-to-all of the rows of `tensor` (grouped by destination, send_counts
    rows each); bf16 rows (an even width) travel as int32 pairs of bit
    patterns, which every backend carries."""
    bf16 = tensor.dtype == torch.bfloat16
    src = tensor.contiguous()
    if bf16:
        src = (src.view(torch.int32) if src.numel() else
               torch.empty(tuple(src.shape[:-1]) + (src.shape[-1] // 2,), dtype=torch.int32, device=src.device))
    out = torch.empty((int(sum(recv_counts)),) + tuple(src.shape[1:]), dtype=src.dtype, device=tensor.device)
    dist.all_to_all_single(out, src, output_split_sizes=list(recv_counts), input_split_sizes=list(send_counts))
    return out.view(torch.bfloat16) if bf16 else out


class ExpertParallelLayer:
    """The layer with its experts split over the processes of `dist` (an
    initialised torch.distributed module or group wrapper exposing
    get_world_size, get_rank and all_to_all_single).

    `local_layer`: this process's layer over its E / G experts with top_k = 1
    and max_tokens = `capacity` (the most slots it may receive in one step),
    e.g. ``binding.Layer.create(E // G, 1, H, I, r, alpha, L, capacity, ...)``
    on this process's slices of the base and LoRA tensors."""

    def __init__(self, dist, experts: int, top_k: int, local_layer, capacity: int, ops: Optional[KernelOps] = None):
        self.dist = dist
        self.world = dist.get_world_size()
        self.rank = dist.get_rank()
        if experts % self.world:
            raise ValueError(f"experts ({experts}) must split evenly over {self.world} processes")
        self.experts = experts
        self.per_rank = experts // self.world
        self.top_k = top_k
        self.local = local_layer
        self.capacity = capacity
        self.ops = ops or library_ops()
        self._ctx = None

    # ------------------------------------------------------------------ plan
    def _plan(self, expert_ids: torch.Tensor):
        q, k = expert_ids.shape
        dev = expert_ids.device
        owner = owner_of(expert_ids, self.per_rank).contiguous()
        offsets = torch.empty(self.world + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(max(q * k, 1), dtype=torch.int32, device=dev)
        inv = torch.empty(max(q * k, 1), dtype=torch.int32, device=dev)
        self.ops.permute(owner, self.world, offsets, perm, inv)
        send_counts = (offsets[1:] - offsets[:-1]).to(torch.int64)
        recv_counts = torch.empty_like(send_counts)
        self.dist.all_to_all_single(recv_counts, send_counts)
        send = send_counts.tolist()
        recv = recv_counts.tolist()
        return perm, inv, send, recv

    # --------------------------------------------------------------- forward
    def forward(self, expert_ids: torch.Tensor, route_weights: torch.Tensor, x: torch.Tensor,
                save_for_backward: bool = True) -> torch.Tensor:
        q, k = expert_ids.shape
        if k != self.top_k:
            raise ValueError(f"expert_ids has {k} slots per token, the layer top_k is {self.top_k}")
        h = x.shape[1]
        perm, inv, send, recv = self._plan(expert_ids)
        n_send, n_recv = int(sum(send)), int(sum(recv))
        if n_recv > self.capacity:
            raise RuntimeError(f"process {self.rank} receives {n_recv} slots, its capacity is {self.capacity}")
        x_send = torch.empty((n_send, h), dtype=torch.bfloat16, device=x.device)
        if n_send:
            self.ops.dispatch_rows(x, perm, n_send, k, x_send)
        slots = perm[:n_send].to(torch.int64)
        local_ids = torch.remainder(expert_ids.reshape(-1)[slots], self.per_rank)
        weights = route_weights.reshape(-1)[slots].contiguous()
        x_recv = _exchange(self.dist, x_send, send, recv)
        ids_recv = _exchange(self.dist, local_ids.contiguous(), send, recv)
        w_recv = _exchange(self.dist, weights, send, recv)
        y_recv = self.local.forward(ids_recv.view(-1, 1), w_recv.view(-1, 1), x_recv,
                                    save_for_backward=save_for_backward)
        y_send = _exchange(self.dist, y_recv, recv, send)
        out = torch.empty((q, h), dtype=torch.bfloat16, device=x.device)
        self.ops.combine_slots(y_send, inv, q, k, out)
        self._ctx = (perm, inv, send, recv, q, k, h) if save_for_backward else None
        return out

    # -------------------------------------------------------------- backward
    def backward(self, grad_out: torch.Tensor, grads: Dict[str, torch.Tensor], accumulate: bool = False,
                 grad_scale: float = 1.0, grad_in: Optional[torch.Tensor] = None,
                 grad_route: Optional[torch.Tensor] = None) -> torch.Tensor:
        """`grads`: this process's LoRA gradient buffers (its E / G experts),
        with the gradient-window semantics of the single-process layer."""
        if self._ctx is None:
            raise RuntimeError("backward without a saved forward")
        perm, inv, send, recv, q, k, h = self._ctx
        self._ctx = None
        n_send, n_recv = int(sum(send)), int(sum(recv))
        g_send = torch.empty((n_send, h), dtype=torch.bfloat16, device=grad_out.device)
        if n_send:
            self.ops.dispatch_rows(grad_out, perm, n_send, k, g_send)
        g_recv = _exchange(self.dist, g_send, send, recv)
        gin_recv = torch.empty((n_recv, h), dtype=torch.bfloat16, device=grad_out.device)
        gr_recv = torch.empty((n_recv, 1), dtype=torch.float32, device=grad_out.device)
        self.local.backward(g_recv, grads, accumulate=accumulate, grad_scale=grad_scale, grad_in=gin_recv,
                            grad_route=gr_recv)
        gin_send = _exchange(self.dist, gin_recv, recv, send)
        gr_send = _exchange(self.dist, gr_recv.view(-1), recv, send)
        if grad_in is None:
            grad_in = torch.empty((q, h), dtype=torch.bfloat16, device=grad_out.device)
        self.ops.combine_slots(gin_send, inv, q, k, grad_in)
        if grad_route is not None:
            self.ops.gather_slots(gr_send, inv, grad_route.view(-1))
        return grad_in
