"""Seeded synthetic inputs for the routed RAWINT4 MoE-LoRA layer.

This module is shared by the CUDA path's tests/bench and by the CPU oracle's
tests. It draws random numbers and nothing else: no decoding, no GEMM, no
SwiGLU, no gradient. Routing is generated here (top-k of seeded logits and a
softmax over the selected logits) because the router sits upstream of the
layer; the layer receives ``expert_ids`` and ``route_weights`` as inputs.

Workload shapes follow the five layer configurations the method is exercised
on (tiny oracle-scale layer, rectangular clamp case, memory-bound and
compute-bound large-MoE layers, and the largest layer). The value
distributions follow the RAWINT4 contract test
(``ktransformers/kt-kernel/test/per_commit/test_rawint4_sft_numerical.py``,
``_make_projection``): uniform codes 0..15 (drawn here as uniform bytes, i.e.
two independent uniform codes), bf16 group scales uniform in [0.01, 0.07).
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Dict, Optional

import torch

SEED = 20261001
GROUP = 32

LORA_NAMES = ("gate_lora_a", "gate_lora_b", "up_lora_a", "up_lora_b", "down_lora_a", "down_lora_b")


@dataclass(frozen=True)
class LayerConfig:
    name: str
    experts: int
    top_k: int
    hidden: int
    inter: int
    rank: int
    alpha: float
    qlen: int
    swiglu_limit: float
    routing: str  # "normal_topk" | "uniform_topk" | "zipf_topk"
    x_std: float = 1.0
    lora_std: float = 0.02
    zipf_s: float = 1.1
    weight_format: str = "rawint4"  # or "mxfp4": E2M1 codes, UE8M0 scale bytes

    @property
    def routed(self) -> int:
        return self.qlen * self.top_k

    @property
    def scaling(self) -> float:
        return self.alpha / self.rank


# The five layer configurations. Config 3 takes alpha = 2 * rank like configs
# 1, 2 and 4 (its description names no alpha).
CONFIGS = {
    0: LayerConfig("tiny", 4, 2, 256, 256, 8, 16.0, 5, 0.0, "normal_topk"),
    1: LayerConfig("rect_clamp", 8, 2, 1024, 512, 16, 32.0, 128, 2.0, "normal_topk", x_std=2.0),
    2: LayerConfig("large_membound", 256, 8, 7168, 2048, 16, 32.0, 512, 0.0, "uniform_topk"),
    3: LayerConfig("large_zipf", 256, 8, 7168, 2048, 16, 32.0, 4096, 7.0, "zipf_topk"),
    4: LayerConfig("largest", 384, 8, 7168, 2048, 32, 64.0, 8192, 0.0, "uniform_topk"),
}

# The adjacent Gemma-4 MoE layer shape (test_gemma4_moe.py,
# TestGemma4FullLayerIntegration.real_config: hidden 2816, 128 experts, top-8,
# expert intermediate 704) with a 4096-token batch and a rank-16 adapter.
GEMMA4 = LayerConfig("gemma4_layer", 128, 8, 2816, 704, 16, 32.0, 4096, 0.0, "normal_topk")


def lora_shapes(cfg: LayerConfig) -> Dict[str, tuple]:
    E, H, I, r = cfg.experts, cfg.hidden, cfg.inter, cfg.rank
    return {
        "gate_lora_a": (E, r, H),
        "gate_lora_b": (E, I, r),
        "up_lora_a": (E, r, H),
        "up_lora_b": (E, I, r),
        "down_lora_a": (E, r, I),
        "down_lora_b": (E, H, r),
    }


@dataclass
class Workload:
    """All tensors of one layer call. Host or device tensors, contiguous."""

    cfg: LayerConfig
    gate_q: torch.Tensor  # uint8 [E, I, H/2]
    gate_s: torch.Tensor  # bf16  [E, I, H/32]
    up_q: torch.Tensor  # uint8 [E, I, H/2]
    up_s: torch.Tensor  # bf16  [E, I, H/32]
    down_q: torch.Tensor  # uint8 [E, H, I/2]
    down_s: torch.Tensor  # bf16  [E, H, I/32]
    lora: Dict[str, torch.Tensor]  # bf16, shapes from lora_shapes()
    x: torch.Tensor  # bf16 [Q, H]
    expert_ids: torch.Tensor  # int64 [Q, k]
    route_weights: torch.Tensor  # fp32 [Q, k]
    grad_out: torch.Tensor  # bf16 [Q, H]

    def to(self, device) -> "Workload":
        mv = lambda t: t.to(device).contiguous()
        return Workload(
            self.cfg,
            mv(self.gate_q), mv(self.gate_s), mv(self.up_q), mv(self.up_s), mv(self.down_q), mv(self.down_s),
            {k: mv(v) for k, v in self.lora.items()},
            mv(self.x), mv(self.expert_ids), mv(self.route_weights), mv(self.grad_out),
        )


def _uniform_bytes(shape, gen, device):
    return torch.randint(0, 256, shape, generator=gen, dtype=torch.uint8, device=device)


def _scales(shape, gen, device):
    return (torch.rand(shape, generator=gen, dtype=torch.float32, device=device) * 0.06 + 0.01).to(torch.bfloat16)


# MXFP4 scale bytes: 2^(e - 127) for e in [119, 123], i.e. group scales from
# 2^-8 to 2^-4; with E2M1 magnitudes up to 6 the weights span the same range
# as the RAWINT4 ones ((code - 8) times a scale in [0.01, 0.07)).
MXFP4_SCALE_BYTES = (119, 124)


def _scale_bytes(shape, gen, device):
    return torch.randint(MXFP4_SCALE_BYTES[0], MXFP4_SCALE_BYTES[1], shape, generator=gen, dtype=torch.uint8,
                         device=device)


def _normal_bf16(shape, std, gen, device):
    return (torch.randn(shape, generator=gen, dtype=torch.float32, device=device) * std).to(torch.bfloat16)


def make_base(cfg: LayerConfig, gen: torch.Generator, device="cpu"):
    """Draw gate/up/down packed bytes and scales, expert by expert."""
    E, H, I = cfg.experts, cfg.hidden, cfg.inter
    mx = cfg.weight_format == "mxfp4"
    sdt = torch.uint8 if mx else torch.bfloat16
    draw_s = _scale_bytes if mx else _scales
    gate_q = torch.empty((E, I, H // 2), dtype=torch.uint8, device=device)
    up_q = torch.empty_like(gate_q)
    down_q = torch.empty((E, H, I // 2), dtype=torch.uint8, device=device)
    gate_s = torch.empty((E, I, H // GROUP), dtype=sdt, device=device)
    up_s = torch.empty_like(gate_s)
    down_s = torch.empty((E, H, I // GROUP), dtype=sdt, device=device)
    for e in range(E):
        gate_q[e] = _uniform_bytes((I, H // 2), gen, device)
        gate_s[e] = draw_s((I, H // GROUP), gen, device)
        up_q[e] = _uniform_bytes((I, H // 2), gen, device)
        up_s[e] = draw_s((I, H // GROUP), gen, device)
        down_q[e] = _uniform_bytes((H, I // 2), gen, device)
        down_s[e] = draw_s((H, I // GROUP), gen, device)
    return gate_q, gate_s, up_q, up_s, down_q, down_s


def make_lora(cfg: LayerConfig, gen: torch.Generator, device="cpu"):
    return {name: _normal_bf16(shape, cfg.lora_std, gen, device).contiguous() for name, shape in lora_shapes(cfg).items()}


def make_routing(cfg: LayerConfig, gen: torch.Generator, device="cpu", qlen: Optional[int] = None):
    """Top-k routing from seeded logits; weights = softmax over the k selected logits.

    normal_topk : logits ~ N(0,1)
    uniform_topk: logits ~ U(0,1) (softmax over all E renormalised over the
                  selected k equals the softmax over the selected logits)
    zipf_topk   : logits ~ N(0,1) + ln p_{pi(e)}, p proportional to rank^-s over a
                  seeded permutation pi of the experts
    """
    Q = cfg.qlen if qlen is None else qlen
    E, k = cfg.experts, cfg.top_k
    if cfg.routing == "normal_topk":
        logits = torch.randn((Q, E), generator=gen, dtype=torch.float32, device=device)
    elif cfg.routing == "uniform_topk":
        logits = torch.rand((Q, E), generator=gen, dtype=torch.float32, device=device)
    elif cfg.routing == "zipf_topk":
        pi = torch.randperm(E, generator=gen, device=device)
        ranks = torch.arange(1, E + 1, dtype=torch.float64, device=device)
        p = ranks.pow(-cfg.zipf_s)
        p = p / p.sum()
        bias = torch.empty(E, dtype=torch.float64, device=device)
        bias[pi] = torch.log(p)
        logits = torch.randn((Q, E), generator=gen, dtype=torch.float32, device=device) + bias.to(torch.float32)
    else:
        raise ValueError(f"unknown routing {cfg.routing}")
    top, ids = torch.topk(logits, k, dim=1)
    weights = torch.softmax(top, dim=1).to(torch.float32)
    return ids.to(torch.int64).contiguous(), weights.contiguous()


def make_workload(cfg: LayerConfig, device="cpu", seed: int = SEED, qlen: Optional[int] = None) -> Workload:
    """Full seeded workload. Draw order: base (per expert: gate bytes, gate
    scales, up bytes, up scales, down bytes, down scales), the six LoRA tensors,
    x, routing, grad_output. Drawing on a CUDA device uses that device's
    generator, so the values differ from a CPU draw with the same seed."""
    dev = torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(seed)
    Q = cfg.qlen if qlen is None else qlen
    base = make_base(cfg, gen, dev)
    lora = make_lora(cfg, gen, dev)
    x = _normal_bf16((Q, cfg.hidden), cfg.x_std, gen, dev).contiguous()
    ids, w = make_routing(cfg, gen, dev, Q)
    g = _normal_bf16((Q, cfg.hidden), 1.0, gen, dev).contiguous()
    return Workload(cfg, *[t.contiguous() for t in base], lora, x, ids, w, g)


def make_batch(cfg: LayerConfig, seed: int, device="cpu", qlen: Optional[int] = None):
    """A fresh (x, expert_ids, route_weights, grad_out) for an existing layer."""
    dev = torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(seed)
    Q = cfg.qlen if qlen is None else qlen
    x = _normal_bf16((Q, cfg.hidden), cfg.x_std, gen, dev).contiguous()
    ids, w = make_routing(cfg, gen, dev, Q)
    g = _normal_bf16((Q, cfg.hidden), 1.0, gen, dev).contiguous()
    return x, ids, w, g


def with_batch(wl: Workload, x, ids, w, g) -> Workload:
    return replace(wl, cfg=replace(wl.cfg, qlen=x.shape[0]), x=x, expert_ids=ids, route_weights=w, grad_out=g)


def expert_counts(expert_ids: torch.Tensor, experts: int) -> torch.Tensor:
    ids = expert_ids.reshape(-1).cpu()
    valid = ids[(ids >= 0) & (ids < experts)]
    return torch.bincount(valid, minlength=experts)


def small_config(name, experts, top_k, hidden, inter, rank, qlen, swiglu_limit=0.0, routing="normal_topk",
                 alpha=None, x_std=1.0, weight_format="rawint4") -> LayerConfig:
    return LayerConfig(name, experts, top_k, hidden, inter, rank, float(alpha if alpha is not None else 2 * rank),
                       qlen, swiglu_limit, routing, x_std=x_std, weight_format=weight_format)
