"""Where the clamped workload's grad_in error comes from (CPU, oracle only).

Config 3 clamps at L = 7 with Zipf routing. On the B200 its sampled grad_in has
rel-L2 4.7e-3 against the oracle, while every unclamped output sits at the
bf16 rounding floor of about 1.7e-3. This script takes the same four sampled
tokens as ``report_parity`` and reports two things:

* the oracle's float64 pre-activations G, U that lie closest to the clamp
  bounds (the gate bound +L, the up bounds -L and +L);
* how much grad_in changes when the mask decision of each such element flips
  (the element is pushed just across its bound).

A kernel accumulates G and U in fp32 on the tensor cores, so it can land on
the other side of a bound for an element whose exact value is within its
accumulation error of it. Each flip moves a whole row of W^T dG into that
token's dX.

    python -m tests.report_clamp_margin
"""

from __future__ import annotations

import copy

import numpy as np
import torch

from oracle import metrics
from oracle import moe as omoe
from oracle import rawint4 as orq
from tests.test_gpu_fullsize import bits, sub_layer
from workloads import CONFIGS, make_workload


def main(cfg_id: int = 3, show: int = 12) -> None:
    cfg = CONFIGS[cfg_id]
    L = cfg.swiglu_limit
    wl = make_workload(cfg)
    Q = cfg.qlen
    toks = sorted({0, Q // 3, Q // 2, Q - 1})
    ids = wl.expert_ids.numpy()
    experts = sorted({int(e) for e in ids[toks].reshape(-1)})
    remap = {e: i for i, e in enumerate(experts)}
    layer = sub_layer(wl, experts)
    t = torch.as_tensor(toks)
    x = orq.bf16_bits_to_f64(bits(wl.x.index_select(0, t)))
    dy = orq.bf16_bits_to_f64(bits(wl.grad_out.index_select(0, t)))
    rw = wl.route_weights.numpy()[toks].astype(np.float64)
    _, ctx = omoe.forward(layer, x, np.vectorize(remap.get)(ids[toks]), rw)
    gin0, _, _ = omoe.backward(layer, ctx, dy)

    near = []  # (distance, expert, token, "G"/"U", feature, value)
    for e, ec in ctx.experts.items():
        for j, tok in enumerate(ec.tokens):
            dg = np.abs(ec.G[j] - L)
            du = np.minimum(np.abs(ec.U[j] - L), np.abs(ec.U[j] + L))
            for i in np.argsort(dg)[:3]:
                near.append((float(dg[i]), e, int(tok), "G", int(i), float(ec.G[j, i])))
            for i in np.argsort(du)[:3]:
                near.append((float(du[i]), e, int(tok), "U", int(i), float(ec.U[j, i])))
    near.sort()

    def flip(entry):
        _, e, tok, which, i, v = entry
        c2 = copy.deepcopy(ctx)
        ec = c2.experts[e]
        j = int(np.nonzero(ec.tokens == tok)[0][0])
        arr = ec.G if which == "G" else ec.U
        bound = L if v > 0 else -L
        inside = abs(v) < L
        arr[j, i] = bound + (1e-6 if inside else -1e-6) * np.sign(bound)
        return c2

    print(f"config {cfg_id}: L = {L}, sampled tokens {toks}, {sum(ec.G.size for ec in ctx.experts.values())} "
          "G values and as many U values")
    print("distance to bound | value | flip changes grad_in by (rel-L2)")
    for entry in near[:show]:
        gin1, _, _ = omoe.backward(layer, flip(entry), dy)
        rel, _ = metrics.relative_l2_and_cosine(gin1, gin0)
        d, e, tok, which, i, v = entry
        print(f"  {d:.2e} | expert {experts[e]} token {toks[tok]} {which}[{i}] = {v:.9f} | {rel:.3e}")


if __name__ == "__main__":
    main()
