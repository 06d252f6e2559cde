#!/usr/bin/env python3
"""Throughput of one forward + backward of the routed RAWINT4 MoE-LoRA layer.

A step is one pass of the whole layer (routing permutation, gate/up, down,
combine; backward gather, down^T, gate/up^T, combine, six LoRA gradients)
over one synthetic batch. Default workload: the largest layer (E=384, top-8,
H=7168, I=2048, rank 32, alpha 64, 8192 tokens, no clamp) on one B200.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference] [--config C] [--mode infer]

Prints one JSON line (rank 0). Under torchrun each rank runs a data-parallel
replica on its own batch (weak scaling) and the six LoRA gradient buffers are
summed over ranks with NCCL after every backward.

--mode infer times the frozen-base inference forward instead (no LoRA, no
saved context; routing, gather, gate/up, down, combine) on the same workload.
"""

from __future__ import annotations

import argparse
import csv
import io
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from workloads import CONFIGS, GEMMA4, LORA_NAMES, LayerConfig, expert_counts, lora_shapes, make_batch, make_workload  # noqa: E402

METRIC = "routed tokens/s per MoE layer (fwd+bwd) and % of HBM/tensor roofline, 1×B200"
METRIC_INFER = "routed tokens/s per MoE layer (frozen-base inference forward) and % of HBM/tensor roofline, 1×B200"
UNIT = "routed tokens/s"


# ----------------------------------------------------------------- helpers

def gemm_source_hash():
    import hashlib
    d = os.path.join(ROOT, "int4_quantised_moe_b200", "csrc")
    src = b"".join(open(os.path.join(d, f), "rb").read() for f in ("gemm_tm.cu", "gemm_pair.cu", "gemm_tm_narrow.cu", "gemm_pair_narrow.cu",
                                                                  "gemm.cuh", "common.cuh", "route.cuh"))
    return hashlib.sha256(src).hexdigest()[:16]


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {"hbm_gbs": d["hbm_gbs"], "tflops": d["bf16_tflops"], "tflops_sustained": d["bf16_tflops_sustained"],
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "tflops": 1590.0, "tflops_sustained": 1400.0, "source": "fallback"}


def weight_bytes_per_value(cfg: LayerConfig) -> float:
    """Packed code plus group-scale bytes per base weight: half a byte, and a
    bf16 (RAWINT4) or UE8M0 byte (MXFP4) scale per 32 weights."""
    return 0.5 + (1.0 / 32.0 if cfg.weight_format == "mxfp4" else 2.0 / 32.0)


def algorithmic(cfg: LayerConfig, counts: torch.Tensor, infer: bool = False):
    """Algorithmic bytes and FLOPs of one fwd+bwd (weights of hit experts read
    in fwd and bwd, LoRA params read twice and grads written, x/out/dY/grad_in
    and a second read of x in bf16; saved activations not counted), or of one
    base-only forward (weights of hit experts once, x and out)."""
    Q, k, H, I, r = cfg.qlen, cfg.top_k, cfg.hidden, cfg.inter, cfg.rank
    R = int(counts.sum())
    hit = int((counts > 0).sum())
    w_e = 3 * H * I * weight_bytes_per_value(cfg)
    if infer:
        return w_e * hit + 4 * Q * H, 6 * R * H * I + 2 * R * I, R, hit
    flops = 12 * R * H * I + 18 * R * r * (H + I) + 2 * R * I
    l_e = 2 * r * (3 * H + 3 * I)
    nbytes = 2 * w_e * hit + 3 * l_e * hit + 10 * Q * H
    return nbytes, flops, R, hit


def gemm_flops(name: str, R: int, cfg: LayerConfig, lora: bool = True) -> float:
    H, I, r = cfg.hidden, cfg.inter, (cfg.rank if lora else 0)
    return {
        "gemm_gate_up": 2 * R * H * 2 * I + 2 * R * 2 * I * r,
        "gemm_down": 2 * R * I * H + 2 * R * H * r,
        "gemm_down_t": 2 * R * H * I + 2 * R * I * r,
        "gemm_gate_up_t": 2 * R * 2 * I * H + 2 * R * 2 * r * H,
    }.get(name, 0.0)


def phase_times(launches, steps: int) -> dict:
    """Kernel time per step of the forward and of the backward launches (the
    per-launch CUDA events, in issue order): a step's backward runs from its
    header_bwd launch up to the next header_fwd."""
    fwd = bwd = 0.0
    in_bwd = False
    for name, ms in launches:
        if name == "header_fwd":
            in_bwd = False
        elif name == "header_bwd":
            in_bwd = True
        if in_bwd:
            bwd += ms
        else:
            fwd += ms
    n = max(1, steps)
    return {"fwd_kernel_ms": round(fwd / n, 4), "bwd_kernel_ms": round(bwd / n, 4)}


def count_stats(counts: torch.Tensor) -> dict:
    """Realised routed rows per expert: min, median, max and empty experts."""
    c = counts.to(torch.int64)
    return {"min": int(c.min()), "median": float(c.double().median()), "max": int(c.max()), "empty": int((c == 0).sum())}


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", sel], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        rows = [r for r in csv.reader(io.StringIO(out)) if len(r) >= 9]
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for nm, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------ CPU oracle

def oracle_sample(wl, target_s: float, infer: bool = False):
    """Time the float64 oracle on whole experts of the workload until about
    `target_s` seconds of CPU work; returns (routed rows, seconds, experts).
    infer: the base-only forward (LoRA B zeroed, no backward)."""
    import numpy as np
    from oracle import moe as omoe
    from oracle import rawint4 as orq

    def bits(t):
        return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)

    ids = wl.expert_ids.cpu().numpy()
    counts = np.bincount(ids.reshape(-1)[(ids.reshape(-1) >= 0) & (ids.reshape(-1) < wl.cfg.experts)],
                         minlength=wl.cfg.experts)
    order = [int(e) for e in np.argsort(-counts, kind="stable") if counts[e] > 0]
    rows = 0
    spent = 0.0
    used = []
    mx = wl.cfg.weight_format == "mxfp4"

    def scales(t):
        # UE8M0 scale bytes as stored (MXFP4), else bf16 bit patterns
        return t.detach().cpu().contiguous().numpy() if mx else bits(t)

    for e in order:
        sel = np.nonzero((ids == e).any(axis=1))[0]
        sub_ids = np.where(ids[sel] == e, 0, -1)
        layer = omoe.Layer(
            gate_q=wl.gate_q[e:e + 1].cpu().numpy(), gate_s=scales(wl.gate_s[e:e + 1]),
            up_q=wl.up_q[e:e + 1].cpu().numpy(), up_s=scales(wl.up_s[e:e + 1]),
            down_q=wl.down_q[e:e + 1].cpu().numpy(), down_s=scales(wl.down_s[e:e + 1]),
            lora={n: (0.0 if infer and n.endswith("_b") else 1.0) * orq.bf16_bits_to_f64(bits(wl.lora[n][e:e + 1]))
                  for n in LORA_NAMES},
            alpha=wl.cfg.alpha, swiglu_limit=wl.cfg.swiglu_limit, weight_format=wl.cfg.weight_format)
        x = orq.bf16_bits_to_f64(bits(wl.x[torch.as_tensor(sel, device=wl.x.device)]))
        dy = orq.bf16_bits_to_f64(bits(wl.grad_out[torch.as_tensor(sel, device=wl.x.device)]))
        rw = wl.route_weights.cpu().numpy()[sel].astype(np.float64)
        t0 = time.perf_counter()
        _, ctx = omoe.forward(layer, x, sub_ids, rw)
        if not infer:
            omoe.backward(layer, ctx, dy)
        spent += time.perf_counter() - t0
        rows += int(counts[e])
        used.append(e)
        if spent >= target_s:
            break
    return rows, spent, used


def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


# --------------------------------------------------------------------- main

def peak_basis(clocks: dict) -> str:
    """Which measured tensor peak a kernel timed in this run is compared with:
    the burst figure when the SM clock held within 5 % of its maximum during the
    timed region, the sustained (power-capped) figure otherwise."""
    sm, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    if sm is None or mx is None or mx <= 0:
        return "burst"
    return "burst" if sm >= 0.95 * mx else "sustained"


def rooflines(kern: dict, R: int, cfg: LayerConfig, infer: bool, nbytes: float, flops: float, ms_step: float,
              clocks: dict, config_index: int):
    """Dominant-GEMM roofline and whole-step roofline against the measured peaks."""
    pk = peaks()
    basis = peak_basis(clocks)
    p_t = pk["tflops"] if basis == "burst" else pk["tflops_sustained"]
    dom = max((n for n in kern if n.startswith("gemm_")), key=lambda n: kern[n]["avg_ms"] * kern[n]["launches"])
    dom_flops = gemm_flops(dom, R, cfg, lora=not infer)
    achieved = dom_flops / (kern[dom]["avg_ms"] / 1e3) / 1e12
    traffic = None
    tfile = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tfile):
        # DRAM bytes of one launch from an ncu capture; void once the GEMM
        # sources differ from the ones the counters were taken on
        tj = json.load(open(tfile))
        if not infer and tj.get("config") == config_index and tj.get("source_sha256_16") == gemm_source_hash():
            traffic = tj.get("kernels", {}).get(dom, {}).get("dram_bytes_per_launch")
    roofline = {"bound": "tensor", "kernel": dom, "achieved": round(achieved, 2), "peak": p_t, "unit": "TFLOP/s",
                "frac": round(achieved / p_t, 4), "traffic": traffic,
                "frac_burst": round(achieved / pk["tflops"], 4),
                "frac_sustained": round(achieved / pk["tflops_sustained"], 4),
                "peak_source": f"{pk['source']} bf16 {basis} (SM clock median {clocks.get('sm_mhz')} of "
                               f"{clocks.get('sm_max_mhz')} MHz; fp16 dense rate equals bf16)"}
    t_hbm = nbytes / (pk["hbm_gbs"] * 1e9) * 1e3
    t_tc = flops / (p_t * 1e12) * 1e3
    t_roof = max(t_hbm, t_tc)
    step = {"bound": "tensor" if t_tc > t_hbm else "hbm", "t_roof_ms": round(t_roof, 4),
            "frac": round(t_roof / ms_step, 4), "peak_basis": basis,
            "frac_burst": round(max(t_hbm, flops / (pk["tflops"] * 1e12) * 1e3) / ms_step, 4),
            "frac_sustained": round(max(t_hbm, flops / (pk["tflops_sustained"] * 1e12) * 1e3) / ms_step, 4),
            "algorithmic_bytes": int(nbytes), "algorithmic_flops": int(flops),
            "achieved_hbm_gbs": round(nbytes / (ms_step / 1e3) / 1e9, 1),
            "hbm_frac": round(nbytes / (ms_step / 1e3) / 1e9 / pk["hbm_gbs"], 4),
            "routed_rows": R}
    return roofline, step


def kernel_table(launches) -> dict:
    per = {}
    for name, ms in launches:
        per.setdefault(name, []).append(ms)
    tot = max(1e-9, sum(sum(v) for v in per.values()))
    return {n: {"launches": len(v), "avg_ms": sum(v) / len(v), "share": sum(v) / tot} for n, v in per.items()}


def kernel_summary(kern: dict) -> dict:
    return {n: {"launches": v["launches"], "avg_ms": round(v["avg_ms"], 4), "share": round(v["share"], 4)}
            for n, v in sorted(kern.items(), key=lambda kv: -kv[1]["share"])}


def device_timed(step, steps: int, warmup: int, layer, B, dev, stream, barrier, max_over_ranks):
    """W warm-up steps, then K steps between CUDA events on the launching
    stream, with the library's per-launch events and the sampled SM clocks."""
    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    st = layer.status()
    if st:
        raise RuntimeError(f"device status after warm-up: {st:#x}")
    barrier()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(dev.index or 0)
    time.sleep(0.3)
    B.profile_begin(64 * steps)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for _ in range(steps):
        step()
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    launches = B.profile_end(64 * steps)
    clocks = sampler.stop()
    barrier()
    ms_total = max_over_ranks(t_start.elapsed_time(t_end))
    return ms_total / steps, launches, clocks


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", type=int, default=4)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end pass")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="skip the extra measurements of the memory-bound and skewed layers")
    ap.add_argument("--experts", type=int, default=None, help="override the expert count (profiling cases)")
    ap.add_argument("--qlen", type=int, default=None, help="override the token count (profiling cases)")
    ap.add_argument("--format", default="rawint4", choices=["rawint4", "mxfp4"],
                    help="base weight format of the layer (the sibling MXFP4 base: E2M1 codes, UE8M0 scales)")
    ap.add_argument("--shape", default=None, choices=["gemma4"],
                    help="gemma4: the Gemma-4 MoE layer shape (E=128, top-8, H=2816, I=704) instead of --config")
    ap.add_argument("--mode", default="train", choices=["train", "infer"],
                    help="train: fwd+bwd step (default); infer: frozen-base inference forward")
    args = ap.parse_args()
    infer = args.mode == "infer"
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    import dataclasses
    cfg = GEMMA4 if args.shape == "gemma4" else CONFIGS[args.config]
    if args.experts is not None or args.qlen is not None:
        cfg = dataclasses.replace(cfg, name=cfg.name + "_override", experts=args.experts or cfg.experts,
                                  qlen=args.qlen or cfg.qlen)
    if args.format != cfg.weight_format:
        cfg = dataclasses.replace(cfg, name=cfg.name + "_" + args.format, weight_format=args.format)
    # the ncu traffic counters were taken on the default workload's kernels
    traffic_key = args.config if (args.shape is None and args.format == "rawint4") else None
    workload_name = describe(cfg)

    if args.impl == "reference":
        if rank != 0:
            return 0
        return run_reference(args, cfg, workload_name)

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist

    from int4_quantised_moe_b200 import binding as B
    from int4_quantised_moe_b200 import dp

    def barrier():
        if pg is not None:
            pg.barrier()

    def max_over_ranks(v: float) -> float:
        return dp.max_over_ranks(v, device=dev)

    # layer (same on every rank) and this rank's batch
    wl = make_workload(cfg, device=dev)
    if rank > 0:
        x, ids, w, g = make_batch(cfg, seed=dp.rank_batch_seed(rank), device=dev)
        wl.x, wl.expert_ids, wl.route_weights, wl.grad_out = x, ids, w, g
    counts = expert_counts(wl.expert_ids, cfg.experts)
    nbytes, flops, R, hit = algorithmic(cfg, counts, infer)
    layer = B.Layer.create(cfg.experts, cfg.top_k, cfg.hidden, cfg.inter, cfg.rank, cfg.alpha, cfg.swiglu_limit,
                           cfg.qlen, wl.gate_q, wl.gate_s, wl.up_q, wl.up_s, wl.down_q, wl.down_s, wl.lora,
                           weight_format=cfg.weight_format)
    grads = {n: torch.zeros(s, dtype=torch.bfloat16, device=dev) for n, s in lora_shapes(cfg).items()}
    out = torch.empty_like(wl.x)
    gin = torch.empty_like(wl.x)
    groute = torch.empty(wl.expert_ids.shape, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        if infer:
            layer.forward(wl.expert_ids, wl.route_weights, wl.x, out=out, save_for_backward=False, use_lora=False)
            return
        layer.forward(wl.expert_ids, wl.route_weights, wl.x, out=out, save_for_backward=True)
        layer.backward(wl.grad_out, grads, accumulate=False, grad_scale=1.0, grad_in=gin, grad_route=groute)
        if pg is not None:
            dp.reduce_window_grads(grads)  # one-step window: reduce at its end

    # ---- device-timed region (inputs resident in HBM) with per-launch events
    ms_step, launches, clocks = device_timed(step, args.steps, args.warmup, layer, B, dev, stream, barrier,
                                             max_over_ranks)
    value = cfg.qlen * cfg.top_k * world / (ms_step / 1e3)
    kern = kernel_table(launches)
    roofline, step_roofline = rooflines(kern, R, cfg, infer, nbytes, flops, ms_step, clocks, traffic_key)
    step_roofline["experts_hit"] = hit

    # ---- end to end through the public API from pinned host buffers. Steps
    # are pipelined as a host loop would run them: the inputs of step i+1 go
    # up and the outputs of step i-1 come down on two copy streams while step
    # i's kernels run; device inputs and outputs are double-buffered, and
    # events order each buffer's upload, use and download. Every step still
    # copies its whole input from pinned host memory and its whole result
    # back, all inside the timed region (from the first upload to the last
    # download).
    e2e = None
    if not args.no_e2e:
        h_x = wl.x.cpu().pin_memory()
        h_ids = wl.expert_ids.cpu().pin_memory()
        h_w = wl.route_weights.cpu().pin_memory()
        h_g = wl.grad_out.cpu().pin_memory()
        h_out = [torch.empty_like(h_x).pin_memory() for _ in range(2)]
        h_gin = [torch.empty_like(h_x).pin_memory() for _ in range(2)]
        h_gr = [torch.empty(groute.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
        d_in = [(torch.empty_like(wl.x), torch.empty_like(wl.expert_ids), torch.empty_like(wl.route_weights),
                 torch.empty_like(wl.grad_out)) for _ in range(2)]
        d_res = [(torch.empty_like(out), torch.empty_like(gin), torch.empty_like(groute)) for _ in range(2)]
        up = torch.cuda.Stream(device=dev)
        down = torch.cuda.Stream(device=dev)
        ev = lambda: torch.cuda.Event()  # noqa: E731
        uploaded = [ev(), ev()]    # inputs of buffer b on the device
        computed = [ev(), ev()]    # kernels of buffer b done (inputs free, results ready)
        downloaded = [ev(), ev()]  # results of buffer b on the host (result buffers free)
        used = [False, False]

        def e2e_step(i):
            b = i & 1
            d_x, d_ids, d_w, d_g = d_in[b]
            r_out, r_gin, r_gr = d_res[b]
            with torch.cuda.stream(up):
                if used[b]:
                    up.wait_event(computed[b])
                d_x.copy_(h_x, non_blocking=True)
                d_ids.copy_(h_ids, non_blocking=True)
                d_w.copy_(h_w, non_blocking=True)
                if not infer:
                    d_g.copy_(h_g, non_blocking=True)
                uploaded[b].record(up)
            stream.wait_event(uploaded[b])
            if used[b]:
                stream.wait_event(downloaded[b])
            if infer:
                layer.forward(d_ids, d_w, d_x, out=r_out, save_for_backward=False, use_lora=False)
            else:
                layer.forward(d_ids, d_w, d_x, out=r_out, save_for_backward=True)
                layer.backward(d_g, grads, accumulate=False, grad_scale=1.0, grad_in=r_gin, grad_route=r_gr)
                if pg is not None:
                    dp.reduce_window_grads(grads)  # one-step window: reduce at its end
            computed[b].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(computed[b])
                h_out[b].copy_(r_out, non_blocking=True)
                if not infer:
                    h_gin[b].copy_(r_gin, non_blocking=True)
                    h_gr[b].copy_(r_gr, non_blocking=True)
                downloaded[b].record(down)
            used[b] = True

        e2e_step(0)
        e2e_step(1)
        torch.cuda.synchronize(dev)
        barrier()
        e_start = torch.cuda.Event(enable_timing=True)
        e_end = torch.cuda.Event(enable_timing=True)
        e_start.record(stream)
        up.wait_event(e_start)
        for i in range(args.steps):
            e2e_step(i)
        for b in range(2):
            stream.wait_event(downloaded[b])
        e_end.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        e_ms = max_over_ranks(e_start.elapsed_time(e_end)) / args.steps
        h2d = sum(t.numel() * t.element_size() for t in ((h_x, h_ids, h_w) if infer else (h_x, h_ids, h_w, h_g)))
        d2h = sum(t.numel() * t.element_size() for t in ((h_out[0],) if infer else (h_out[0], h_gin[0], h_gr[0])))
        e2e = {"value": round(cfg.qlen * cfg.top_k * world / (e_ms / 1e3), 1), "unit": UNIT,
               "ms_per_step": round(e_ms, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "pipelined": "uploads of step i+1 and downloads of step i-1 overlap step i on two copy streams"}

    st = layer.status()
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rows, secs, used = oracle_sample(wl, args.cpu_seconds, infer)
        what = "base-only fwd" if infer else "fwd+bwd"
        cpu = {"value": round(rows / secs, 2), "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
               "sample": f"float64 NumPy oracle {what} of {len(used)} whole expert(s) of this workload "
                         f"({rows} routed rows, {secs:.1f} s)"}
    cfg_obj = arm_config(cfg, world, workload_name, R, hit, counts)
    del layer, wl, grads, out, gin, groute
    torch.cuda.empty_cache()

    # ---- the memory-bound and the skewed layer, and the base-only forward of
    # the memory-bound one (one GPU, default workload only)
    others = None
    if (world == 1 and args.config == 4 and args.shape is None and args.format == "rawint4" and args.experts is None
            and args.qlen is None and not args.no_other_configs):
        others = [other_config(c, m, B, dev, stream, key) for c, m, key in (
            (CONFIGS[2], "train", 2), (CONFIGS[3], "train", 3), (CONFIGS[2], "infer", 2),
            (dataclasses.replace(CONFIGS[4], name="largest_mxfp4", weight_format="mxfp4"), "train", None),
            (GEMMA4, "train", None))]

    if rank == 0:
        line = {
            "metric": METRIC_INFER if infer else METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic", "config": cfg_obj,
            "roofline": roofline, "step_roofline": step_roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": len(launches), "phases": phase_times(launches, args.steps), "clocks": clocks,
            "device_status": st, "kernels": kernel_summary(kern), "other_configs": others,
        }
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()
    return 0


def describe(cfg: LayerConfig) -> str:
    return (f"{cfg.name}: E={cfg.experts} top_k={cfg.top_k} H={cfg.hidden} I={cfg.inter} r={cfg.rank} "
            f"alpha={cfg.alpha:g} qlen={cfg.qlen} swiglu_limit={cfg.swiglu_limit:g} routing={cfg.routing}")


def other_config(cfg: LayerConfig, mode: str, B, dev, stream, traffic_key, steps: int = 10, warmup: int = 3) -> dict:
    """Device-timed steps of another workload (no e2e pass, no CPU baseline)."""
    infer = mode == "infer"
    wl = make_workload(cfg, device=dev)
    counts = expert_counts(wl.expert_ids, cfg.experts)
    nbytes, flops, R, hit = algorithmic(cfg, counts, infer)
    layer = B.Layer.create(cfg.experts, cfg.top_k, cfg.hidden, cfg.inter, cfg.rank, cfg.alpha, cfg.swiglu_limit,
                           cfg.qlen, wl.gate_q, wl.gate_s, wl.up_q, wl.up_s, wl.down_q, wl.down_s, wl.lora,
                           weight_format=cfg.weight_format)
    grads = {n: torch.zeros(s, dtype=torch.bfloat16, device=dev) for n, s in lora_shapes(cfg).items()}
    out = torch.empty_like(wl.x)
    gin = torch.empty_like(wl.x)
    groute = torch.empty(wl.expert_ids.shape, dtype=torch.float32, device=dev)

    def step():
        if infer:
            layer.forward(wl.expert_ids, wl.route_weights, wl.x, out=out, save_for_backward=False, use_lora=False)
            return
        layer.forward(wl.expert_ids, wl.route_weights, wl.x, out=out, save_for_backward=True)
        layer.backward(wl.grad_out, grads, accumulate=False, grad_scale=1.0, grad_in=gin, grad_route=groute)

    ms_step, launches, clocks = device_timed(step, steps, warmup, layer, B, dev, stream, lambda: None, lambda v: v)
    kern = kernel_table(launches)
    roofline, step_roofline = rooflines(kern, R, cfg, infer, nbytes, flops, ms_step, clocks, traffic_key)
    res = {"workload": describe(cfg), "weight_format": cfg.weight_format, "mode": mode, "steps": steps, "warmup": warmup,
           "ms_per_step": round(ms_step, 4), "value": round(cfg.qlen * cfg.top_k / (ms_step / 1e3), 1), "unit": UNIT,
           "expert_rows": count_stats(counts), "experts_hit": hit, "step_roofline": step_roofline,
           "roofline": roofline, "clocks": clocks, "device_status": layer.status(), "kernels": kernel_summary(kern)}
    del layer, wl, grads, out, gin, groute
    torch.cuda.empty_cache()
    return res


def arm_config(cfg: LayerConfig, world: int, workload_name: str, R: int, hit: int, counts: torch.Tensor) -> dict:
    """The `config` object of the JSON line, shared by both arms."""
    return {"workload": workload_name, "parallelism": f"dp{world}" if world > 1 else "single",
            "global_batch_tokens": cfg.qlen * world, "routed_rows_per_gpu": R,
            "expert_rows": count_stats(counts),
            "l2": "inputs larger than L2: every step streams all hit experts' packed weights "
                  f"({2 * hit * 3 * cfg.hidden * cfg.inter * weight_bytes_per_value(cfg) / 1e9:.1f} GB)",
            "weight_format": cfg.weight_format}


def run_reference(args, cfg: LayerConfig, workload_name: str) -> int:
    """The oracle as it stands on the host cores; each step a bounded sample."""
    wl = make_workload(cfg, device="cuda" if torch.cuda.is_available() else "cpu")
    infer = args.mode == "infer"
    per_step = max(1.0, min(args.cpu_seconds, 60.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(wl, per_step, infer)
    rows_t, secs_t = 0, 0.0
    for _ in range(args.steps):
        rows, secs, used = oracle_sample(wl, per_step, infer)
        rows_t += rows
        secs_t += secs
    value = rows_t / secs_t
    world = int(os.environ.get("WORLD_SIZE", "1"))
    counts = expert_counts(wl.expert_ids, cfg.experts)
    _, _, R, hit = algorithmic(cfg, counts, infer)
    line = {
        "impl": "reference", "metric": METRIC_INFER if infer else METRIC, "value": round(value, 2), "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * secs_t / args.steps, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": arm_config(cfg, world, workload_name, R, hit, counts),
        "cpu_baseline": {"value": round(value, 2), "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                         "sample": f"each step: float64 NumPy oracle {'base-only fwd' if infer else 'fwd+bwd'} of whole "
                                   f"experts for about {per_step:.1f} s"},
        "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
