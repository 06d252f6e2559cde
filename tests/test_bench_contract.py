"""The reference arm of bench.py (the float64 oracle on the host cores) prints
one JSON line with the keys of the benchmark contract. CPU only: small
workload, one short timed step."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*extra):
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "0", "--steps", "1",
           "--warmup", "3", "--cpu-seconds", "0.2", *extra]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout
    return json.loads(lines[0])


@pytest.mark.parametrize("mode", ["train", "infer"])
def test_reference_arm_line(mode):
    d = _run("--mode", mode)
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["value"] > 0 and d["unit"] == "routed tokens/s"
    assert d["steps"] == 1 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["vs_baseline"] is None
    assert ("inference" in d["metric"]) == (mode == "infer")
    assert d["config"]["workload"].startswith("tiny:")
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_reports_expert_rows():
    d = _run()
    er = d["config"]["expert_rows"]
    assert set(er) == {"min", "median", "max", "empty"}
    assert 0 <= er["min"] <= er["median"] <= er["max"] and 0 <= er["empty"] <= 4


def test_reference_arm_other_format_and_shape():
    """--format mxfp4 times the layer with an MXFP4 base; --shape gemma4 the
    Gemma-4 layer shape (here with fewer experts and tokens for speed)."""
    d = _run("--format", "mxfp4")
    assert d["config"]["weight_format"] == "mxfp4" and "mxfp4" in d["config"]["workload"]
    g = _run("--shape", "gemma4", "--experts", "8", "--qlen", "8")
    assert g["config"]["workload"].startswith("gemma4_layer") and "H=2816 I=704" in g["config"]["workload"]
    assert g["config"]["weight_format"] == "rawint4"


def test_weight_bytes_per_value():
    """Half a byte of code per weight plus the group scale: a bf16 (RAWINT4)
    or a UE8M0 byte (MXFP4) per 32 weights."""
    sys.path.insert(0, ROOT)
    import dataclasses
    import bench
    from workloads import CONFIGS
    assert bench.weight_bytes_per_value(CONFIGS[4]) == 0.5 + 2 / 32
    assert bench.weight_bytes_per_value(dataclasses.replace(CONFIGS[4], weight_format="mxfp4")) == 0.5 + 1 / 32


def test_phase_split_of_launches():
    """Forward and backward kernel time per step from the launch list in issue order."""
    sys.path.insert(0, ROOT)
    import bench
    step = [("header_fwd", 0.01), ("route", 0.05), ("gemm_gate_up", 5.0), ("gemm_down", 3.0), ("combine_out", 0.3),
            ("header_bwd", 0.01), ("gemm_down_t", 3.5), ("gemm_gate_up_t", 5.0), ("lora_grads", 1.0),
            ("header_end", 0.01)]
    ph = bench.phase_times(step * 2, 2)
    assert ph == {"fwd_kernel_ms": 8.36, "bwd_kernel_ms": 9.52}
    inf = [("header_fwd", 0.01), ("gemm_gate_up", 5.0), ("gemm_down", 3.0)] * 3
    assert bench.phase_times(inf, 3) == {"fwd_kernel_ms": 8.01, "bwd_kernel_ms": 0.0}


def test_reference_arm_under_torchrun():
    """Launched the way the driver launches N > 1 (torchrun, one process per
    rank): rank 0 alone runs the oracle and prints the line, with n_gpus = N;
    the other ranks exit 0 without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), os.path.join(ROOT, "bench.py"),
           "--gpus", "2", "--impl", "reference", "--config", "0", "--steps", "1", "--warmup", "3", "--cpu-seconds", "0.2"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="1")
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0


def _free_port() -> int:
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]
