"""GPU parity of the whole layer against the float64 oracle, through the C ABI.

Covers the small configurations element by element, the contract test's
lifecycle (test_rawint4_sft_numerical.py: GAS1 overwrite with sentinel
buffers, accumulation, the lazy clear of a new window, checkpoint-recompute
cache replacement, frozen-base fail-fast, base bytes unchanged), the
clamp-boundary fixture, the rectangular multiblock variant, the inference
regression with zero LoRA, the base-only (lora = NULL) inference forward, bad
expert ids, qlen = 0 and a missing saved forward.
"""

import hashlib

import numpy as np
import pytest
import torch

from oracle import metrics, moe as omoe
from tests._gpu import (TOL_DX, TOL_LORA, TOL_OUT, TOL_ROUTE, grad_buffers, make_layer, run_fwd_bwd)
from tests._util import f64, oracle_layer
from workloads import CONFIGS, LORA_NAMES, Workload, lora_shapes, make_workload, small_config

pytestmark = pytest.mark.gpu
DEV = "cuda"


def close(name, actual, expected, tol):
    a = actual.float().cpu().numpy() if isinstance(actual, torch.Tensor) else np.asarray(actual)
    e = np.asarray(expected, dtype=np.float64)
    assert np.all(np.isfinite(a)), f"{name}: non-finite values"
    assert np.count_nonzero(e), f"{name}: reference has no signal"
    rel, cos = metrics.relative_l2_and_cosine(a, e)
    assert rel <= tol[0] and cos >= tol[1], f"{name}: rel-L2 {rel:.3e} (<= {tol[0]}), cos {cos:.6f} (>= {tol[1]})"
    return rel, cos


def oracle(wl: Workload):
    layer = oracle_layer(wl)
    out, ctx = omoe.forward(layer, f64(wl.x), wl.expert_ids.cpu().numpy(), f64(wl.route_weights))
    gin, groute, grads = omoe.backward(layer, ctx, f64(wl.grad_out))
    return out, gin, groute, grads


MASK_DELTA = 4e-3  # bound on |G_gpu - G_oracle| (fp32 accumulation vs float64), as in test_gpu_fullsize


def oracle_gpu_masks(wl: Workload, perm, G, U):
    """The oracle with the clamp masks decided the GPU's way inside the band
    where both decisions are correct within fp32 (|G - L|, |U +- L| below
    MASK_DELTA): the GPU's saved fp32 pre-activations (perm, G, U from
    Layer.saved_preacts) must lie within MASK_DELTA of the oracle's, and
    every mask decision outside the band is the oracle's own. Returns the
    oracle's (out, grad_in, grad_route, grads) and the number of elements
    decided inside the band."""
    layer = oracle_layer(wl)
    L = float(wl.cfg.swiglu_limit)
    k = wl.cfg.top_k
    out, ctx = omoe.forward(layer, f64(wl.x), wl.expert_ids.cpu().numpy(), f64(wl.route_weights))
    perm_h = perm.cpu().numpy()
    inv = np.full(perm_h.size, -1, dtype=np.int64)
    inv[perm_h] = np.arange(perm_h.size)
    Gh, Uh = G.double().cpu().numpy(), U.double().cpu().numpy()
    masks, band = {}, 0
    for e, c in ctx.experts.items():
        rows = inv[c.slots]
        g_gpu, u_gpu = Gh[rows], Uh[rows]
        assert np.abs(g_gpu - c.G).max() <= MASK_DELTA and np.abs(u_gpu - c.U).max() <= MASK_DELTA, e
        if L > 0:
            pass_g, pass_u = c.G <= L, (c.U >= -L) & (c.U <= L)
            near_g = np.abs(c.G - L) < MASK_DELTA
            near_u = (np.abs(c.U - L) < MASK_DELTA) | (np.abs(c.U + L) < MASK_DELTA)
            pass_g = np.where(near_g, g_gpu <= L, pass_g)
            pass_u = np.where(near_u, (u_gpu >= -L) & (u_gpu <= L), pass_u)
            band += int(near_g.sum() + near_u.sum())
            masks[e] = (pass_g, pass_u)
    gin, groute, grads = omoe.backward(layer, ctx, f64(wl.grad_out), masks=masks if L > 0 else None)
    return (out, gin, groute, grads), band


def base_hash(wl: Workload) -> str:
    h = hashlib.sha256()
    for t in (wl.gate_q, wl.gate_s, wl.up_q, wl.up_s, wl.down_q, wl.down_s):
        b = t.detach().cpu().contiguous().view(torch.uint8).numpy().tobytes()
        h.update(len(b).to_bytes(8, "little"))
        h.update(b)
    return h.hexdigest()


# ----------------------------------------------------- contract-test fixtures

def contract_workload(inter=256, qlen=5, limit=0.0, seed=20261001):
    """Layer of the contract test (E=4, k=2, H=256, r=8, alpha=16): uniform codes,
    scales U[0.01, 0.07), signed extremes, one zero scale, LoRA N(0, 0.04^2)."""
    cfg = small_config("contract", 4, 2, 256, inter, 8, qlen, swiglu_limit=limit, alpha=16.0)
    wl = make_workload(cfg, seed=seed)
    for n in LORA_NAMES:
        wl.lora[n] = (wl.lora[n].float() * 2.0).to(torch.bfloat16)  # std 0.04
    wl.gate_q[0, 0].fill_(0x00)
    wl.up_q[0, 0].fill_(0xFF)
    wl.gate_q[0, 1].fill_(0xFF)
    wl.up_q[0, 1].fill_(0x00)
    wl.gate_s[0, :2].fill_(0.0625)
    wl.up_s[0, :2].fill_(0.0625)
    wl.down_s[3, -1, -1] = 0.0
    return wl


def contract_batch(wl: Workload, pair, seed):
    """_make_batch of the contract test: x ~ N(0, 0.2^2) with rows 0/1 at +1/-1,
    grad_output ~ N(0, 0.1^2), alternating expert pairs, linspace route weights."""
    Q, H = wl.cfg.qlen, wl.cfg.hidden
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn((Q, H), generator=g) * 0.2).to(torch.bfloat16)
    x[0].fill_(1.0)
    x[1].fill_(-1.0)
    dy = (torch.randn((Q, H), generator=g) * 0.1).to(torch.bfloat16)
    a, b = pair
    ids = torch.tensor([[a, b] if t % 2 == 0 else [b, a] for t in range(Q)], dtype=torch.int64)
    w = torch.stack((torch.linspace(0.55, 0.75, Q), torch.linspace(0.45, 0.25, Q)), 1).float()
    return Workload(wl.cfg, wl.gate_q, wl.gate_s, wl.up_q, wl.up_s, wl.down_q, wl.down_s, wl.lora, x, ids, w, dy)


def on_gpu(wl: Workload) -> Workload:
    return wl.to(DEV)


# ------------------------------------------------------------------ tests

@pytest.mark.parametrize("cfg_id", [0, 1])
def test_config_parity(cfg_id):
    wl = make_workload(CONFIGS[cfg_id])
    out_r, gin_r, groute_r, grads_r = oracle(wl)
    g = on_gpu(wl)
    layer = make_layer(g)
    grads = grad_buffers(g)
    out, gin, groute = run_fwd_bwd(layer, g, grads)
    assert layer.status() == 0
    close("out", out, out_r, TOL_OUT)
    close("grad_in", gin, gin_r, TOL_DX)
    close("grad_route", groute, groute_r, TOL_ROUTE)
    for n in LORA_NAMES:
        close(n, grads[n], grads_r[n], TOL_LORA)


@pytest.mark.parametrize("limit", [0.0, 2.0])
def test_rectangular_multiblock(limit):
    """I = 384, Q = 17: every active expert gets 17 rows (a ragged token tile)."""
    wl = contract_workload(inter=384, qlen=17, limit=limit)
    b = contract_batch(wl, (0, 1), 3000)
    out_r, gin_r, groute_r, grads_r = oracle(b)
    g = on_gpu(b)
    layer = make_layer(g)
    grads = grad_buffers(g)
    out, gin, groute = run_fwd_bwd(layer, g, grads, grad_scale=0.5)
    close("out", out, out_r, TOL_OUT)
    close("grad_in", gin, gin_r, TOL_DX)
    close("grad_route", groute, groute_r, TOL_ROUTE)
    for n in LORA_NAMES:
        close(n, grads[n], 0.5 * grads_r[n], TOL_LORA)
        for e in (2, 3):
            assert torch.count_nonzero(grads[n][e]) == 0


def test_gradient_window_lifecycle():
    """GAS1 overwrite (sentinel 7.0), GAS2/GAS8 accumulation, lazy clear of a new
    window, checkpoint-recompute cache replacement, frozen base, base unchanged."""
    wl = contract_workload()
    h0 = base_hash(wl)
    scale = 0.5
    pairs = ((0, 1), (1, 2), (2, 3), (0, 3)) * 2
    batches = [contract_batch(wl, p, 3000 + i) for i, p in enumerate(pairs)]
    refs = [oracle(b) for b in batches]
    gw = on_gpu(wl)
    layer = make_layer(gw, max_tokens=32)
    grads = grad_buffers(gw)  # sentinel 7.0
    gb = [on_gpu(b) for b in batches]

    out, gin, groute = run_fwd_bwd(layer, gb[0], grads, accumulate=False, grad_scale=scale)
    close("gas1.out", out, refs[0][0], TOL_OUT)
    close("gas1.dX", gin, refs[0][1], TOL_DX)
    close("gas1.dRoute", groute, refs[0][2], TOL_ROUTE)

    def window(stage, idx, active):
        for n in LORA_NAMES:
            exp = sum(refs[i][3][n] for i in idx) * scale
            close(f"{stage}.{n}", grads[n], exp, TOL_LORA)
            for e in range(4):
                if e not in active:
                    assert torch.count_nonzero(grads[n][e]) == 0, f"{stage}.{n}: stale expert {e}"

    window("gas1", [0], {0, 1})
    run_fwd_bwd(layer, gb[1], grads, accumulate=True, grad_scale=scale)
    window("gas2", [0, 1], {0, 1, 2})
    for i in range(2, 8):
        run_fwd_bwd(layer, gb[i], grads, accumulate=True, grad_scale=scale)
    window("gas8", list(range(8)), {0, 1, 2, 3})

    nw = contract_batch(wl, (2, 3), 4001)
    nref = oracle(nw)
    run_fwd_bwd(layer, on_gpu(nw), grads, accumulate=False, grad_scale=scale)
    for n in LORA_NAMES:
        close(f"lazy_clear.{n}", grads[n], nref[3][n] * scale, TOL_LORA)
        for e in (0, 1):
            assert torch.count_nonzero(grads[n][e]) == 0

    # two saved forwards, then one backward: the second replaces the first
    first, second = contract_batch(wl, (0, 1), 5001), contract_batch(wl, (1, 3), 5002)
    fr, sr = oracle(first), oracle(second)
    f_g, s_g = on_gpu(first), on_gpu(second)
    layer.forward(f_g.expert_ids, f_g.route_weights, f_g.x)
    layer.forward(s_g.expert_ids, s_g.route_weights, s_g.x)
    s_dx = torch.empty_like(s_g.x)
    s_dr = torch.empty(s_g.expert_ids.shape, dtype=torch.float32, device=DEV)
    layer.backward(s_g.grad_out, grads, accumulate=False, grad_scale=scale, grad_in=s_dx, grad_route=s_dr)
    layer.forward(f_g.expert_ids, f_g.route_weights, f_g.x)
    f_dx = torch.empty_like(f_g.x)
    f_dr = torch.empty(f_g.expert_ids.shape, dtype=torch.float32, device=DEV)
    layer.backward(f_g.grad_out, grads, accumulate=True, grad_scale=scale, grad_in=f_dx, grad_route=f_dr)
    close("lifo.second.dX", s_dx, sr[1], TOL_DX)
    close("lifo.second.dRoute", s_dr, sr[2], TOL_ROUTE)
    close("lifo.first.dX", f_dx, fr[1], TOL_DX)
    close("lifo.first.dRoute", f_dr, fr[2], TOL_ROUTE)
    for n in LORA_NAMES:
        close(f"cache_replacement.{n}", grads[n], (sr[3][n] + fr[3][n]) * scale, TOL_LORA)
        assert torch.count_nonzero(grads[n][2]) == 0
    assert layer.status() == 0

    # frozen base: a base-gradient buffer is refused before anything is written
    from int4_quantised_moe_b200 import binding as B
    fb = on_gpu(contract_batch(wl, (0, 1), 7001))
    layer.forward(fb.expert_ids, fb.route_weights, fb.x)
    sentinel = torch.full_like(fb.x, 3.0)
    forbidden = torch.empty(1, dtype=torch.bfloat16, device=DEV)
    before = {n: grads[n].clone() for n in LORA_NAMES}
    with pytest.raises(ValueError, match="frozen"):
        layer.backward(fb.grad_out, grads, grad_in=sentinel, base_grad_gate=forbidden)
    torch.cuda.synchronize()
    assert torch.all(sentinel == 3.0)
    for n in LORA_NAMES:
        assert torch.equal(grads[n], before[n])
    # the saved context is still pending: the proper backward runs
    layer.backward(fb.grad_out, grads, grad_in=sentinel)
    assert layer.status() == 0
    assert base_hash(gw) == h0 == base_hash(wl)


def test_clamp_boundary_fixture():
    """Contract test's clamp fixture: pre-activations below, on and above +-L,
    two of them rounding onto the bound in bf16 but masked in exact arithmetic."""
    from tests.test_oracle_moe import _clamp_fixture
    gold, wl = _clamp_fixture()
    out_r, gin_r, groute_r, grads_r = oracle(wl)
    g = on_gpu(wl)
    layer = make_layer(g)
    grads = grad_buffers(g)
    out, gin, groute = run_fwd_bwd(layer, g, grads)
    close("clamp.out", out, out_r, TOL_OUT)
    close("clamp.dX", gin, gin_r, TOL_DX)
    close("clamp.dRoute", groute, groute_r, TOL_ROUTE)
    for n in LORA_NAMES:
        if np.count_nonzero(grads_r[n]):
            close(f"clamp.{n}", grads[n], grads_r[n], TOL_LORA)
        else:
            assert torch.count_nonzero(grads[n]) == 0, n


def test_inference_regression_zero_lora():
    wl = contract_workload()
    b = contract_batch(wl, (0, 2), 6001)
    for n in LORA_NAMES:
        b.lora[n] = torch.zeros_like(b.lora[n])
    layer_o = oracle_layer(b)
    out_r, _ = omoe.forward(layer_o, f64(b.x), b.expert_ids.numpy(), f64(b.route_weights))
    g = on_gpu(b)
    layer = make_layer(g)
    out = layer.forward(g.expert_ids, g.route_weights, g.x, save_for_backward=False)
    close("inference.out", out, out_r, TOL_OUT)


def test_base_only_inference_forward():
    """lora = NULL: the frozen-base inference forward. Its output equals, bit
    for bit, the LoRA forward with every LoRA B zeroed (the rank stage then adds
    exact zeros to the accumulators), is close to the oracle's base-only layer,
    leaves the base bytes unchanged, and refuses to save a context."""
    from tests._gpu import B
    wl = make_workload(CONFIGS[1])
    zero_b = {n: (torch.zeros_like(t) if n.endswith("_b") else t) for n, t in wl.lora.items()}
    zb = Workload(wl.cfg, wl.gate_q, wl.gate_s, wl.up_q, wl.up_s, wl.down_q, wl.down_s, zero_b, wl.x,
                  wl.expert_ids, wl.route_weights, wl.grad_out)
    out_r, _ = omoe.forward(oracle_layer(zb), f64(zb.x), zb.expert_ids.numpy(), f64(zb.route_weights))
    g = on_gpu(wl)
    before = base_hash(g)
    layer = make_layer(g)
    out = layer.forward(g.expert_ids, g.route_weights, g.x, save_for_backward=False, use_lora=False)
    assert layer.status() == 0
    close("base_only.out", out, out_r, TOL_OUT)
    gz = on_gpu(zb)
    out_z = make_layer(gz).forward(gz.expert_ids, gz.route_weights, gz.x, save_for_backward=False)
    assert torch.equal(out.view(torch.int16), out_z.view(torch.int16))
    with pytest.raises(B.RawInt4Error) as ei:
        layer.forward(g.expert_ids, g.route_weights, g.x, save_for_backward=True, use_lora=False)
    assert ei.value.code == B.INVALID_ARGUMENT
    assert base_hash(g) == before


def test_bad_expert_id_and_status():
    wl = make_workload(CONFIGS[0])
    ids = wl.expert_ids.clone()
    ids[2, 1] = wl.cfg.experts  # sentinel id: that slot contributes nothing
    bad = Workload(wl.cfg, wl.gate_q, wl.gate_s, wl.up_q, wl.up_s, wl.down_q, wl.down_s, wl.lora, wl.x, ids,
                   wl.route_weights, wl.grad_out)
    out_r, gin_r, groute_r, grads_r = oracle(bad)
    g = on_gpu(bad)
    layer = make_layer(g)
    grads = grad_buffers(g)
    out, gin, groute = run_fwd_bwd(layer, g, grads)
    from int4_quantised_moe_b200 import binding as B
    st = layer.status()
    assert st & B.DEV_BAD_EXPERT_ID
    assert layer.status() == 0  # reading clears
    close("bad.out", out, out_r, TOL_OUT)
    close("bad.grad_in", gin, gin_r, TOL_DX)
    assert float(groute[2, 1]) == 0.0


def test_backward_without_saved_forward_does_nothing():
    from int4_quantised_moe_b200 import binding as B
    wl = on_gpu(make_workload(CONFIGS[0]))
    layer = make_layer(wl)
    grads = grad_buffers(wl)
    gin = torch.full_like(wl.x, 3.0)
    layer.backward(wl.grad_out, grads, grad_in=gin)
    assert layer.status() & B.DEV_NO_SAVED_FORWARD
    assert torch.all(gin == 3.0) and all(torch.all(grads[n] == 7.0) for n in LORA_NAMES)
    # one backward per saving forward; a forward without saving invalidates
    layer.forward(wl.expert_ids, wl.route_weights, wl.x, save_for_backward=True)
    layer.backward(wl.grad_out, grads, grad_in=gin)
    assert layer.status() == 0
    gin2 = torch.full_like(wl.x, 3.0)
    layer.backward(wl.grad_out, grads, grad_in=gin2)
    assert layer.status() & B.DEV_NO_SAVED_FORWARD
    assert torch.all(gin2 == 3.0)
    layer.forward(wl.expert_ids, wl.route_weights, wl.x, save_for_backward=False)
    layer.backward(wl.grad_out, grads, grad_in=gin2)
    assert layer.status() & B.DEV_NO_SAVED_FORWARD


def test_qlen_zero():
    wl = on_gpu(make_workload(CONFIGS[0]))
    layer = make_layer(wl)
    grads = grad_buffers(wl)
    empty_x = wl.x[:0]
    out = layer.forward(wl.expert_ids[:0], wl.route_weights[:0], empty_x)
    # the backward needs real buffers; with a saved qlen of 0 it writes none of them
    layer.backward(wl.grad_out, grads, accumulate=True, grad_in=torch.empty_like(wl.x))
    assert all(torch.all(grads[n] == 7.0) for n in LORA_NAMES)
    layer.forward(wl.expert_ids[:0], wl.route_weights[:0], empty_x)
    layer.backward(wl.grad_out, grads, accumulate=False, grad_in=torch.empty_like(wl.x))
    assert all(torch.count_nonzero(grads[n]) == 0 for n in LORA_NAMES)
    assert layer.status() == 0


def test_smaller_qlen_than_workspace():
    """A workspace sized for more tokens than the call uses (ragged last tile)."""
    cfg = small_config("ragged", 8, 2, 256, 256, 16, 37, swiglu_limit=2.0, x_std=2.0)
    wl = make_workload(cfg, seed=99)
    out_r, gin_r, groute_r, grads_r = oracle(wl)
    g = on_gpu(wl)
    layer = make_layer(g, max_tokens=300)
    grads = grad_buffers(g)
    out, gin, groute = run_fwd_bwd(layer, g, grads)
    close("out", out, out_r, TOL_OUT)
    close("grad_in", gin, gin_r, TOL_DX)
    close("grad_route", groute, groute_r, TOL_ROUTE)
    for n in LORA_NAMES:
        close(n, grads[n], grads_r[n], TOL_LORA)


@pytest.mark.parametrize("cfg_id", [0, 1])
@pytest.mark.parametrize("dy_exp", [-30, -20, 20])
def test_grad_out_magnitudes(cfg_id, dy_exp):
    """grad_out scaled by 2^dy_exp (exact in bf16). Per-element output gradients
    of a loss averaged over many tokens sit far below fp16's normal range; the
    backward scales grad_out by a power of two before its fp16 operands are
    formed and undoes it in fp32, so every output keeps the same relative
    accuracy at any magnitude (and large gradients do not overflow)."""
    wl = make_workload(CONFIGS[cfg_id])
    dy = (wl.grad_out.float() * 2.0 ** dy_exp).to(torch.bfloat16)
    assert torch.equal(dy.float(), wl.grad_out.float() * 2.0 ** dy_exp)  # the scaling is exact
    wl = Workload(wl.cfg, wl.gate_q, wl.gate_s, wl.up_q, wl.up_s, wl.down_q, wl.down_s, wl.lora, wl.x,
                  wl.expert_ids, wl.route_weights, dy)
    out_r, gin_r, groute_r, grads_r = oracle(wl)
    g = on_gpu(wl)
    layer = make_layer(g)
    grads = grad_buffers(g)
    out, gin, groute = run_fwd_bwd(layer, g, grads)
    assert layer.status() == 0
    close("out", out, out_r, TOL_OUT)
    close("grad_in", gin, gin_r, TOL_DX)
    close("grad_route", groute, groute_r, TOL_ROUTE)
    for n in LORA_NAMES:
        close(n, grads[n], grads_r[n], TOL_LORA)


def test_fp16_overflow_is_reported():
    """An activation beyond the fp16 operand range (one x element of 1e5) sets
    the fp16-overflow status bit instead of passing silently; reading the
    status clears it, and the next in-range call reports nothing."""
    from int4_quantised_moe_b200 import binding as B
    wl = make_workload(CONFIGS[0])
    g = on_gpu(wl)
    layer = make_layer(g)
    x = g.x.clone()
    x[1, 3] = 1e5
    assert float(x[1, 3]) > 65504.0
    layer.forward(g.expert_ids, g.route_weights, x, save_for_backward=False)
    assert layer.status() & B.DEV_FP16_OVERFLOW
    assert layer.status() == 0
    layer.forward(g.expert_ids, g.route_weights, g.x, save_for_backward=False)
    assert layer.status() == 0


def test_wait_timeout_aborts_cleanly():
    """A pipeline-wait bound far below a normal wait (1 ns) sends the GEMM
    kernels down their abort path on purpose: the call reports
    RAWINT4_DEV_TIMEOUT, and with the default bound restored the next call is
    correct, so every warp left, every copy and MMA in flight landed, and the
    tensor memory was released (the contract test's fail-fast intent: an
    error surfaces, nothing hangs)."""
    from int4_quantised_moe_b200 import binding as B
    wl = make_workload(CONFIGS[0])
    out_r, gin_r, groute_r, grads_r = oracle(wl)
    g = on_gpu(wl)
    layer = make_layer(g)
    try:
        B.set_wait_limit_ns(1)
        layer.forward(g.expert_ids, g.route_weights, g.x, save_for_backward=False)
        assert layer.status() & B.DEV_TIMEOUT
    finally:
        B.set_wait_limit_ns(0)
    grads = grad_buffers(g)
    out, gin, groute = run_fwd_bwd(layer, g, grads)
    assert layer.status() == 0
    close("out", out, out_r, TOL_OUT)
    close("grad_in", gin, gin_r, TOL_DX)
    close("grad_route", groute, groute_r, TOL_ROUTE)
    for n in LORA_NAMES:
        close(n, grads[n], grads_r[n], TOL_LORA)


@pytest.mark.parametrize("limit", [0.0, 5.0])
def test_gemma4_shape_parity(limit):
    """The adjacent MoE system's layer shape (test_gemma4_moe.py,
    TestGemma4FullLayerIntegration.real_config: hidden 2816, 128 experts,
    top-8, intermediate 704). H and I are multiples of 64 but I is not one of
    128 or 256, so the last output-feature block of gate/up and of down^T is
    partial and its missing rows must neither be read nor written."""
    cfg = small_config("gemma4", 128, 8, 2816, 704, 8, 48, swiglu_limit=limit, routing="normal_topk", x_std=1.0)
    wl = make_workload(cfg, seed=2026)
    out_r, gin_r, groute_r, grads_r = oracle(wl)
    g = on_gpu(wl)
    layer = make_layer(g)
    grads = grad_buffers(g)
    out, gin, groute = run_fwd_bwd(layer, g, grads)
    assert layer.status() == 0
    close("out", out, out_r, TOL_OUT)
    close("grad_in", gin, gin_r, TOL_DX)
    close("grad_route", groute, groute_r, TOL_ROUTE)
    for n in LORA_NAMES:
        close(n, grads[n], grads_r[n], TOL_LORA)


@pytest.mark.parametrize("rank,fmt,limit", [(40, "rawint4", 0.0), (64, "rawint4", 0.0), (64, "mxfp4", 0.0),
                                            (40, "rawint4", 2.0), (64, "rawint4", 2.0)])
def test_large_rank_parity(rank, fmt, limit):
    """LoRA ranks above 32 (the boundary allows any positive rank; the
    kernels take up to 64): the gate and up rank blocks no longer share one
    64-wide reduction stage, so the gate/up GEMMs run two LoRA stages, the
    rank-side matrices two segments, and the gate/up LoRA gradients one job
    per buffer. Config 1's shape, training step against the oracle, with the
    accumulate/grad_scale window. With the clamp, mask decisions inside the
    fp32 band are taken from the GPU's saved pre-activations (at rank 40 a
    gate pre-activation lies 2.6e-5 from the bound)."""
    import dataclasses
    cfg = dataclasses.replace(CONFIGS[1], rank=rank, alpha=2.0 * rank, weight_format=fmt, swiglu_limit=limit)
    wl = make_workload(cfg)
    g = on_gpu(wl)
    layer = make_layer(g)
    grads = grad_buffers(g)
    out = layer.forward(g.expert_ids, g.route_weights, g.x)
    perm, G, U = layer.saved_preacts()
    (out_r, gin_r, groute_r, grads_r), band = oracle_gpu_masks(wl, perm, G, U)
    gin = torch.full_like(g.x, float("nan"))
    groute = torch.full(g.expert_ids.shape, float("nan"), dtype=torch.float32, device=DEV)
    layer.backward(g.grad_out, grads, accumulate=False, grad_scale=0.5, grad_in=gin, grad_route=groute)
    assert layer.status() == 0
    print(f"rank {rank} {fmt} L={limit}: clamp elements within {MASK_DELTA} of a bound: {band}")
    close("out", out, out_r, TOL_OUT)
    close("grad_in", gin, gin_r, TOL_DX)
    close("grad_route", groute, groute_r, TOL_ROUTE)
    for n in LORA_NAMES:
        close(n, grads[n], 0.5 * grads_r[n], TOL_LORA)
    # a second micro-step of the window adds to the buffers
    run_fwd_bwd(layer, g, grads, grad_scale=0.5, accumulate=True)
    for n in LORA_NAMES:
        close(n, grads[n], grads_r[n], TOL_LORA)
    # the frozen-base forward of the same layer ignores the LoRA tensors
    base = layer.forward(g.expert_ids, g.route_weights, g.x, save_for_backward=False, use_lora=False)
    assert torch.isfinite(base.float()).all()


@pytest.mark.parametrize("tiles", ["narrow", "wide"])
@pytest.mark.parametrize("shape", [("h64_i64", 4, 2, 64, 64, 8, 9, "rawint4"), ("h128_i64", 4, 2, 128, 64, 8, 9, "rawint4"),
                                   ("one_expert_top1", 1, 1, 256, 128, 16, 7, "rawint4"),
                                   ("h64_i192_top3", 3, 3, 64, 192, 4, 11, "rawint4"),
                                   ("mxfp4_h128_i128", 4, 2, 128, 128, 8, 9, "mxfp4")], ids=lambda c: c[0])
def test_smallest_shapes(shape, tiles, monkeypatch):
    """The smallest layers the boundary accepts (H and I of one 64-wide stage,
    a single expert with top_k = 1, I = 192 = three stages with top_k = 3,
    the smallest MXFP4 layer), in both tile configurations."""
    name, E, k, H, I, r, Q, fmt = shape
    monkeypatch.setenv("RAWINT4_TILES", tiles)
    wl = make_workload(small_config(name, E, k, H, I, r, Q, weight_format=fmt), seed=11)
    out_r, gin_r, groute_r, grads_r = oracle(wl)
    g = on_gpu(wl)
    layer = make_layer(g)
    grads = grad_buffers(g)
    out, gin, groute = run_fwd_bwd(layer, g, grads)
    assert layer.status() == 0
    close("out", out, out_r, TOL_OUT)
    close("grad_in", gin, gin_r, TOL_DX)
    close("grad_route", groute, groute_r, TOL_ROUTE)
    for n in LORA_NAMES:
        close(n, grads[n], grads_r[n], TOL_LORA)


@pytest.mark.parametrize("tiles", ["narrow", "wide"])
@pytest.mark.parametrize("case", ["config1", "gemma4_clamp", "rank64", "rank12", "mxfp4"])
def test_tile_configurations(case, tiles, monkeypatch):
    """Both token-tile configurations of the GEMMs on the same inputs: narrow
    (tiles of at most 64 rows, hand-off groups of four stages; chosen for
    layers with few rows per expert) and wide (tiles of up to 192 rows,
    groups of two), forced through RAWINT4_TILES. Config 1 has 32 rows per
    expert on average (some experts need two narrow tiles); the Gemma-4 shape
    has partial feature blocks; rank 64 (without the clamp, whose decisions
    near a bound the plain oracle may take the other way) runs two LoRA
    stages; rank 12 (not a multiple of 8) takes the shared-memory transposes
    of the LoRA fp16 copies; the last case has an MXFP4 base."""
    import dataclasses
    monkeypatch.setenv("RAWINT4_TILES", tiles)
    if case == "config1":
        wl = make_workload(CONFIGS[1])
    elif case == "gemma4_clamp":
        cfg = small_config("gemma4", 128, 8, 2816, 704, 8, 48, swiglu_limit=5.0, routing="normal_topk", x_std=1.0)
        wl = make_workload(cfg, seed=2027)
    elif case == "rank64":
        wl = make_workload(dataclasses.replace(CONFIGS[1], rank=64, alpha=128.0, swiglu_limit=0.0))
    elif case == "rank12":
        wl = make_workload(dataclasses.replace(CONFIGS[1], rank=12, alpha=24.0, swiglu_limit=0.0))
    else:
        wl = make_workload(dataclasses.replace(CONFIGS[1], weight_format="mxfp4", swiglu_limit=0.0))
    out_r, gin_r, groute_r, grads_r = oracle(wl)
    g = on_gpu(wl)
    layer = make_layer(g)
    grads = grad_buffers(g)
    out, gin, groute = run_fwd_bwd(layer, g, grads)
    assert layer.status() == 0
    close("out", out, out_r, TOL_OUT)
    close("grad_in", gin, gin_r, TOL_DX)
    close("grad_route", groute, groute_r, TOL_ROUTE)
    for n in LORA_NAMES:
        close(n, grads[n], grads_r[n], TOL_LORA)


@pytest.mark.parametrize("cfg_id,limit", [(0, 0.0), (1, 2.0), (1, 0.0)])
def test_mxfp4_base_parity(cfg_id, limit):
    """The sibling MXFP4 base (E2M1 codes, UE8M0 group scales; the
    ext_bindings.cpp commit log's MXFP4 routed-expert LoRA kernels): the same
    layer, LoRA, clamp, transpose-free backward and gradient window with
    only the dequantisation changed, against the oracle's MXFP4 layer."""
    import dataclasses
    cfg = dataclasses.replace(CONFIGS[cfg_id], weight_format="mxfp4", swiglu_limit=limit)
    wl = make_workload(cfg)
    assert wl.gate_s.dtype == torch.uint8
    out_r, gin_r, groute_r, grads_r = oracle(wl)
    g = on_gpu(wl)
    layer = make_layer(g)
    grads = grad_buffers(g)
    out, gin, groute = run_fwd_bwd(layer, g, grads)
    assert layer.status() == 0
    close("out", out, out_r, TOL_OUT)
    close("grad_in", gin, gin_r, TOL_DX)
    close("grad_route", groute, groute_r, TOL_ROUTE)
    for n in LORA_NAMES:
        close(n, grads[n], grads_r[n], TOL_LORA)
    # frozen-base inference forward of the MXFP4 layer
    zero_b = {n: (torch.zeros_like(t) if n.endswith("_b") else t) for n, t in wl.lora.items()}
    zb = Workload(wl.cfg, wl.gate_q, wl.gate_s, wl.up_q, wl.up_s, wl.down_q, wl.down_s, zero_b, wl.x,
                  wl.expert_ids, wl.route_weights, wl.grad_out)
    base_r, _ = omoe.forward(oracle_layer(zb), f64(zb.x), zb.expert_ids.numpy(), f64(zb.route_weights))
    base = layer.forward(g.expert_ids, g.route_weights, g.x, save_for_backward=False, use_lora=False)
    assert layer.status() == 0
    close("base_only.out", base, base_r, TOL_OUT)
