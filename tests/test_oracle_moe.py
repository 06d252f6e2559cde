"""Pins for oracle.moe and oracle.metrics (no GPU).

Checks the oracle against things other than itself: brute-force sorting, a
textbook SwiGLU FFN, the contract test's closed-form clamp fixture, the
page's per-token loop, float64 finite differences, torch autograd, and the
window/zero-row invariants of the contract test.
"""

import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import metrics, moe as omoe, rawint4 as orq
from tests._util import f64, oracle_layer
from workloads import CONFIGS, LORA_NAMES, make_workload, small_config

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _tiny(limit=0.0, seed=7, E=4, k=2, H=64, I=96, r=4, Q=6, x_std=1.0):
    cfg = small_config("t", E, k, H, I, r, Q, swiglu_limit=limit, x_std=x_std)
    return make_workload(cfg, seed=seed)


# ------------------------------------------------------------------ metric

def test_metric_closed_forms():
    e = np.array([3.0, -4.0, 0.0])
    assert metrics.relative_l2_and_cosine(e, e) == (0.0, 1.0)
    rel, cos = metrics.relative_l2_and_cosine(1.1 * e, e)
    assert abs(rel - 0.1) < 1e-12 and abs(cos - 1.0) < 1e-12
    rel, cos = metrics.relative_l2_and_cosine(np.array([0.0, 0.0, 5.0]), e)
    assert abs(cos) < 1e-12 and abs(rel - np.sqrt(50.0) / 5.0) < 1e-12


# ------------------------------------------------------------ permutation

@pytest.mark.parametrize("seed", range(6))
def test_permutation_brute_force(seed):
    rng = np.random.default_rng(seed)
    E, Q, k = 5, 11, 3
    ids = rng.integers(0, E, (Q, k))
    if seed % 2:
        ids[rng.integers(0, Q), rng.integers(0, k)] = E + 2  # out-of-range id
        ids[rng.integers(0, Q), rng.integers(0, k)] = -1
    counts, offsets, perm, inv = omoe.stable_expert_permutation(ids, E)
    flat = ids.reshape(-1)
    expect = sorted([f for f in range(Q * k) if 0 <= flat[f] < E], key=lambda f: (flat[f], f))
    assert perm.tolist() == expect
    assert counts.sum() == len(expect) == offsets[-1]
    for e in range(E):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert np.all(flat[seg] == e) and np.all(np.diff(seg) > 0)
    for p, f in enumerate(perm):
        assert inv[f] == p
    assert np.all(inv[(flat < 0) | (flat >= E)] == -1)


# ---------------------------------------------------------------- forward

def test_single_expert_is_textbook_swiglu_ffn():
    """E=1, top-1, w=1, L=0, LoRA B=0: out = (silu(x Wg^T) * (x Wu^T)) Wd^T."""
    wl = _tiny(E=1, k=1)
    wl.route_weights.fill_(1.0)
    for n in ("gate_lora_b", "up_lora_b", "down_lora_b"):
        wl.lora[n].zero_()
    layer = oracle_layer(wl)
    out, _ = omoe.forward(layer, f64(wl.x), wl.expert_ids.numpy(), f64(wl.route_weights))
    # dense weights through the page's transpose-free loop (dY = identity)
    Wg = orq.transpose_free_dx(np.eye(layer.inter), layer.gate_q[0], layer.gate_s[0])
    Wu = orq.transpose_free_dx(np.eye(layer.inter), layer.up_q[0], layer.up_s[0])
    Wd = orq.transpose_free_dx(np.eye(layer.hidden), layer.down_q[0], layer.down_s[0])
    x = torch.from_numpy(f64(wl.x))
    ref = F.linear(F.silu(F.linear(x, torch.from_numpy(Wg))) * F.linear(x, torch.from_numpy(Wu)), torch.from_numpy(Wd))
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-12, atol=1e-10)


def test_lora_b_zero_equals_base_only():
    wl = _tiny(limit=2.0, x_std=2.0)
    layer = oracle_layer(wl)
    for n in ("gate_lora_b", "up_lora_b", "down_lora_b"):
        layer.lora[n][:] = 0.0
    out_b0, _ = omoe.forward(layer, f64(wl.x), wl.expert_ids.numpy(), f64(wl.route_weights))
    for n in LORA_NAMES:
        layer.lora[n][:] = 0.0
    out_base, _ = omoe.forward(layer, f64(wl.x), wl.expert_ids.numpy(), f64(wl.route_weights))
    assert np.array_equal(out_b0, out_base)
    assert np.count_nonzero(out_base)


def test_token_loop_matches_expert_loop():
    for limit in (0.0, 2.0):
        wl = _tiny(limit=limit, x_std=2.0)
        layer = oracle_layer(wl)
        a, _ = omoe.forward(layer, f64(wl.x), wl.expert_ids.numpy(), f64(wl.route_weights))
        b = omoe.forward_token_loop(layer, f64(wl.x), wl.expert_ids.numpy(), f64(wl.route_weights))
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)


def _clamp_fixture():
    """The contract test's clamp-boundary layer (E=4, k=2, H=I=256, r=8, Q=9)."""
    gold = json.load(open(os.path.join(GOLDEN, "clamp_boundary.json")))
    cfg = small_config("clamp", 4, 2, 256, 256, 8, 9, swiglu_limit=gold["swiglu_limit"])
    wl = make_workload(cfg)
    wl.gate_q.fill_(0x99)
    wl.up_q.fill_(0x99)
    wl.up_q[:, 1::2].fill_(0x77)
    wl.gate_s.fill_(0.5)
    wl.up_s.fill_(0.5)
    for n in ("gate_lora_b", "up_lora_b", "down_lora_b"):
        wl.lora[n].zero_()
    wl.x.zero_()
    wl.x[:, 0] = torch.tensor(gold["x_col0"])
    wl.x[:, 1] = torch.tensor(gold["x_col1"])
    wl.expert_ids.copy_(torch.tensor([[0, 1] if t % 2 == 0 else [1, 0] for t in range(9)]))
    wl.route_weights.copy_(torch.stack((torch.linspace(0.55, 0.75, 9), torch.linspace(0.45, 0.25, 9)), 1))
    return gold, wl


def test_clamp_boundary_closed_form():
    gold, wl = _clamp_fixture()
    layer = oracle_layer(wl)
    _, ctx = omoe.forward(layer, f64(wl.x), wl.expert_ids.numpy(), f64(wl.route_weights))
    for e, ec in ctx.experts.items():
        G_exp = np.array(gold["G"])[ec.tokens]
        assert np.array_equal(ec.G, np.repeat(G_exp[:, None], 256, 1))
        sign = np.where(np.arange(256) % 2 == 0, 1.0, -1.0)
        assert np.array_equal(ec.U, G_exp[:, None] * sign[None, :])
        Gc, Uc, mg, mu = omoe.clamp_preacts(ec.G, ec.U, gold["swiglu_limit"])
        assert np.array_equal(Gc[:, 0], np.array(gold["G_clamped"])[ec.tokens])
        assert np.array_equal(Uc[:, 0], np.array(gold["U_even_clamped"])[ec.tokens])
        assert np.array_equal(Uc[:, 1], np.array(gold["U_odd_clamped"])[ec.tokens])
        assert np.array_equal(mg[:, 0], np.array(gold["gate_grad_passes"])[ec.tokens])
        assert np.array_equal(mu[:, 0], np.array(gold["up_grad_passes"])[ec.tokens])
        # h = silu(G') U' with the library silu
        h_ref = F.silu(torch.from_numpy(Gc)).numpy() * Uc
        np.testing.assert_allclose(ec.h, h_ref, rtol=1e-14, atol=1e-14)
    # rows 7/8 round onto the bound in bf16 but must keep the masked gradient
    Gb = torch.tensor(gold["G"], dtype=torch.float32).to(torch.bfloat16).float().tolist()
    assert Gb == gold["G_bf16_rounded"]


def test_clamp_boundary_gradients_follow_masks():
    gold, wl = _clamp_fixture()
    layer = oracle_layer(wl)
    _, ctx = omoe.forward(layer, f64(wl.x), wl.expert_ids.numpy(), f64(wl.route_weights))
    gin, groute, grads = omoe.backward(layer, ctx, f64(wl.grad_out))
    # gate rows 6,7 and up rows 0,6,7,8 are blocked: with LoRA B = 0 the base
    # dX of a token is W_g^T dG + W_u^T dU, so check dG/dU directly
    for e, ec in ctx.experts.items():
        g = f64(wl.grad_out)[ec.tokens]
        dy = ec.w[:, None] * g
        Wg, Wu, Wd = layer.dense(e)
        dh = dy @ Wd
        dG, dU = omoe.swiglu_backward(ec.G, ec.U, dh, 2.0)
        blocked_g = ~np.array(gold["gate_grad_passes"])[ec.tokens]
        blocked_u = ~np.array(gold["up_grad_passes"])[ec.tokens]
        assert np.all(dG[blocked_g] == 0) and np.all(dU[blocked_u] == 0)
        live = ec.G[:, 0] != 0  # G = 0 gives U' = 0 and silu(0) = 0, so both gradients vanish there
        assert np.all(dG[~blocked_g & live][:, :4] != 0) and np.all(dU[~blocked_u & live][:, :4] != 0)


# --------------------------------------------------------------- backward

def _objective(layer, x, ids, rw, gout):
    out, _ = omoe.forward(layer, x, ids, rw)
    return float(np.sum(out * gout))


def test_backward_finite_differences():
    wl = _tiny(limit=2.0, x_std=2.0, seed=11, E=3, H=64, I=64, Q=5)
    layer = oracle_layer(wl)
    x, ids, rw, gout = f64(wl.x), wl.expert_ids.numpy(), f64(wl.route_weights), f64(wl.grad_out)
    _, ctx = omoe.forward(layer, x, ids, rw)
    margin = min(min(np.min(np.abs(ec.G - 2.0)), np.min(np.abs(np.abs(ec.U) - 2.0))) for ec in ctx.experts.values())
    assert margin > 1e-4  # no kink within the step
    assert any(np.any(ec.G > 2.0) for ec in ctx.experts.values())  # the clamp is exercised
    gin, groute, grads = omoe.backward(layer, ctx, gout)
    rng = np.random.default_rng(0)
    step = 1e-6

    def check(arr, analytic, n=6):
        for _ in range(n):
            idx = tuple(rng.integers(0, s) for s in arr.shape)
            old = arr[idx]
            arr[idx] = old + step
            jp = _objective(layer, x, ids, rw, gout)
            arr[idx] = old - step
            jm = _objective(layer, x, ids, rw, gout)
            arr[idx] = old
            fd = (jp - jm) / (2 * step)
            assert abs(fd - analytic[idx]) <= 1e-6 * max(1.0, abs(fd)), (idx, fd, analytic[idx])

    check(x, gin)
    check(rw, groute)
    for n in LORA_NAMES:
        # only rows of routed experts carry gradient; sample there
        check(layer.lora[n], grads[n])


def test_backward_matches_torch_autograd():
    """The page's oracle differentiates its per-token equation with autograd."""
    wl = _tiny(limit=2.0, x_std=2.0, seed=5)
    layer = oracle_layer(wl)
    c = layer.scaling
    x = torch.tensor(f64(wl.x), requires_grad=True)
    rw = torch.tensor(f64(wl.route_weights), requires_grad=True)
    lo = {n: torch.tensor(layer.lora[n], requires_grad=True) for n in LORA_NAMES}
    dense = {e: [torch.from_numpy(w) for w in layer.dense(e)] for e in range(layer.experts)}
    ids = wl.expert_ids.numpy()
    L = 2.0
    rows = []
    for t in range(ids.shape[0]):
        acc = 0
        for s in range(ids.shape[1]):
            e = int(ids[t, s])
            Wg, Wu, Wd = dense[e]
            xt = x[t:t + 1]
            g = F.linear(xt, Wg) + c * F.linear(F.linear(xt, lo["gate_lora_a"][e]), lo["gate_lora_b"][e])
            u = F.linear(xt, Wu) + c * F.linear(F.linear(xt, lo["up_lora_a"][e]), lo["up_lora_b"][e])
            g = torch.where(g <= L, g, torch.full_like(g, L))
            u = torch.where(u < -L, torch.full_like(u, -L), torch.where(u > L, torch.full_like(u, L), u))
            h = F.silu(g) * u
            y = F.linear(h, Wd) + c * F.linear(F.linear(h, lo["down_lora_a"][e]), lo["down_lora_b"][e])
            acc = acc + y * rw[t, s]
        rows.append(acc)
    out = torch.cat(rows, 0)
    gout = torch.from_numpy(f64(wl.grad_out))
    res = torch.autograd.grad(out, [x, rw] + [lo[n] for n in LORA_NAMES], grad_outputs=gout)
    o_out, ctx = omoe.forward(layer, f64(wl.x), ids, f64(wl.route_weights))
    gin, groute, grads = omoe.backward(layer, ctx, f64(wl.grad_out))
    np.testing.assert_allclose(o_out, out.detach().numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(gin, res[0].numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(groute, res[1].numpy(), rtol=1e-11, atol=1e-12)
    for n, r_ in zip(LORA_NAMES, res[2:]):
        np.testing.assert_allclose(grads[n], r_.numpy(), rtol=1e-11, atol=1e-12, err_msg=n)


def test_dense_and_transpose_free_backward_agree():
    wl = _tiny(limit=2.0, x_std=2.0, seed=9, H=64, I=64)
    layer = oracle_layer(wl)
    _, ctx = omoe.forward(layer, f64(wl.x), wl.expert_ids.numpy(), f64(wl.route_weights))
    a = omoe.backward(layer, ctx, f64(wl.grad_out))
    b = omoe.backward(layer, ctx, f64(wl.grad_out), transpose_free=True)
    np.testing.assert_allclose(a[0], b[0], rtol=1e-12, atol=1e-12)
    for n in LORA_NAMES:
        np.testing.assert_allclose(a[2][n], b[2][n], rtol=1e-12, atol=1e-12)


def test_unrouted_experts_have_zero_grads_and_window():
    wl = _tiny(E=6, seed=3)
    wl.expert_ids.copy_(torch.tensor([[1, 4] if t % 2 == 0 else [4, 1] for t in range(wl.cfg.qlen)]))
    layer = oracle_layer(wl)
    _, ctx = omoe.forward(layer, f64(wl.x), wl.expert_ids.numpy(), f64(wl.route_weights))
    _, _, grads = omoe.backward(layer, ctx, f64(wl.grad_out))
    for n in LORA_NAMES:
        for e in (0, 2, 3, 5):
            assert np.count_nonzero(grads[n][e]) == 0
        for e in (1, 4):
            assert np.count_nonzero(grads[n][e]) > 0
    sentinel = {n: np.full(v.shape, 7.0) for n, v in grads.items()}
    w1 = omoe.grad_window(sentinel, grads, accumulate=False, grad_scale=0.5)
    w2 = omoe.grad_window(w1, grads, accumulate=True, grad_scale=0.5)
    for n in LORA_NAMES:
        np.testing.assert_array_equal(w1[n], 0.5 * grads[n])
        np.testing.assert_allclose(w2[n], grads[n], rtol=1e-15)
        assert np.count_nonzero(w1[n][[0, 2, 3, 5]]) == 0


def test_out_of_range_ids_contribute_nothing():
    wl = _tiny(seed=4)
    layer = oracle_layer(wl)
    ids = wl.expert_ids.numpy().copy()
    ids[2, 1] = layer.experts  # sentinel id
    out, ctx = omoe.forward(layer, f64(wl.x), ids, f64(wl.route_weights))
    _, groute, _ = omoe.backward(layer, ctx, f64(wl.grad_out))
    assert groute[2, 1] == 0.0
    ids2 = ids.copy()
    rw2 = f64(wl.route_weights).copy()
    rw2[2, 1] = 0.0
    ids2[2, 1] = ids2[2, 0]
    out2, _ = omoe.forward(layer, f64(wl.x), ids2, rw2)
    np.testing.assert_allclose(out, out2, rtol=1e-13, atol=1e-13)


def test_config0_runs_and_has_signal():
    wl = make_workload(CONFIGS[0])
    layer = oracle_layer(wl)
    out, ctx = omoe.forward(layer, f64(wl.x), wl.expert_ids.numpy(), f64(wl.route_weights))
    gin, groute, grads = omoe.backward(layer, ctx, f64(wl.grad_out))
    for arr in [out, gin, groute] + list(grads.values()):
        assert np.all(np.isfinite(arr)) and np.count_nonzero(arr)


def test_duplicate_expert_slots_are_independent():
    """A token routed twice to the same expert (top-k never does this, the
    layer accepts it): the forward is linear in the route weights, so slots
    (e, w1), (e, w2) give the output of one slot (e, w1 + w2) next to a
    zero-weight slot; both duplicate slots see the same dRoute = <dY, y_e>,
    and the LoRA gradients are those of the merged slot."""
    wl = _tiny(seed=11)
    layer = oracle_layer(wl)
    Q = wl.cfg.qlen
    x, dy = f64(wl.x), f64(wl.grad_out)
    dup = np.array([[t % 4, t % 4] for t in range(Q)], dtype=np.int64)
    w = np.stack([np.linspace(0.2, 0.7, Q), np.linspace(0.5, 0.1, Q)], 1)
    merged = np.array([[t % 4, (t + 1) % 4] for t in range(Q)], dtype=np.int64)
    wm = np.stack([w[:, 0] + w[:, 1], np.zeros(Q)], 1)
    out_d, ctx_d = omoe.forward(layer, x, dup, w)
    out_m, ctx_m = omoe.forward(layer, x, merged, wm)
    np.testing.assert_allclose(out_d, out_m, rtol=1e-12, atol=1e-12)
    gin_d, gr_d, gd = omoe.backward(layer, ctx_d, dy)
    gin_m, gr_m, gm = omoe.backward(layer, ctx_m, dy)
    np.testing.assert_allclose(gin_d, gin_m, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(gr_d[:, 0], gr_d[:, 1], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(gr_d[:, 0], gr_m[:, 0], rtol=1e-12, atol=1e-12)
    for n in LORA_NAMES:
        np.testing.assert_allclose(gd[n], gm[n], rtol=1e-11, atol=1e-11)


def test_mask_override_reproduces_and_flips_one_decision():
    """backward(masks=...) with the clamp's own decisions is bit-identical to
    backward(); flipping one gate decision of one row changes that row's
    token alone, by the closed-form term dh U' silu'(G') times the gate row of
    W_g (plus its LoRA term)."""
    wl = _tiny(limit=1.0, x_std=2.0)
    layer = oracle_layer(wl)
    out, ctx = omoe.forward(layer, f64(wl.x), wl.expert_ids.numpy(), f64(wl.route_weights))
    gin, groute, grads = omoe.backward(layer, ctx, f64(wl.grad_out))
    own = {}
    for e, ec in ctx.experts.items():
        _, _, mg, mu = omoe.clamp_preacts(ec.G, ec.U, layer.swiglu_limit)
        own[e] = (mg, mu)
    gin2, groute2, grads2 = omoe.backward(layer, ctx, f64(wl.grad_out), masks=own)
    assert np.array_equal(gin, gin2) and np.array_equal(groute, groute2)
    for n in LORA_NAMES:
        assert np.array_equal(grads[n], grads2[n])
    # flip the decision of one clamped gate element
    e = next(e for e, (mg, _) in own.items() if not mg.all())
    row, col = map(int, np.argwhere(~own[e][0])[0])
    flipped = {k: (mg.copy(), mu.copy()) for k, (mg, mu) in own.items()}
    flipped[e][0][row, col] = True
    gin3, _, _ = omoe.backward(layer, ctx, f64(wl.grad_out), masks=flipped)
    tok = int(ctx.experts[e].tokens[row])
    diff = gin3 - gin
    assert np.count_nonzero(np.abs(diff).sum(axis=1)) == 1 and np.abs(diff[tok]).sum() > 0
