"""Pins for oracle.router (no GPU): torch autograd of the literal router
composition, finite differences, and the closed-form structure of the score
gradient."""

import numpy as np
import torch
import torch.nn.functional as F

from oracle import router as orouter


def _case(seed=3, Q=6, E=16, k=4):
    rng = np.random.default_rng(seed)
    z = rng.normal(0, 1.5, (Q, E))
    c = rng.uniform(0.5, 1.5, E)
    g = rng.normal(0, 1, (Q, k))
    return z, c, g, k


def test_forward_matches_the_literal_router():
    z, c, _, k = _case()
    p, ids, w, r = orouter.forward(z, k, c)
    zt = torch.from_numpy(z)
    pt = F.softmax(zt, dim=-1)
    tw, ti = torch.topk(pt, k=k, dim=-1)
    tw = tw / tw.sum(dim=-1, keepdim=True)
    tw = tw * torch.from_numpy(c)[ti]
    assert np.array_equal(ids, ti.numpy())
    np.testing.assert_allclose(w, tw.numpy(), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(r.sum(-1), 1.0, rtol=1e-14)


def test_ties_go_to_the_lower_index():
    z = np.zeros((1, 6))
    z[0, 4] = z[0, 1] = 2.0
    _, ids, _, _ = orouter.forward(z, 3)
    assert ids.tolist() == [[1, 4, 0]]


def test_backward_matches_autograd():
    z, c, g, k = _case()
    _, ids, _, _ = orouter.forward(z, k, c)
    dz, dc = orouter.backward(z, ids, g, c)
    zt = torch.from_numpy(z).requires_grad_(True)
    ct = torch.from_numpy(c).requires_grad_(True)
    it = torch.from_numpy(ids)
    pt = F.softmax(zt, dim=-1)
    sel = torch.gather(pt, 1, it)
    w = sel / sel.sum(-1, keepdim=True) * ct[it]
    (w * torch.from_numpy(g)).sum().backward()
    np.testing.assert_allclose(dz, zt.grad.numpy(), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dc, ct.grad.numpy(), rtol=1e-12, atol=1e-14)


def test_backward_finite_differences():
    z, c, g, k = _case(seed=9, Q=3, E=10, k=3)
    _, ids, _, _ = orouter.forward(z, k, c)
    dz, _ = orouter.backward(z, ids, g, c)
    eps = 1e-6

    def loss(zz):  # the selection is held fixed (a valid subgradient of the piecewise map)
        p = orouter.softmax(zz)
        sel = np.take_along_axis(p, ids, -1)
        return float((sel / sel.sum(-1, keepdims=True) * c[ids] * g).sum())

    num = np.zeros_like(z)
    for i in range(z.shape[0]):
        for j in range(z.shape[1]):
            zp, zm = z.copy(), z.copy()
            zp[i, j] += eps
            zm[i, j] -= eps
            num[i, j] = (loss(zp) - loss(zm)) / (2 * eps)
    np.testing.assert_allclose(dz, num, rtol=1e-6, atol=1e-8)


def test_score_gradient_structure():
    """Outside the k selected experts the gradient is zero (the E-wide
    normalisation cancels in the renormalised weights), and over the k it
    sums to zero (the weights are invariant to a common shift of scores)."""
    z, c, g, k = _case(seed=5)
    _, ids, _, _ = orouter.forward(z, k, c)
    dz, _ = orouter.backward(z, ids, g, c)
    mask = np.zeros_like(z, dtype=bool)
    np.put_along_axis(mask, ids, True, axis=-1)
    assert np.all(np.abs(dz[~mask]) < 1e-15)
    np.testing.assert_allclose(dz.sum(-1), 0.0, atol=1e-14)
