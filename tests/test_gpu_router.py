"""GPU parity of the router hand-off (rawint4_moe_router_topk / _bwd) with
the float64 router oracle (test_gemma4_moe.py, Gemma4TextRouter.forward).

Scores are seeded N(0, 1.5^2) draws, so equal probabilities do not occur and
the selected experts must match exactly; the weights and gradients are
compared within fp32 accuracy (the GPU computes in fp32)."""

import numpy as np
import pytest
import torch

from oracle import metrics
from oracle import router as orouter

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("Q,E,k", [(257, 128, 8), (5, 384, 8), (64, 16, 2), (3, 4096, 32)])
def test_router_topk_and_handoff(Q, E, k):
    from int4_quantised_moe_b200 import binding as B
    g = torch.Generator().manual_seed(1000 + Q + E + k)
    z = (torch.randn((Q, E), generator=g) * 1.5).float()
    c = (torch.rand(E, generator=g) + 0.5).float()
    dr = torch.randn((Q, k), generator=g).float()
    ids, w = B.router_topk(z.cuda(), k, c.cuda())
    _, o_ids, o_w, _ = orouter.forward(z.double().numpy(), k, c.double().numpy())
    assert np.array_equal(ids.cpu().numpy(), o_ids)
    np.testing.assert_allclose(w.cpu().numpy(), o_w, rtol=2e-5, atol=1e-7)
    dz, dc = B.router_bwd(z.cuda(), ids, dr.cuda(), c.cuda(), want_escale_grad=True)
    o_dz, o_dc = orouter.backward(z.double().numpy(), o_ids, dr.double().numpy(), c.double().numpy())
    for name, got, ref in (("dscores", dz, o_dz), ("descale", dc, o_dc)):
        rel, cos = metrics.relative_l2_and_cosine(got.double().cpu().numpy(), ref)
        assert rel <= 1e-5 and cos >= 0.99999, (name, rel, cos)
    # outside the selected experts the gradient is exactly zero
    mask = torch.zeros((Q, E), dtype=torch.bool)
    mask.scatter_(1, ids.cpu(), True)
    assert torch.count_nonzero(dz.cpu()[~mask]) == 0


def test_router_rejects_bad_arguments():
    from int4_quantised_moe_b200 import binding as B
    z = torch.zeros((4, 8), device="cuda")
    with pytest.raises(B.RawInt4Error):
        B.router_topk(z, 9)
    with pytest.raises(B.RawInt4Error):
        B.router_topk(torch.zeros((4, 40), device="cuda"), 33)
