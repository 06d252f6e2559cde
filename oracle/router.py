"""Top-k softmax router hand-off: forward selection and the backward of the
route weights into the router's expert scores.

Test infrastructure only (see the package header).

The router of the adjacent MoE system (``test_gemma4_moe.py``,
``Gemma4TextRouter.forward``) turns expert scores z [Q, E] into
    p = softmax(z) over all E experts
    top-k of p (ids, in descending order of p)
    r_s = p_{id_s} / sum_{s'} p_{id_s'}          (renormalised over the k)
    w_s = r_s * per_expert_scale[id_s]           (the layer's route weights)
The layer returns dRoute = dL/dw. The hand-off computes dL/dz and
dL/dper_expert_scale from it. Written out by the chain rule (this module
evaluates it step by step, without simplification):
    h_s = dRoute_s * per_expert_scale[id_s]                       dL/dr_s
    dL/dp_j = (h_j - sum_s h_s r_s) / P   for selected j (P = sum of the k p), else 0
    dL/dz_i = p_i (dL/dp_i - sum_j p_j dL/dp_j)
    dL/dper_expert_scale[e] = sum over slots routed to e of dRoute_s * r_s

Readings where the pages are silent: equal probabilities are ordered by the
lower expert index first (the selection is then unique); the scores are the
router's output in float32, the hand-off computes in float64 here.

Pins (tests/test_oracle_router.py): torch autograd of the literal
softmax -> topk -> renormalise -> scale composition; central finite
differences; the closed form that the gradient vanishes outside the
selected experts and sums to zero over each token's k scores.
"""

from __future__ import annotations

import numpy as np


def softmax(z: np.ndarray) -> np.ndarray:
    z = np.asarray(z, dtype=np.float64)
    m = z.max(axis=-1, keepdims=True)
    e = np.exp(z - m)
    return e / e.sum(axis=-1, keepdims=True)


def topk_ids(p: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest entries per row, largest first, ties to the lower index."""
    p = np.asarray(p)
    q, E = p.shape
    order = np.lexsort((np.broadcast_to(np.arange(E), (q, E)), -p), axis=-1)  # primary: -p, secondary: index
    return order[:, :k].astype(np.int64)


def forward(scores: np.ndarray, top_k: int, per_expert_scale=None):
    """(probabilities [Q, E], ids [Q, k], route weights w [Q, k], renormalised r [Q, k])."""
    p = softmax(scores)
    ids = topk_ids(p, top_k)
    sel = np.take_along_axis(p, ids, axis=-1)
    r = sel / sel.sum(axis=-1, keepdims=True)
    c = np.ones(p.shape[-1]) if per_expert_scale is None else np.asarray(per_expert_scale, dtype=np.float64)
    w = r * c[ids]
    return p, ids, w, r


def backward(scores: np.ndarray, ids: np.ndarray, grad_route: np.ndarray, per_expert_scale=None):
    """(dL/dscores [Q, E], dL/dper_expert_scale [E]) for dRoute = dL/dw."""
    p = softmax(scores)
    Q, E = p.shape
    ids = np.asarray(ids, dtype=np.int64)
    g = np.asarray(grad_route, dtype=np.float64)
    c = np.ones(E) if per_expert_scale is None else np.asarray(per_expert_scale, dtype=np.float64)
    sel = np.take_along_axis(p, ids, axis=-1)
    P = sel.sum(axis=-1, keepdims=True)
    r = sel / P
    h = g * c[ids]
    dp = np.zeros((Q, E))
    hbar = (h * r).sum(axis=-1, keepdims=True)
    np.put_along_axis(dp, ids, (h - hbar) / P, axis=-1)
    dz = p * (dp - (p * dp).sum(axis=-1, keepdims=True))
    dc = np.zeros(E)
    np.add.at(dc, ids.reshape(-1), (g * r).reshape(-1))
    return dz, dc
