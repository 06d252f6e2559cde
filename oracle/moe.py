"""Routed RAWINT4 MoE-LoRA layer: forward, hand-derived backward, gradient window.

Test infrastructure only (see the package header). float64 throughout; bf16
inputs are converted exactly.

What it computes (``routed_rawint4_lora`` / ``run_routed_reference`` of
rawint4_sft_reference.py, with ``_base_linear``, ``_lora_linear`` and
``rawint4_swiglu``). For token t, slot s, expert e = ids[t, s], weight
w = route_weights[t, s], c = alpha / rank and clamp limit L:

    G  = W_g x + c B_g (A_g x)          U = W_u x + c B_u (A_u x)
    G' = min(G, L) if L > 0 else G      U' = min(max(U, -L), L) if L > 0 else U
    h  = silu(G') U'
    y  = W_d h + c B_d (A_d h)
    out[t] = sum_s w y

W_p is the dense dequantisation of expert e's projection p (oracle.rawint4).
The backward is the chain rule of that equation written out by hand (see
``backward``); the clamp passes the gradient where G <= L and where
-L <= U <= L, both bounds included (the explicit ``torch.where`` of
``rawint4_swiglu``), decided on the unrounded pre-activation. The LoRA
gradients follow the contract test's authoritative window
(``test_rawint4_sft_numerical.py``, ``_expected_window`` and the
``accumulate`` / ``grad_scale`` arguments of ``_backward``).

Readings where the pages are silent: ids outside [0, E) contribute nothing
and get a zero routing gradient; the permutation within one expert is
ascending in the flat slot index f = t * top_k + s.

Pins (tests/test_oracle_moe.py): brute-force permutation; a single-expert,
top-1, unit-weight, unclamped layer equals a textbook SwiGLU FFN; LoRA B = 0
equals the base-only MoE; the clamp-boundary fixture of the contract test
(closed form, tests/golden/clamp_boundary.json); the per-token loop of the
page against the per-expert loop; float64 central finite differences and
torch autograd against the hand-derived backward; dense against
transpose-free dX; zero gradients for unrouted experts; accumulation.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, Iterable, List, Optional

import numpy as np

from . import mxfp4, rawint4

LORA_NAMES = ("gate_lora_a", "gate_lora_b", "up_lora_a", "up_lora_b", "down_lora_a", "down_lora_b")


@dataclass
class Layer:
    """Frozen base (packed bytes + float scales) and float64 LoRA tensors.

    gate_q/up_q: uint8 [E, I, H/2]; down_q: uint8 [E, H, I/2];
    *_s: scales [E, N, K/32], float64 or bf16 bit patterns (uint16);
    lora[name]: float64 with the shapes
    A: [E, r, K_in], B: [E, N_out, r].
    """

    gate_q: np.ndarray
    gate_s: np.ndarray
    up_q: np.ndarray
    up_s: np.ndarray
    down_q: np.ndarray
    down_s: np.ndarray
    lora: Dict[str, np.ndarray]
    alpha: float
    swiglu_limit: float = 0.0
    # "rawint4" (scales: float64 or bf16 bit patterns) or "mxfp4" (E2M1
    # codes, scales: UE8M0 bytes, uint8); only the dequantisation differs
    weight_format: str = "rawint4"

    @property
    def experts(self) -> int:
        return self.gate_q.shape[0]

    @property
    def inter(self) -> int:
        return self.gate_q.shape[1]

    @property
    def hidden(self) -> int:
        return self.down_q.shape[1]

    @property
    def rank(self) -> int:
        return self.lora["gate_lora_a"].shape[1]

    @property
    def scaling(self) -> float:
        return self.alpha / self.rank

    @staticmethod
    def _scale(arr: np.ndarray, e: int) -> np.ndarray:
        """Scales of expert e as float64 (bf16 bit patterns are widened exactly)."""
        s = arr[e]
        return rawint4.bf16_bits_to_f64(s) if s.dtype == np.uint16 else s

    def dense(self, e: int):
        """Dense float64 W_g, W_u [I, H] and W_d [H, I] of expert e."""
        if self.weight_format == "mxfp4":
            return (mxfp4.dequantize_mxfp4(self.gate_q[e], self.gate_s[e]),
                    mxfp4.dequantize_mxfp4(self.up_q[e], self.up_s[e]),
                    mxfp4.dequantize_mxfp4(self.down_q[e], self.down_s[e]))
        if self.weight_format != "rawint4":
            raise ValueError(f"unknown weight format {self.weight_format!r}")
        return (rawint4.dequantize_rawint4(self.gate_q[e], self._scale(self.gate_s, e)),
                rawint4.dequantize_rawint4(self.up_q[e], self._scale(self.up_s, e)),
                rawint4.dequantize_rawint4(self.down_q[e], self._scale(self.down_s, e)))


# ---------------------------------------------------------------------------
# Permutation (stable counting sort of the flat slot index by expert)
# ---------------------------------------------------------------------------

def stable_expert_permutation(expert_ids: np.ndarray, experts: int):
    """Histogram -> exclusive prefix sum -> stable scatter.

    Returns counts [E], offsets [E+1] (offsets[e] = first permuted row of
    expert e), perm [n_valid] (permuted row p -> flat slot f = t*k + s) and
    inv [Q*k] (flat slot -> permuted row, -1 for ids outside [0, E)).
    """
    ids = np.asarray(expert_ids, dtype=np.int64).reshape(-1)
    counts = np.zeros(experts, dtype=np.int64)
    for e in ids:
        if 0 <= e < experts:
            counts[e] += 1
    offsets = np.zeros(experts + 1, dtype=np.int64)
    for e in range(experts):
        offsets[e + 1] = offsets[e] + counts[e]
    cursor = offsets[:-1].copy()
    perm = np.zeros(int(offsets[-1]), dtype=np.int64)
    inv = np.full(ids.shape[0], -1, dtype=np.int64)
    for f, e in enumerate(ids):
        if 0 <= e < experts:
            perm[cursor[e]] = f
            inv[f] = cursor[e]
            cursor[e] += 1
    return counts, offsets, perm, inv


# ---------------------------------------------------------------------------
# SwiGLU with the optional clamp (rawint4_sft_reference.py, rawint4_swiglu)
# ---------------------------------------------------------------------------

def sigmoid(z: np.ndarray) -> np.ndarray:
    """1 / (1 + exp(-z)); exp overflow for very negative z gives exactly 0."""
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-np.asarray(z, dtype=np.float64)))


def clamp_preacts(G: np.ndarray, U: np.ndarray, limit: float):
    """Clamp (gate upper-only, up both sides) and the gradient-pass masks."""
    if limit > 0:
        Gc = np.where(G <= limit, G, limit)
        Uc = np.where(U < -limit, -limit, np.where(U > limit, limit, U))
        mask_g = G <= limit
        mask_u = (U >= -limit) & (U <= limit)
    else:
        Gc, Uc = G, U
        mask_g = np.ones(G.shape, dtype=bool)
        mask_u = np.ones(U.shape, dtype=bool)
    return Gc, Uc, mask_g, mask_u


def swiglu(G: np.ndarray, U: np.ndarray, limit: float) -> np.ndarray:
    Gc, Uc, _, _ = clamp_preacts(G, U, limit)
    return Gc * sigmoid(Gc) * Uc


def swiglu_backward(G: np.ndarray, U: np.ndarray, dh: np.ndarray, limit: float, masks=None):
    """d/dG and d/dU of h = silu(G') U' given dh (subgradient 1 on the bounds).

    ``masks`` = (pass_g, pass_u) replaces the clamp's own gradient-pass
    decisions (used to check a GPU result whose pre-activation landed on the
    other side of a bound within its fp32 accumulation error)."""
    Gc, Uc, mask_g, mask_u = clamp_preacts(G, U, limit)
    if masks is not None:
        mask_g, mask_u = masks
    sg = sigmoid(Gc)
    silu = Gc * sg
    dsilu = sg * (1.0 + Gc * (1.0 - sg))
    dG = np.where(mask_g, dh * Uc * dsilu, 0.0)
    dU = np.where(mask_u, dh * silu, 0.0)
    return dG, dU


# ---------------------------------------------------------------------------
# Forward (per-expert loop over the equation of routed_rawint4_lora)
# ---------------------------------------------------------------------------

@dataclass
class ExpertCtx:
    slots: np.ndarray  # flat slot indices f of the expert's rows, ascending
    tokens: np.ndarray  # f // top_k
    w: np.ndarray  # route weight per row
    X: np.ndarray  # [M, H]
    G: np.ndarray  # [M, I]
    U: np.ndarray
    h: np.ndarray
    y: np.ndarray  # [M, H], unweighted expert output


@dataclass
class Ctx:
    qlen: int
    top_k: int
    experts: Dict[int, ExpertCtx] = field(default_factory=dict)


def _expert_rows(ids_flat: np.ndarray, e: int) -> np.ndarray:
    return np.nonzero(ids_flat == e)[0]


def forward(layer: Layer, x, expert_ids, route_weights, experts: Optional[Iterable[int]] = None):
    """Routed forward. ``experts`` restricts the sum to a subset (sampling).

    Returns (out float64 [Q, H], ctx for ``backward``).
    """
    x = np.asarray(x, dtype=np.float64)
    ids = np.asarray(expert_ids, dtype=np.int64)
    rw = np.asarray(route_weights, dtype=np.float64)
    Q, k = ids.shape
    if x.shape != (Q, layer.hidden) or rw.shape != ids.shape:
        raise ValueError("inputs and routing tensors disagree on shapes")
    c = layer.scaling
    L = layer.swiglu_limit
    ids_flat = ids.reshape(-1)
    out = np.zeros((Q, layer.hidden), dtype=np.float64)
    ctx = Ctx(Q, k)
    todo = range(layer.experts) if experts is None else sorted(set(int(e) for e in experts))
    for e in todo:
        slots = _expert_rows(ids_flat, e)
        if slots.size == 0:
            continue
        tokens = slots // k
        w = rw.reshape(-1)[slots]
        X = x[tokens]
        Wg, Wu, Wd = layer.dense(e)
        lo = {n: layer.lora[n][e] for n in LORA_NAMES}
        G = X @ Wg.T + c * (X @ lo["gate_lora_a"].T) @ lo["gate_lora_b"].T
        U = X @ Wu.T + c * (X @ lo["up_lora_a"].T) @ lo["up_lora_b"].T
        h = swiglu(G, U, L)
        y = h @ Wd.T + c * (h @ lo["down_lora_a"].T) @ lo["down_lora_b"].T
        np.add.at(out, tokens, w[:, None] * y)
        ctx.experts[e] = ExpertCtx(slots, tokens, w, X, G, U, h, y)
    return out, ctx


def forward_token_loop(layer: Layer, x, expert_ids, route_weights):
    """Second forward: the page's per-token, per-slot loop (tiny shapes only)."""
    x = np.asarray(x, dtype=np.float64)
    ids = np.asarray(expert_ids, dtype=np.int64)
    rw = np.asarray(route_weights, dtype=np.float64)
    c = layer.scaling
    dense = {}
    out = np.zeros((ids.shape[0], layer.hidden), dtype=np.float64)
    for t in range(ids.shape[0]):
        xt = x[t]
        for s in range(ids.shape[1]):
            e = int(ids[t, s])
            if not 0 <= e < layer.experts:
                continue
            if e not in dense:
                dense[e] = layer.dense(e)
            Wg, Wu, Wd = dense[e]
            lo = {n: layer.lora[n][e] for n in LORA_NAMES}
            g = Wg @ xt + c * lo["gate_lora_b"] @ (lo["gate_lora_a"] @ xt)
            u = Wu @ xt + c * lo["up_lora_b"] @ (lo["up_lora_a"] @ xt)
            h = swiglu(g, u, layer.swiglu_limit)
            y = Wd @ h + c * lo["down_lora_b"] @ (lo["down_lora_a"] @ h)
            out[t] += rw[t, s] * y
    return out


# ---------------------------------------------------------------------------
# Backward (hand-derived chain rule of the forward above)
# ---------------------------------------------------------------------------

def backward(layer: Layer, ctx: Ctx, grad_out, transpose_free: bool = False, masks=None):
    """Gradients of sum(grad_out * out) w.r.t. x, route weights and the LoRA tensors.

    Per expert, with g = grad_out rows, dy = w g, c = alpha / rank:
      dRoute = <g, y>                      (y = unweighted expert output)
      gd     = dy B_d                      dh = dy W_d + c gd A_d
      dB_d   = c dy^T (h A_d^T)            dA_d = c gd^T h
      dG, dU = SwiGLU backward of dh (clamp masks on the unrounded G, U)
      dx     = dG W_g + dU W_u + c (dG B_g) A_g + c (dU B_u) A_u
      dB_g   = c dG^T (X A_g^T)            dA_g = c (dG B_g)^T X      (same for up)
    LoRA gradients are raw sums over this call (unscaled by grad_scale).
    ``transpose_free`` computes the base part of dh and dx with the
    group-at-a-time loop of oracle.rawint4 instead of the dense matrix.
    ``masks`` maps an expert to (pass_g, pass_u) boolean [M, I] arrays (rows in
    the order of its ExpertCtx) that replace the clamp's own decisions.
    """
    g_all = np.asarray(grad_out, dtype=np.float64)
    Q, k = ctx.qlen, ctx.top_k
    c = layer.scaling
    L = layer.swiglu_limit
    E, H, I, r = layer.experts, layer.hidden, layer.inter, layer.rank
    grad_in = np.zeros((Q, H), dtype=np.float64)
    grad_route = np.zeros(Q * k, dtype=np.float64)
    shapes = {"gate_lora_a": (E, r, H), "gate_lora_b": (E, I, r), "up_lora_a": (E, r, H),
              "up_lora_b": (E, I, r), "down_lora_a": (E, r, I), "down_lora_b": (E, H, r)}
    grads = {n: np.zeros(s, dtype=np.float64) for n, s in shapes.items()}
    for e, ec in ctx.experts.items():
        lo = {n: layer.lora[n][e] for n in LORA_NAMES}
        Wg, Wu, Wd = layer.dense(e)
        g = g_all[ec.tokens]
        grad_route[ec.slots] = np.sum(g * ec.y, axis=1)
        dy = ec.w[:, None] * g
        gd = dy @ lo["down_lora_b"]
        if transpose_free and layer.weight_format != "rawint4":
            raise ValueError("the transpose-free loop is written for RAWINT4 storage")
        if transpose_free:
            dh_base = rawint4.transpose_free_dx(dy, layer.down_q[e], Layer._scale(layer.down_s, e))
        else:
            dh_base = dy @ Wd
        dh = dh_base + c * gd @ lo["down_lora_a"]
        grads["down_lora_b"][e] = c * dy.T @ (ec.h @ lo["down_lora_a"].T)
        grads["down_lora_a"][e] = c * gd.T @ ec.h
        dG, dU = swiglu_backward(ec.G, ec.U, dh, L, None if masks is None else masks.get(e))
        gb_g = dG @ lo["gate_lora_b"]
        gb_u = dU @ lo["up_lora_b"]
        if transpose_free:
            dx = (rawint4.transpose_free_dx(dG, layer.gate_q[e], Layer._scale(layer.gate_s, e))
                  + rawint4.transpose_free_dx(dU, layer.up_q[e], Layer._scale(layer.up_s, e)))
        else:
            dx = dG @ Wg + dU @ Wu
        dx = dx + c * gb_g @ lo["gate_lora_a"] + c * gb_u @ lo["up_lora_a"]
        np.add.at(grad_in, ec.tokens, dx)
        grads["gate_lora_b"][e] = c * dG.T @ (ec.X @ lo["gate_lora_a"].T)
        grads["gate_lora_a"][e] = c * gb_g.T @ ec.X
        grads["up_lora_b"][e] = c * dU.T @ (ec.X @ lo["up_lora_a"].T)
        grads["up_lora_a"][e] = c * gb_u.T @ ec.X
    return grad_in, grad_route.reshape(Q, k), grads


# ---------------------------------------------------------------------------
# Authoritative gradient window (test_rawint4_sft_numerical.py)
# ---------------------------------------------------------------------------

def grad_window(prev: Optional[Dict[str, np.ndarray]], grads: Dict[str, np.ndarray],
                accumulate: bool, grad_scale: float) -> Dict[str, np.ndarray]:
    """buf = (accumulate ? prev : 0) + grad_scale * grads.

    ``grads`` is zero on experts that no slot of the call reached, so such
    rows are cleared by an overwriting call and kept by an accumulating one.
    """
    out = {}
    for n, gval in grads.items():
        base = np.asarray(prev[n], dtype=np.float64) if (accumulate and prev is not None) else 0.0
        out[n] = base + grad_scale * gval
    return out


def active_experts(expert_ids, experts: int) -> List[int]:
    ids = np.asarray(expert_ids, dtype=np.int64).reshape(-1)
    return sorted({int(e) for e in ids if 0 <= e < experts})
