"""ctypes binding of librawint4_moe.so (include/rawint4_moe.h).

Argument marshalling only: torch tensors are passed as raw device pointers,
every computation happens in the library's CUDA kernels. There is no CPU
fallback: importing this module fails loudly when the library is missing.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Dict, Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librawint4_moe.so")

OK = 0
INVALID_ARGUMENT = 1
FROZEN_BASE = 2
NO_SAVED_FORWARD = 3
CUDA_ERROR = 4
BAD_EXPERT_ID = 5
DEVICE_TIMEOUT = 6
FP16_OVERFLOW = 7
UNSUPPORTED = 8
STATIC_SCRATCH_TOO_SMALL = 9

DEV_BAD_EXPERT_ID = 1 << 0
DEV_NO_SAVED_FORWARD = 1 << 1
DEV_TIMEOUT = 1 << 2
DEV_FP16_OVERFLOW = 1 << 3

EXPORTED_SYMBOLS = (
    "rawint4_moe_lora_workspace_size",
    "rawint4_moe_lora_fwd",
    "rawint4_moe_lora_bwd",
    "rawint4_moe_lora_status",
    "rawint4_moe_lora_strerror",
    "rawint4_decode",
    "rawint4_moe_permute_workspace_size",
    "rawint4_moe_permute",
    "rawint4_moe_profile_begin",
    "rawint4_moe_profile_end",
    "rawint4_moe_permute_static",
    "rawint4_moe_permute_static_max_bytes",
    "rawint4_moe_set_wait_limit_ns",
    "rawint4_moe_lora_saved_preacts",
    "rawint4_moe_router_topk",
    "rawint4_moe_router_bwd",
    "rawint4_mxfp4_decode",
    "rawint4_moe_dispatch_rows",
    "rawint4_moe_combine_slots",
    "rawint4_moe_gather_slots",
)


class Cfg(ctypes.Structure):
    _fields_ = [("experts", ctypes.c_int32), ("top_k", ctypes.c_int32), ("hidden", ctypes.c_int32),
                ("inter", ctypes.c_int32), ("rank", ctypes.c_int32), ("alpha", ctypes.c_float),
                ("swiglu_limit", ctypes.c_float), ("max_tokens", ctypes.c_int32), ("weight_format", ctypes.c_int32)]


class Base(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("gate_q", "up_q", "down_q", "gate_s", "up_s", "down_s")]


class Lora(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("gate_a", "gate_b", "up_a", "up_b", "down_a", "down_b")]


class LoraGrads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("gate_a", "gate_b", "up_a", "up_b", "down_a", "down_b")]


class RawInt4Error(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {strerror(code)} (code {code})")


class FrozenBaseError(RawInt4Error, ValueError):
    pass


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m int4_quantised_moe_b200.build` "
            "(the layer has no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, sz, i32, i64, f32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
    P = ctypes.POINTER
    lib.rawint4_moe_lora_workspace_size.argtypes = [P(Cfg), P(sz)]
    lib.rawint4_moe_lora_fwd.argtypes = [P(Cfg), P(Base), P(Lora), i32, vp, vp, vp, vp, ctypes.c_int, vp, sz, vp]
    lib.rawint4_moe_lora_bwd.argtypes = [P(Cfg), P(Base), P(Lora), vp, vp, vp, P(LoraGrads), vp, vp, vp,
                                         ctypes.c_int, f32, vp, sz, vp]
    lib.rawint4_moe_lora_status.argtypes = [vp, vp, P(ctypes.c_uint32)]
    lib.rawint4_moe_lora_strerror.argtypes = [ctypes.c_int]
    lib.rawint4_moe_lora_strerror.restype = ctypes.c_char_p
    lib.rawint4_decode.argtypes = [vp, vp, i64, i64, vp, vp, vp]
    lib.rawint4_moe_permute_workspace_size.argtypes = [i32, i32, i32, P(sz)]
    lib.rawint4_moe_permute.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp, sz, vp]
    lib.rawint4_moe_permute_static.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp]
    lib.rawint4_moe_permute_static_max_bytes.argtypes = []
    lib.rawint4_moe_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.rawint4_moe_lora_saved_preacts.argtypes = [P(Cfg), vp, sz, vp, vp, vp, P(i32), vp]
    lib.rawint4_moe_router_topk.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp]
    lib.rawint4_moe_router_bwd.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp, vp, vp]
    lib.rawint4_mxfp4_decode.argtypes = [vp, vp, i64, i64, vp, vp, vp]
    lib.rawint4_moe_dispatch_rows.argtypes = [vp, vp, i32, i32, i32, vp, vp]
    lib.rawint4_moe_combine_slots.argtypes = [vp, vp, i32, i32, i32, vp, vp]
    lib.rawint4_moe_gather_slots.argtypes = [vp, vp, i32, vp, vp]
    for name in EXPORTED_SYMBOLS:
        if name != "rawint4_moe_lora_strerror":
            getattr(lib, name).restype = ctypes.c_int  # raises AttributeError if the library lacks it
    lib.rawint4_moe_permute_static_max_bytes.restype = ctypes.c_size_t
    return lib


_lib = _load()


def library() -> ctypes.CDLL:
    return _lib


def strerror(code: int) -> str:
    return _lib.rawint4_moe_lora_strerror(int(code)).decode()


def _check(code: int, what: str):
    if code == FROZEN_BASE:
        raise FrozenBaseError(code, what)
    if code != OK:
        raise RawInt4Error(code, what)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to the layer must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


FORMAT_RAWINT4 = 0
FORMAT_MXFP4 = 1
FORMATS = {"rawint4": FORMAT_RAWINT4, "mxfp4": FORMAT_MXFP4}


def make_cfg(experts, top_k, hidden, inter, rank, alpha, swiglu_limit, max_tokens, weight_format="rawint4") -> Cfg:
    return Cfg(int(experts), int(top_k), int(hidden), int(inter), int(rank), float(alpha), float(swiglu_limit),
               int(max_tokens), FORMATS[weight_format])


def rawint4_moe_lora_workspace_size(cfg: Cfg) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.rawint4_moe_lora_workspace_size(ctypes.byref(cfg), ctypes.byref(n)), "rawint4_moe_lora_workspace_size")
    return int(n.value)


def make_base(gate_q, gate_s, up_q, up_s, down_q, down_s) -> Base:
    return Base(_ptr(gate_q), _ptr(up_q), _ptr(down_q), _ptr(gate_s), _ptr(up_s), _ptr(down_s))


def make_lora(lora: Dict[str, torch.Tensor]) -> Lora:
    return Lora(*[_ptr(lora[n]) for n in ("gate_lora_a", "gate_lora_b", "up_lora_a", "up_lora_b",
                                          "down_lora_a", "down_lora_b")])


def make_grads(grads: Dict[str, torch.Tensor]) -> LoraGrads:
    return LoraGrads(*[_ptr(grads[n]) for n in ("gate_lora_a", "gate_lora_b", "up_lora_a", "up_lora_b",
                                                "down_lora_a", "down_lora_b")])


def rawint4_moe_lora_fwd(cfg: Cfg, base: Base, lora: Optional[Lora], qlen: int, expert_ids, route_weights, x, out,
                         save_for_backward: bool, workspace: torch.Tensor, stream=None) -> None:
    """lora=None: frozen-base inference forward (save_for_backward must be False)."""
    lora_ref = ctypes.byref(lora) if lora is not None else None
    rc = _lib.rawint4_moe_lora_fwd(ctypes.byref(cfg), ctypes.byref(base), lora_ref, int(qlen),
                                   _ptr(expert_ids), _ptr(route_weights), _ptr(x), _ptr(out),
                                   1 if save_for_backward else 0, _ptr(workspace), workspace.numel(),
                                   _stream(stream))
    _check(rc, "rawint4_moe_lora_fwd")


def rawint4_moe_lora_bwd(cfg: Cfg, base: Base, lora: Lora, grad_out, grad_in, grad_route, grads: LoraGrads,
                         accumulate: bool, grad_scale: float, workspace: torch.Tensor, stream=None,
                         base_grad_gate=None, base_grad_up=None, base_grad_down=None) -> None:
    rc = _lib.rawint4_moe_lora_bwd(ctypes.byref(cfg), ctypes.byref(base), ctypes.byref(lora), _ptr(grad_out),
                                   _ptr(grad_in), _ptr(grad_route), ctypes.byref(grads), _ptr(base_grad_gate),
                                   _ptr(base_grad_up), _ptr(base_grad_down), 1 if accumulate else 0,
                                   float(grad_scale), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "rawint4_moe_lora_bwd")


def rawint4_moe_lora_status(workspace: torch.Tensor, stream=None) -> int:
    v = ctypes.c_uint32(0)
    _check(_lib.rawint4_moe_lora_status(_ptr(workspace), _stream(stream), ctypes.byref(v)), "rawint4_moe_lora_status")
    return int(v.value)


def rawint4_decode(q: torch.Tensor, s: torch.Tensor, out_f32=None, out_f16=None, stream=None) -> None:
    n, k2 = q.shape[-2], q.shape[-1]
    rows = q.numel() // k2
    _check(_lib.rawint4_decode(_ptr(q), _ptr(s), rows, 2 * k2, _ptr(out_f32), _ptr(out_f16), _stream(stream)),
           "rawint4_decode")


def rawint4_mxfp4_decode(q: torch.Tensor, s: torch.Tensor, out_f32=None, out_f16=None, stream=None) -> None:
    """MXFP4 check decode: q uint8 [N, K/2], s uint8 [N, K/32] -> fp32 and/or fp16 [N, K]."""
    k2 = q.shape[-1]
    rows = q.numel() // k2
    _check(_lib.rawint4_mxfp4_decode(_ptr(q), _ptr(s), rows, 2 * k2, _ptr(out_f32), _ptr(out_f16), _stream(stream)),
           "rawint4_mxfp4_decode")


def rawint4_moe_permute(expert_ids: torch.Tensor, experts: int, offsets, perm, inv, stream=None) -> None:
    q, k = expert_ids.shape
    n = ctypes.c_size_t(0)
    _check(_lib.rawint4_moe_permute_workspace_size(q, k, experts, ctypes.byref(n)), "permute_workspace_size")
    ws = torch.empty(max(int(n.value), 256), dtype=torch.uint8, device=expert_ids.device)
    _check(_lib.rawint4_moe_permute(_ptr(expert_ids), q, k, experts, _ptr(offsets), _ptr(perm), _ptr(inv),
                                    _ptr(ws), ws.numel(), _stream(stream)), "rawint4_moe_permute")


def rawint4_moe_permute_static(expert_ids: torch.Tensor, experts: int, offsets, perm, inv, stream=None) -> None:
    """rawint4_moe_permute without caller scratch: for callers that cannot
    allocate device memory; uses the library's fixed 1 MiB device array."""
    q, k = expert_ids.shape
    _check(_lib.rawint4_moe_permute_static(_ptr(expert_ids), q, k, experts, _ptr(offsets), _ptr(perm), _ptr(inv),
                                           _stream(stream)), "rawint4_moe_permute_static")


def rawint4_moe_permute_static_max_bytes() -> int:
    return int(_lib.rawint4_moe_permute_static_max_bytes())


def rawint4_moe_dispatch_rows(src: torch.Tensor, perm: torch.Tensor, n: int, top_k: int, dst: torch.Tensor,
                              stream=None) -> None:
    """dst[p] = src[perm[p] // top_k] for p < n (bf16 rows)."""
    _require(src, torch.bfloat16, src.device, "src")
    _require(dst, torch.bfloat16, src.device, "dst")
    _require(perm, torch.int32, src.device, "perm")
    if dst.shape[0] < n or dst.shape[1] != src.shape[1] or perm.numel() < n:
        raise ValueError("dispatch_rows: dst must hold n rows of src's width and perm n entries")
    _check(_lib.rawint4_moe_dispatch_rows(_ptr(src), _ptr(perm), int(n), int(top_k), src.shape[1], _ptr(dst),
                                          _stream(stream)), "rawint4_moe_dispatch_rows")


def rawint4_moe_combine_slots(src: torch.Tensor, inv: torch.Tensor, qlen: int, top_k: int, out: torch.Tensor,
                              stream=None) -> None:
    """out[t] = bf16(sum over s of src[inv[t * top_k + s]]) in slot order (fp32 sums)."""
    _require(out, torch.bfloat16, out.device, "out")
    _require(inv, torch.int32, out.device, "inv")
    if src.numel():
        _require(src, torch.bfloat16, out.device, "src")
        if src.shape[1] != out.shape[1]:
            raise ValueError("combine_slots: src and out widths differ")
    if out.shape[0] < qlen or inv.numel() < qlen * top_k:
        raise ValueError("combine_slots: out needs qlen rows and inv qlen * top_k entries")
    _check(_lib.rawint4_moe_combine_slots(_ptr(src) if src.numel() else None, _ptr(inv), int(qlen), int(top_k),
                                          out.shape[1], _ptr(out), _stream(stream)), "rawint4_moe_combine_slots")


def rawint4_moe_gather_slots(src: torch.Tensor, inv: torch.Tensor, out: torch.Tensor, stream=None) -> None:
    """out[f] = src[inv[f]] where inv[f] >= 0, else 0 (fp32)."""
    _require(out, torch.float32, out.device, "out")
    _require(inv, torch.int32, out.device, "inv")
    if src.numel():
        _require(src, torch.float32, out.device, "src")
    if inv.numel() < out.numel():
        raise ValueError("gather_slots: inv needs one entry per output")
    _check(_lib.rawint4_moe_gather_slots(_ptr(src) if src.numel() else None, _ptr(inv), out.numel(), _ptr(out),
                                         _stream(stream)), "rawint4_moe_gather_slots")


# ---------------------------------------------------------------------------
# Convenience holder used by tests and the bench: keeps the layer's tensors
# and one workspace together and calls the two entry points.
# ---------------------------------------------------------------------------

def _require(t, dtype: torch.dtype, device: torch.device, name: str) -> None:
    """Like _expect, without a fixed shape."""
    _expect(t, name, dtype, tuple(t.shape) if isinstance(t, torch.Tensor) else (), device)


def _expect(t, name: str, dtype: torch.dtype, shape: tuple, device: Optional[torch.device] = None) -> None:
    """Host-side argument check: the C ABI sees raw pointers only, so a wrong
    dtype, shape, device or layout is caught here with a readable message."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected dtype {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_cuda:
        raise ValueError(f"{name}: expected a CUDA tensor, got one on {t.device}")
    if device is not None and t.device != device:
        raise ValueError(f"{name}: expected a tensor on {device}, got one on {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: tensors passed to the layer must be contiguous")


LORA_TENSOR_NAMES = ("gate_lora_a", "gate_lora_b", "up_lora_a", "up_lora_b", "down_lora_a", "down_lora_b")


def lora_tensor_shapes(experts: int, hidden: int, inter: int, rank: int) -> Dict[str, tuple]:
    """Shapes of the six LoRA tensors (and of their gradient buffers)."""
    E, H, I, r = experts, hidden, inter, rank
    return {"gate_lora_a": (E, r, H), "gate_lora_b": (E, I, r), "up_lora_a": (E, r, H), "up_lora_b": (E, I, r),
            "down_lora_a": (E, r, I), "down_lora_b": (E, H, r)}

@dataclass
class Layer:
    cfg: Cfg
    base: Base
    lora: Lora
    workspace: torch.Tensor
    keep: tuple  # tensors whose pointers live in base/lora

    @classmethod
    def create(cls, experts, top_k, hidden, inter, rank, alpha, swiglu_limit, max_tokens, gate_q, gate_s, up_q, up_s,
               down_q, down_s, lora: Dict[str, torch.Tensor], device=None, weight_format="rawint4"):
        """weight_format "rawint4" (bf16 scales) or "mxfp4" (E2M1 codes, UE8M0 scale bytes, uint8)."""
        cfg = make_cfg(experts, top_k, hidden, inter, rank, alpha, swiglu_limit, max_tokens, weight_format)
        nbytes = rawint4_moe_lora_workspace_size(cfg)  # validates the configuration
        dev = device if device is not None else gate_q.device
        E, H, I = int(experts), int(hidden), int(inter)
        sdt = torch.uint8 if weight_format == "mxfp4" else torch.bfloat16
        for name, t, dt, shape in (("gate_q", gate_q, torch.uint8, (E, I, H // 2)),
                                   ("up_q", up_q, torch.uint8, (E, I, H // 2)),
                                   ("down_q", down_q, torch.uint8, (E, H, I // 2)),
                                   ("gate_s", gate_s, sdt, (E, I, H // 32)),
                                   ("up_s", up_s, sdt, (E, I, H // 32)),
                                   ("down_s", down_s, sdt, (E, H, I // 32))):
            _expect(t, name, dt, shape, gate_q.device)
        for name, shape in lora_tensor_shapes(E, H, I, int(rank)).items():
            if name not in lora:
                raise KeyError(f"lora: missing {name}")
            _expect(lora[name], name, torch.bfloat16, shape, gate_q.device)
        ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        ws[:256].zero_()
        base = make_base(gate_q, gate_s, up_q, up_s, down_q, down_s)
        lo = make_lora(lora)
        return cls(cfg, base, lo, ws, (gate_q, gate_s, up_q, up_s, down_q, down_s, dict(lora)))

    def forward(self, expert_ids, route_weights, x, out=None, save_for_backward=True, stream=None, use_lora=True):
        """use_lora=False: frozen-base inference forward (no LoRA terms, nothing saved)."""
        q, k, H = x.shape[0] if x.dim() == 2 else -1, self.cfg.top_k, self.cfg.hidden
        dev = self.workspace.device
        _expect(x, "x", torch.bfloat16, (q, H), dev)
        _expect(expert_ids, "expert_ids", torch.int64, (q, k), dev)
        _expect(route_weights, "route_weights", torch.float32, (q, k), dev)
        if out is None:
            out = torch.empty_like(x)
        _expect(out, "out", torch.bfloat16, (q, H), dev)
        rawint4_moe_lora_fwd(self.cfg, self.base, self.lora if use_lora else None, q, expert_ids, route_weights, x,
                             out, save_for_backward, self.workspace, stream)
        return out

    def backward(self, grad_out, grads: Dict[str, torch.Tensor], accumulate=False, grad_scale=1.0, grad_in=None,
                 grad_route=None, stream=None, **base_grads):
        dev = self.workspace.device
        q, k, H = grad_out.shape[0] if grad_out.dim() == 2 else -1, self.cfg.top_k, self.cfg.hidden
        _expect(grad_out, "grad_out", torch.bfloat16, (q, H), dev)
        if grad_in is None:
            grad_in = torch.empty_like(grad_out)
        _expect(grad_in, "grad_in", torch.bfloat16, (q, H), dev)
        if grad_route is not None:
            _expect(grad_route, "grad_route", torch.float32, (q, k), dev)
        c = self.cfg
        for name, shape in lora_tensor_shapes(c.experts, c.hidden, c.inter, c.rank).items():
            if name not in grads:
                raise KeyError(f"grads: missing {name}")
            _expect(grads[name], f"grads[{name}]", torch.bfloat16, shape, dev)
        rawint4_moe_lora_bwd(self.cfg, self.base, self.lora, grad_out, grad_in, grad_route, make_grads(grads),
                             accumulate, grad_scale, self.workspace, stream, **base_grads)
        return grad_in

    def status(self, stream=None) -> int:
        return rawint4_moe_lora_status(self.workspace, stream)

    def saved_preacts(self, stream=None):
        """(perm int32 [R], G fp32 [R, I], U fp32 [R, I]) of the pending saved
        forward, R = routed rows (test export; see include/rawint4_moe.h)."""
        c = self.cfg
        rows = int(c.max_tokens) * int(c.top_k)
        dev = self.workspace.device
        perm = torch.empty(rows, dtype=torch.int32, device=dev)
        g = torch.empty((rows, int(c.inter)), dtype=torch.float32, device=dev)
        u = torch.empty_like(g)
        routed = ctypes.c_int32(0)
        rc = _lib.rawint4_moe_lora_saved_preacts(ctypes.byref(self.cfg), _ptr(self.workspace), self.workspace.numel(),
                                                 _ptr(perm), _ptr(g), _ptr(u), ctypes.byref(routed), _stream(stream))
        _check(rc, "rawint4_moe_lora_saved_preacts")
        n = int(routed.value)
        return perm[:n], g[:n], u[:n]


# ---------------------------------------------------------------------------
# Timing hook (measurement only)
# ---------------------------------------------------------------------------

def router_topk(scores: torch.Tensor, top_k: int, escale: Optional[torch.Tensor] = None, stream=None):
    """Expert ids int64 [Q, k] and route weights fp32 [Q, k] from router scores fp32 [Q, E]
    (softmax, top-k, renormalised, times the per-expert scale)."""
    q, E = scores.shape
    _expect(scores, "scores", torch.float32, (q, E))
    if escale is not None:
        _expect(escale, "escale", torch.float32, (E,), scores.device)
    ids = torch.empty((q, int(top_k)), dtype=torch.int64, device=scores.device)
    w = torch.empty((q, int(top_k)), dtype=torch.float32, device=scores.device)
    _check(_lib.rawint4_moe_router_topk(_ptr(scores), q, E, int(top_k), _ptr(escale), _ptr(ids), _ptr(w),
                                        _stream(stream)), "rawint4_moe_router_topk")
    return ids, w


def router_bwd(scores: torch.Tensor, ids: torch.Tensor, grad_route: torch.Tensor, escale: Optional[torch.Tensor] = None,
               want_escale_grad: bool = False, stream=None):
    """dL/dscores fp32 [Q, E] (and dL/descale fp32 [E]) from the layer's grad_route."""
    q, E = scores.shape
    k = ids.shape[1] if ids.dim() == 2 else -1
    _expect(scores, "scores", torch.float32, (q, E))
    _expect(ids, "ids", torch.int64, (q, k), scores.device)
    _expect(grad_route, "grad_route", torch.float32, (q, k), scores.device)
    if escale is not None:
        _expect(escale, "escale", torch.float32, (E,), scores.device)
    dz = torch.empty_like(scores)
    dc = torch.empty(E, dtype=torch.float32, device=scores.device) if want_escale_grad else None
    _check(_lib.rawint4_moe_router_bwd(_ptr(scores), q, E, k, _ptr(ids), _ptr(grad_route), _ptr(escale), _ptr(dz),
                                       _ptr(dc), _stream(stream)), "rawint4_moe_router_bwd")
    return (dz, dc) if want_escale_grad else dz


def set_wait_limit_ns(ns: int) -> None:
    """Bound on every pipeline wait of the GEMM kernels launched from now on
    (0 restores the default of 4 s); see include/rawint4_moe.h."""
    _check(_lib.rawint4_moe_set_wait_limit_ns(int(ns)), "rawint4_moe_set_wait_limit_ns")


def profile_begin(max_launches: int = 4096) -> None:
    _lib.rawint4_moe_profile_begin.argtypes = [ctypes.c_int]
    _lib.rawint4_moe_profile_begin.restype = ctypes.c_int
    _check(_lib.rawint4_moe_profile_begin(int(max_launches)), "rawint4_moe_profile_begin")


def profile_end(max_out: int = 4096):
    """Per launch in issue order: (kernel name, milliseconds)."""
    _lib.rawint4_moe_profile_end.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_int),
                                             ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_float)]
    _lib.rawint4_moe_profile_end.restype = ctypes.c_int
    n = ctypes.c_int(0)
    names = (ctypes.c_char_p * max_out)()
    ms = (ctypes.c_float * max_out)()
    _check(_lib.rawint4_moe_profile_end(max_out, ctypes.byref(n), names, ms), "rawint4_moe_profile_end")
    return [(names[i].decode(), float(ms[i])) for i in range(min(n.value, max_out))]
