"""The C-ABI library loads and exports every entry point include/rawint4_moe.h declares (no GPU).

Only host-side argument checks run here: they return before any CUDA call.
"""

import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rawint4_moe.h")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"RAWINT4_API\s+(?:const\s+)?\w+\*?\s+(\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from int4_quantised_moe_b200 import build as b
    b.build()
    from int4_quantised_moe_b200 import binding
    return binding


def test_header_declares_expected_entry_points():
    names = _declared()
    for n in ("rawint4_moe_lora_fwd", "rawint4_moe_lora_bwd", "rawint4_moe_lora_workspace_size",
              "rawint4_moe_lora_status", "rawint4_moe_lora_strerror", "rawint4_decode", "rawint4_moe_permute"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    cdll = lib.library()
    for n in _declared():
        assert hasattr(cdll, n), n
    assert set(_declared()) <= set(lib.EXPORTED_SYMBOLS) | {"rawint4_moe_permute_workspace_size"}


def test_workspace_size_and_cfg_validation(lib):
    ok = lib.make_cfg(4, 2, 256, 256, 8, 16.0, 0.0, 32)
    n = lib.rawint4_moe_lora_workspace_size(ok)
    assert n > 0 and n % 256 == 0
    big = lib.make_cfg(4, 2, 256, 256, 8, 16.0, 0.0, 1000)
    assert lib.rawint4_moe_lora_workspace_size(big) > n
    gemma = lib.make_cfg(128, 8, 2816, 704, 8, 16.0, 0.0, 32)  # H, I multiples of 64 (not of 128)
    assert lib.rawint4_moe_lora_workspace_size(gemma) > 0
    for r in (33, 48, 64):  # ranks above 32: two rank segments and LoRA stages
        assert lib.rawint4_moe_lora_workspace_size(lib.make_cfg(4, 2, 256, 256, r, 2.0 * r, 0.0, 32)) > 0
    bad = [
        lib.make_cfg(4, 2, 200, 256, 8, 16.0, 0.0, 32),   # H not a multiple of 64
        lib.make_cfg(4, 2, 256, 96, 8, 16.0, 0.0, 32),    # I not a multiple of 64
        lib.make_cfg(4, 5, 256, 256, 8, 16.0, 0.0, 32),   # top_k > experts
        lib.make_cfg(4, 2, 256, 256, 0, 16.0, 0.0, 32),   # rank 0
        lib.make_cfg(4, 2, 256, 256, 65, 16.0, 0.0, 32),  # rank > 64
        lib.make_cfg(4, 2, 256, 256, 8, float("nan"), 0.0, 32),
        lib.make_cfg(4, 2, 256, 256, 8, 16.0, -1.0, 32),  # negative clamp limit
        lib.make_cfg(4, 2, 256, 256, 8, 16.0, float("inf"), 32),
        lib.make_cfg(4, 2, 256, 256, 8, 16.0, 0.0, 0),
    ]
    for cfg in bad:
        with pytest.raises(lib.RawInt4Error) as ei:
            lib.rawint4_moe_lora_workspace_size(cfg)
        assert ei.value.code == lib.INVALID_ARGUMENT


def test_frozen_base_rejected_before_anything_else(lib):
    """A non-null base-gradient pointer fails first, even with every other argument null."""
    cdll = lib.library()
    cfg = lib.make_cfg(4, 2, 256, 256, 8, 16.0, 0.0, 32)
    grads = lib.LoraGrads()
    rc = cdll.rawint4_moe_lora_bwd(ctypes.byref(cfg), None, None, None, None, None, ctypes.byref(grads),
                                   ctypes.c_void_p(16), None, None, 0, 1.0, None, 0, None)
    assert rc == lib.FROZEN_BASE
    assert "frozen" in lib.strerror(rc)


def test_host_argument_errors(lib):
    cdll = lib.library()
    cfg = lib.make_cfg(4, 2, 256, 256, 8, 16.0, 0.0, 32)
    base, lora = lib.Base(), lib.Lora()
    # null base / lora pointers
    rc = cdll.rawint4_moe_lora_fwd(ctypes.byref(cfg), ctypes.byref(base), ctypes.byref(lora), 5, None, None, None,
                                   None, 1, None, 0, None)
    assert rc == lib.INVALID_ARGUMENT
    v = ctypes.c_uint32(0)
    assert cdll.rawint4_moe_lora_status(None, None, ctypes.byref(v)) == lib.INVALID_ARGUMENT
    assert cdll.rawint4_decode(None, None, 4, 64, None, None, None) == lib.INVALID_ARGUMENT
    n = ctypes.c_size_t(0)
    assert cdll.rawint4_moe_permute_workspace_size(5, 2, 4, ctypes.byref(n)) == lib.OK and n.value > 0
    assert cdll.rawint4_moe_permute_workspace_size(5, 0, 4, ctypes.byref(n)) == lib.INVALID_ARGUMENT
    for code in range(0, 9):
        assert lib.strerror(code) != "unknown status code"


def test_base_only_forward_cannot_save(lib):
    """lora = NULL selects the frozen-base inference forward, which saves no
    context: save_for_backward = 1 is an argument error, and so is a backward
    without LoRA. Both are caught on the host before anything is enqueued, so
    the placeholder pointers are never dereferenced."""
    cdll = lib.library()
    cfg = lib.make_cfg(4, 2, 256, 256, 8, 16.0, 0.0, 32)
    nbytes = lib.rawint4_moe_lora_workspace_size(cfg)
    fake = 4096  # aligned, never dereferenced
    base = lib.Base(*([fake] * 6))
    rc = cdll.rawint4_moe_lora_fwd(ctypes.byref(cfg), ctypes.byref(base), None, 5, fake, fake, fake, fake, 1, fake,
                                   nbytes, None)
    assert rc == lib.INVALID_ARGUMENT
    grads = lib.LoraGrads(*([fake] * 6))
    rc = cdll.rawint4_moe_lora_bwd(ctypes.byref(cfg), ctypes.byref(base), None, fake, fake, None, ctypes.byref(grads),
                                   None, None, None, 0, 1.0, fake, nbytes, None)
    assert rc == lib.INVALID_ARGUMENT


def test_binding_rejects_wrong_tensors(lib):
    """The binding checks dtype, shape, device and layout before any C call,
    so a wrong tensor fails with a readable message instead of reaching the
    kernels as a raw pointer. Runs on CPU: every case fails before the
    workspace is allocated."""
    E, k, H, I, r = 4, 2, 256, 256, 8
    shapes = lib.lora_tensor_shapes(E, H, I, r)
    lora = {n: torch.zeros(s, dtype=torch.bfloat16) for n, s in shapes.items()}
    q = dict(gate_q=torch.zeros((E, I, H // 2), dtype=torch.uint8), gate_s=torch.zeros((E, I, H // 32), dtype=torch.bfloat16),
             up_q=torch.zeros((E, I, H // 2), dtype=torch.uint8), up_s=torch.zeros((E, I, H // 32), dtype=torch.bfloat16),
             down_q=torch.zeros((E, H, I // 2), dtype=torch.uint8), down_s=torch.zeros((E, H, I // 32), dtype=torch.bfloat16))

    def create(**over):
        a = dict(q, **over)
        return lib.Layer.create(E, k, H, I, r, 16.0, 0.0, 8, a["gate_q"], a["gate_s"], a["up_q"], a["up_s"],
                                a["down_q"], a["down_s"], over.get("lora", lora))

    with pytest.raises(ValueError, match="CUDA tensor"):
        create()
    # the first tensor checked is gate_q: dtype, then shape, then device
    with pytest.raises(TypeError, match="dtype"):
        create(gate_q=torch.zeros((E, I, H // 2), dtype=torch.int8))
    with pytest.raises(ValueError, match="shape"):
        create(gate_q=torch.zeros((E, I, H // 4), dtype=torch.uint8))
    with pytest.raises(lib.RawInt4Error):
        lib.Layer.create(E, k, 200, I, r, 16.0, 0.0, 8, *q.values(), lora)  # H not a multiple of 64
