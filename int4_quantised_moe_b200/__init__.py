"""B200 (sm_100a) routed RAWINT4 MoE-LoRA layer: forward and backward.

The compute path is the C-ABI library ``librawint4_moe.so`` (header
``include/rawint4_moe.h``); ``binding`` is its thin ctypes wrapper. Names of
the binding are re-exported lazily so that ``int4_quantised_moe_b200.build``
can run before the library exists; touching any of them without the library
raises ImportError (there is no CPU fallback).
"""

_EXPORTS = (
    "Layer", "RawInt4Error", "FrozenBaseError", "library", "make_base", "make_cfg", "make_grads", "make_lora",
    "rawint4_decode", "rawint4_moe_lora_bwd", "rawint4_moe_lora_fwd", "rawint4_moe_lora_status",
    "rawint4_moe_lora_workspace_size", "rawint4_moe_permute", "strerror", "profile_begin", "profile_end",
)


def __getattr__(name):
    if name in _EXPORTS:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
