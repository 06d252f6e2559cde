"""MXFP4 storage format (the sibling frozen-base format of the same layer).

Test infrastructure only (see the package header).

Format, as the pages describe it (the ``ext_bindings.cpp`` commit log:
"MXFP4 MoE operator with E2M1 weights x BF16 activations", "adapt MXFP4 MoE
backend for DeepSeek-V4-Flash", "avoid uint16 lshift in ue8m0->bf16
conversion"; ``backend.py``: weight layout ``mxfp4-e2m1-ue8m0-g32``): every
byte holds two 4-bit E2M1 codes, nibble-packed; one UE8M0 scale byte
multiplies each run of 32 consecutive input features of a row. A projection
with N output rows and K input features is stored as ``uint8 [N, K/2]`` plus
scales ``uint8 [N, K/32]``.

E2M1 (one sign bit, two exponent bits with bias 1, one mantissa bit):
    bit 3 = sign, bits 2-1 = exponent field x, bit 0 = mantissa m
    |value| = m / 2                  if x == 0   (0 or 0.5)
            = 2^(x - 1) * (1 + m/2)  if x > 0    (1, 1.5, 2, 3, 4, 6)

UE8M0 scale byte e: the loader of the pages turns it into a bf16 by placing
e in the bf16 exponent field (bit pattern e << 7, sign and mantissa zero), a
lossless bit-cast. Its value is therefore 2^(e - 127) for e in 1..254, 0 for
e == 0 and +inf for e == 255.

Readings where the pages are silent: the nibble order is low nibble first
(element 2j in the low nibble of byte j), as for RAWINT4 and as the packing
of the MX formats defines it; e == 0 and e == 255 take the values the
bit-cast gives them.

Pins (tests/test_oracle_mxfp4.py): the 16 code values against the format's
definition written independently as (-1)^s 2^x' (1 + m/2) with the
subnormal case; the scale bit-cast against 2^(e - 127) for every byte; pack
and unpack round trip over all 256 bytes; dense dequantisation against a
per-element loop.
"""

from __future__ import annotations

import numpy as np

from . import rawint4

GROUP = 32


def e2m1_value(code: int) -> float:
    """Value of one 4-bit E2M1 code (0..15), from the definition above."""
    code = int(code)
    if not 0 <= code <= 15:
        raise ValueError("an E2M1 code is four bits")
    sign = -1.0 if code & 8 else 1.0
    x = (code >> 1) & 3
    m = code & 1
    mag = m / 2.0 if x == 0 else 2.0 ** (x - 1) * (1.0 + m / 2.0)
    return sign * mag


E2M1_TABLE = np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)


def ue8m0_bf16_bits(e: np.ndarray) -> np.ndarray:
    """The pages' bit-cast of a UE8M0 byte into a bf16 bit pattern (e << 7)."""
    return (np.asarray(e, dtype=np.uint8).astype(np.uint16) << 7).astype(np.uint16)


def ue8m0_scale(e: np.ndarray) -> np.ndarray:
    """float64 value of UE8M0 scale bytes through the bf16 bit-cast."""
    return rawint4.bf16_bits_to_f64(ue8m0_bf16_bits(e))


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    """uint8 [..., K/2] -> codes uint8 [..., K], low nibble first."""
    packed = np.asarray(packed)
    if packed.dtype != np.uint8:
        raise ValueError("packed MXFP4 storage must be uint8")
    out = np.empty(packed.shape[:-1] + (2 * packed.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = packed & 0x0F
    out[..., 1::2] = packed >> 4
    return out


def pack_codes(codes: np.ndarray) -> np.ndarray:
    codes = np.asarray(codes)
    if codes.ndim < 1 or codes.shape[-1] % 2:
        raise ValueError("an odd number of codes cannot be packed two per byte")
    if codes.size and (codes.min() < 0 or codes.max() > 15):
        raise ValueError("a code outside 0..15 does not fit in one nibble")
    c = codes.astype(np.uint8)
    return np.ascontiguousarray(c[..., 0::2] | (c[..., 1::2] << 4))


def validate_layout(packed: np.ndarray, scales: np.ndarray):
    if packed.dtype != np.uint8 or packed.ndim != 2:
        raise ValueError("packed MXFP4 weights must be a rank-2 uint8 array")
    if scales.dtype != np.uint8 or scales.ndim != 2:
        raise ValueError("MXFP4 scales must be a rank-2 uint8 array")
    n, packed_k = packed.shape
    k = 2 * packed_k
    if k % GROUP:
        raise ValueError(f"MXFP4 K={k} is not a multiple of the group size {GROUP}")
    if tuple(scales.shape) != (n, k // GROUP):
        raise ValueError(f"MXFP4 scales have shape {tuple(scales.shape)}, expected {(n, k // GROUP)}")
    return n, k


def dequantize_mxfp4(packed: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Dense float64 [N, K]: E2M1 value of each code times its group's scale."""
    n, k = validate_layout(packed, scales)
    vals = E2M1_TABLE[unpack_codes(packed)]
    return vals * np.repeat(ue8m0_scale(scales), GROUP, axis=1)
