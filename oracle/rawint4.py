"""RAWINT4 storage format, restated from ``rawint4_sft_reference.py``.

Test infrastructure only (see the package header).

Format (module docstring and ``unpack_rawint4`` of rawint4_sft_reference.py;
``get_rawint4_checkpoint_contract`` of backend.py): every byte holds two
4-bit codes, the LOW nibble first. A code c in 0..15 stands for the signed
value c - 8 in [-8, 7]. One bf16 scale multiplies each run of 32 consecutive
input features of a row; there is no zero point. A projection with N output
rows and K input features is stored as ``uint8 [N, K/2]`` plus scales
``bf16 [N, K/32]``.

Pins (tests/test_oracle_rawint4.py): the page fixtures 0x00 -> (-8, -8),
0xFF -> (7, 7), 0x99 -> (1, 1), 0x77 -> (-1, -1); pack/unpack round trip over
all 256 bytes; zero scale -> zero weights; dense dequantisation against the
group-at-a-time transpose-free dX; the fp32 product exactness argument.
"""

from __future__ import annotations

import numpy as np

GROUP = 32


# ---------------------------------------------------------------------------
# bf16 <-> float helpers (plain IEEE definitions)
# ---------------------------------------------------------------------------

def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float32, exact (bf16 is the top half of fp32)."""
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(bits).astype(np.float64)


def f32_to_bf16_bits(values: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest, ties to even.

    Keeps the top 16 bits after adding half an ulp of bf16, plus one when the
    kept part is odd (the tie case). NaNs become a quiet NaN.
    """
    f = np.ascontiguousarray(values, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    rounded = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(f)
    if nan.any():
        rounded = rounded.copy()
        rounded[nan] = np.uint16(0x7FC0)
    return rounded


# ---------------------------------------------------------------------------
# Layout validation (rawint4_sft_reference.py, _validate_rawint4_layout)
# ---------------------------------------------------------------------------

def validate_layout(packed: np.ndarray, scales: np.ndarray, group_size: int = GROUP):
    if group_size != GROUP:
        raise ValueError(f"RAWINT4 requires group_size={GROUP}, got {group_size}")
    if packed.dtype != np.uint8 or packed.ndim != 2:
        raise ValueError("packed RAWINT4 weights must be a rank-2 uint8 array")
    if scales.ndim != 2:
        raise ValueError("RAWINT4 scales must be a rank-2 array")
    n, packed_k = packed.shape
    k = 2 * packed_k
    if k % group_size:
        raise ValueError(f"RAWINT4 K={k} must be divisible by group_size={group_size}")
    if tuple(scales.shape) != (n, k // group_size):
        raise ValueError(f"RAWINT4 scales have shape {tuple(scales.shape)}, expected {(n, k // group_size)}")
    return n, k


# ---------------------------------------------------------------------------
# Codes (rawint4_sft_reference.py, unpack_rawint4 / pack_rawint4_codes)
# ---------------------------------------------------------------------------

def unpack_rawint4(packed: np.ndarray) -> np.ndarray:
    """Bytes -> signed values in [-8, 7]; element 2j is the low nibble of byte j."""
    packed = np.asarray(packed)
    if packed.dtype != np.uint8:
        raise ValueError("packed RAWINT4 storage must be uint8")
    low = (packed & 0x0F).astype(np.int16)
    high = (packed >> 4).astype(np.int16)
    out = np.empty(packed.shape[:-1] + (2 * packed.shape[-1],), dtype=np.int16)
    out[..., 0::2] = low
    out[..., 1::2] = high
    return (out - 8).astype(np.int8)


def pack_rawint4_codes(codes: np.ndarray) -> np.ndarray:
    """Codes in [0, 15] -> bytes, keeping the low-nibble-first order."""
    codes = np.asarray(codes)
    if codes.ndim < 1 or codes.shape[-1] % 2:
        raise ValueError("an odd number of codes cannot be packed two per byte")
    if codes.size and (codes.min() < 0 or codes.max() > 15):
        raise ValueError("a code outside 0..15 does not fit in one nibble")
    c = codes.astype(np.uint8)
    return np.ascontiguousarray(c[..., 0::2] | (c[..., 1::2] << 4))


# ---------------------------------------------------------------------------
# Dequantisation (rawint4_sft_reference.py, dequantize_rawint4)
# ---------------------------------------------------------------------------

def dequantize_rawint4(packed: np.ndarray, scales_f64: np.ndarray) -> np.ndarray:
    """Dense float64 [N, K] matrix: (code - 8) * scale of the element's group."""
    n, k = validate_layout(packed, scales_f64)
    values = unpack_rawint4(packed).astype(np.float64)
    return values * np.repeat(np.asarray(scales_f64, dtype=np.float64), GROUP, axis=1)


def decode_f32(packed: np.ndarray, scale_bits: np.ndarray) -> np.ndarray:
    """(code - 8) * scale evaluated in float32.

    The product of a value in [-8, 7] (at most 4 significant bits) and a bf16
    scale (8 significant bits) has at most 12 significant bits, so the float32
    product is exact whenever it is a normal number; this is the reference
    for a bit-exact decode check.
    """
    validate_layout(packed, scale_bits)
    values = unpack_rawint4(packed).astype(np.float32)
    s = np.repeat(bf16_bits_to_f32(scale_bits), GROUP, axis=1)
    return (values * s).astype(np.float32)


def decode_bf16_bits(packed: np.ndarray, scale_bits: np.ndarray) -> np.ndarray:
    """The decoded weight rounded once to bf16 (RNE of the exact product)."""
    return f32_to_bf16_bits(decode_f32(packed, scale_bits))


# ---------------------------------------------------------------------------
# Transpose-free dX (rawint4_sft_reference.py, transpose_free_rawint4_dx)
# ---------------------------------------------------------------------------

def transpose_free_dx(grad_output: np.ndarray, packed: np.ndarray, scales_f64: np.ndarray) -> np.ndarray:
    """dX = dY @ W using only stored rows, one 32-wide group at a time.

    For every K group, walk the stored output rows n, decode that row's 32
    values of the group and add dY[:, n] times them into the group's slice of
    dX. No transposed or dense copy of W is formed.
    """
    n, k = validate_layout(packed, scales_f64)
    dy = np.asarray(grad_output, dtype=np.float64)
    if dy.ndim != 2 or dy.shape[1] != n:
        raise ValueError(f"grad_output must have shape [M, {n}], got {dy.shape}")
    dx = np.zeros((dy.shape[0], k), dtype=np.float64)
    half = GROUP // 2
    for group in range(k // GROUP):
        k0 = group * GROUP
        for row in range(n):
            codes = packed[row, group * half:(group + 1) * half]
            vals = np.empty(GROUP, dtype=np.float64)
            vals[0::2] = (codes & 0x0F).astype(np.float64) - 8.0
            vals[1::2] = (codes >> 4).astype(np.float64) - 8.0
            vals *= float(scales_f64[row, group])
            dx[:, k0:k0 + GROUP] += dy[:, row:row + 1] * vals[None, :]
    return dx
