"""Pins for oracle.rawint4 (no GPU).

Each check is tied to something outside the oracle's own formula: the byte
fixtures the contract test uses, the round trip through the packer, the
group-at-a-time transpose-free loop of rawint4_sft_reference.py, and
exactness of the fp32 product.
"""

import json
import os

import numpy as np
import pytest

from oracle import rawint4 as orq

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_page_byte_fixtures():
    g = json.load(open(os.path.join(GOLDEN, "rawint4_bytes.json")))
    for byte, vals in g["bytes"].items():
        got = orq.unpack_rawint4(np.array([[int(byte)]], dtype=np.uint8))[0]
        assert got.tolist() == vals, byte
    for case in g["scaled"]:
        packed = np.full((1, 16), case["byte"], dtype=np.uint8)
        scales = np.array([[case["scale"]]], dtype=np.float64)
        dense = orq.dequantize_rawint4(packed, scales)
        assert dense[0, :2].tolist() == case["values"]
        assert np.all(dense[0] == dense[0, 0]) or case["byte"] not in (0, 255, 153, 119)


def test_pack_unpack_roundtrip_all_bytes():
    allbytes = np.arange(256, dtype=np.uint8).reshape(8, 32)
    codes = orq.unpack_rawint4(allbytes).astype(np.int64) + 8
    assert codes.min() == 0 and codes.max() == 15
    assert np.array_equal(orq.pack_rawint4_codes(codes), allbytes)
    # low nibble first: byte 0x1F holds codes (15, 1)
    assert (orq.unpack_rawint4(np.array([[0x1F]], dtype=np.uint8)) + 8).tolist() == [[15, 1]]


def test_pack_rejects_bad_codes():
    with pytest.raises(ValueError):
        orq.pack_rawint4_codes(np.array([0, 16]))
    with pytest.raises(ValueError):
        orq.pack_rawint4_codes(np.array([0, 1, 2]))


def test_layout_validation():
    with pytest.raises(ValueError):
        orq.validate_layout(np.zeros((4, 8), np.uint8), np.zeros((4, 1)))  # K=16 not a multiple of 32
    with pytest.raises(ValueError):
        orq.validate_layout(np.zeros((4, 16), np.uint8), np.zeros((4, 2)))  # wrong scale count
    assert orq.validate_layout(np.zeros((4, 32), np.uint8), np.zeros((4, 2))) == (4, 64)


def test_zero_scale_gives_zero_weights():
    rng = np.random.default_rng(1)
    packed = rng.integers(0, 256, (3, 32), dtype=np.uint8)
    scales = rng.uniform(0.01, 0.07, (3, 2))
    scales[1, 1] = 0.0
    dense = orq.dequantize_rawint4(packed, scales)
    assert np.all(dense[1, 32:] == 0.0)
    assert np.count_nonzero(dense[1, :32]) > 0


def test_dense_matches_transpose_free_loop():
    """dY = identity turns the page's group-at-a-time dX loop into W itself."""
    rng = np.random.default_rng(2)
    n, k = 40, 96
    packed = rng.integers(0, 256, (n, k // 2), dtype=np.uint8)
    scales = rng.uniform(0.01, 0.07, (n, k // 32))
    dense = orq.dequantize_rawint4(packed, scales)
    w_loop = orq.transpose_free_dx(np.eye(n), packed, scales)
    assert np.array_equal(dense, w_loop)
    dy = rng.standard_normal((7, n))
    np.testing.assert_allclose(orq.transpose_free_dx(dy, packed, scales), dy @ dense, rtol=1e-12, atol=1e-12)


def test_bf16_rne_helper():
    # exact values pass through; halfway cases go to even
    f = np.array([1.0, -2.5, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, 0.0, -0.0], dtype=np.float32)
    bits = orq.f32_to_bf16_bits(f)
    back = orq.bf16_bits_to_f32(bits)
    assert back.tolist() == [1.0, -2.5, 1.0, 1.0 + 4 * 2 ** -8, 1.0, 0.0, -0.0]
    assert orq.f32_to_bf16_bits(np.array([np.nan], np.float32))[0] == 0x7FC0


def test_decode_f32_is_exact_product():
    rng = np.random.default_rng(3)
    packed = rng.integers(0, 256, (16, 64), dtype=np.uint8)
    scale_f32 = rng.uniform(0.01, 0.07, (16, 4)).astype(np.float32)
    scale_bits = orq.f32_to_bf16_bits(scale_f32)
    got = orq.decode_f32(packed, scale_bits).astype(np.float64)
    exact = orq.dequantize_rawint4(packed, orq.bf16_bits_to_f64(scale_bits))
    assert np.array_equal(got, exact)
    # bf16 decode = RNE of the exact product; some products are not bf16-representable
    b = orq.bf16_bits_to_f64(orq.decode_bf16_bits(packed, scale_bits))
    assert np.all(np.abs(b - exact) <= np.abs(exact) * 2.0 ** -8)  # half an ulp of an 8-bit significand
    assert np.any(b != exact)


def test_bf16_rne_matches_torch_conversion():
    import torch
    rng = np.random.default_rng(4)
    f = (rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000)).astype(np.float32)
    ours = orq.f32_to_bf16_bits(f)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
