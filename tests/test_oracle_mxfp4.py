"""Pins for oracle.mxfp4 (no GPU).

The E2M1 values are checked against the format's value table (sign and the
eight magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), not against the oracle's own
formula; the UE8M0 bit-cast against powers of two; packing against a
per-byte round trip; the dense dequantisation against a per-element loop;
and an MXFP4 layer against a textbook SwiGLU FFN built from those values.
"""

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import moe as omoe
from oracle import mxfp4 as ofp4
from oracle import rawint4 as orq

# the eight E2M1 magnitudes in code order 0..7 (sign bit clear); codes 8..15
# are the same magnitudes negated
E2M1_MAGNITUDES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def test_e2m1_values_match_the_format_table():
    for code in range(16):
        mag = E2M1_MAGNITUDES[code & 7]
        want = -mag if code & 8 else mag
        assert ofp4.e2m1_value(code) == want, code
    assert np.signbit(ofp4.e2m1_value(8))  # -0
    with pytest.raises(ValueError):
        ofp4.e2m1_value(16)


def test_ue8m0_bitcast_is_a_power_of_two():
    e = np.arange(256, dtype=np.uint8)
    v = ofp4.ue8m0_scale(e)
    for i in range(1, 255):
        assert v[i] == 2.0 ** (i - 127), i
    assert v[0] == 0.0 and np.isinf(v[255])
    # the bit pattern is the byte in the bf16 exponent field
    assert ofp4.ue8m0_bf16_bits(np.array([127], np.uint8))[0] == 0x3F80  # bf16 1.0


def test_pack_unpack_round_trip_all_bytes():
    b = np.arange(256, dtype=np.uint8).reshape(16, 16)
    codes = ofp4.unpack_codes(b)
    assert codes.shape == (16, 32)
    assert np.array_equal(codes[..., 0::2], b & 15)  # low nibble first
    assert np.array_equal(ofp4.pack_codes(codes), b)
    with pytest.raises(ValueError):
        ofp4.pack_codes(np.array([1, 2, 3]))


def test_dequantize_matches_element_loop():
    rng = np.random.default_rng(5)
    n, k = 6, 96
    packed = rng.integers(0, 256, (n, k // 2), dtype=np.uint8)
    scales = rng.integers(115, 131, (n, k // 32), dtype=np.uint8)
    dense = ofp4.dequantize_mxfp4(packed, scales)
    for i in range(n):
        for j in range(k):
            byte = int(packed[i, j // 2])
            code = (byte >> 4) if j % 2 else (byte & 15)
            mag = E2M1_MAGNITUDES[code & 7] * (-1.0 if code & 8 else 1.0)
            assert dense[i, j] == mag * 2.0 ** (int(scales[i, j // 32]) - 127)


def test_mxfp4_layer_is_textbook_swiglu_ffn():
    """One expert, top-1, w = 1, no clamp, LoRA B = 0: the routed layer with
    MXFP4 weights equals silu(x Wg^T) (x Wu^T) Wd^T with the weights from the
    element loop above."""
    rng = np.random.default_rng(11)
    H, I, r, Q = 64, 96, 4, 5
    q = {n: rng.integers(0, 256, (1, rows, cols // 2), dtype=np.uint8)
         for n, rows, cols in (("g", I, H), ("u", I, H), ("d", H, I))}
    s = {n: rng.integers(118, 126, (1, rows, cols // 32), dtype=np.uint8)
         for n, rows, cols in (("g", I, H), ("u", I, H), ("d", H, I))}
    lora = {"gate_lora_a": rng.normal(0, 0.02, (1, r, H)), "gate_lora_b": np.zeros((1, I, r)),
            "up_lora_a": rng.normal(0, 0.02, (1, r, H)), "up_lora_b": np.zeros((1, I, r)),
            "down_lora_a": rng.normal(0, 0.02, (1, r, I)), "down_lora_b": np.zeros((1, H, r))}
    layer = omoe.Layer(q["g"], s["g"], q["u"], s["u"], q["d"], s["d"], lora, alpha=2.0 * r, swiglu_limit=0.0,
                       weight_format="mxfp4")
    x = rng.normal(0, 1, (Q, H))
    ids = np.zeros((Q, 1), dtype=np.int64)
    out, _ = omoe.forward(layer, x, ids, np.ones((Q, 1)))

    def dense(packed, scales):
        rows, half = packed.shape
        w = np.empty((rows, 2 * half))
        for i in range(rows):
            for j in range(2 * half):
                byte = int(packed[i, j // 2])
                code = (byte >> 4) if j % 2 else (byte & 15)
                w[i, j] = E2M1_MAGNITUDES[code & 7] * (-1.0 if code & 8 else 1.0) * 2.0 ** (int(scales[i, j // 32]) - 127)
        return torch.from_numpy(w)

    Wg, Wu, Wd = dense(q["g"][0], s["g"][0]), dense(q["u"][0], s["u"][0]), dense(q["d"][0], s["d"][0])
    xt = torch.from_numpy(x)
    ref = F.linear(F.silu(F.linear(xt, Wg)) * F.linear(xt, Wu), Wd)
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_fp16_holds_every_decoded_value_in_range():
    """Every E2M1 value times 2^(e - 127) is exact in fp16 for e in [104, 140]
    (at most two significant bits, inside fp16's range): the reading behind
    the tensor-core operand type of the MXFP4 variant."""
    for e in (104, 110, 120, 127, 135, 140):
        v = np.array(E2M1_MAGNITUDES) * 2.0 ** (e - 127)
        assert np.array_equal(v.astype(np.float16).astype(np.float64), v), e
    # just outside: the smallest nonzero value no longer fits
    v = 0.5 * 2.0 ** (103 - 127)
    assert float(np.float16(v)) != v
