"""Bit-exact GPU checks through the C ABI: int4 decode and the routing permutation."""

import numpy as np
import pytest
import torch

from oracle import moe as omoe
from oracle import rawint4 as orq
from tests._util import bf16_bits
from workloads import CONFIGS, make_routing, small_config

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from int4_quantised_moe_b200 import binding
    return binding


def _scales(gen, shape):
    return (torch.rand(shape, generator=gen) * 0.06 + 0.01).to(torch.bfloat16)


@pytest.mark.parametrize("n,k", [(64, 256), (37, 96), (1, 32), (512, 7168)])
def test_decode_bit_exact(B, n, k):
    gen = torch.Generator().manual_seed(n * 1000 + k)
    q = torch.randint(0, 256, (n, k // 2), generator=gen, dtype=torch.uint8)
    s = _scales(gen, (n, k // 32))
    # the contract test's signed extremes and a zero scale
    q[0, :16] = 0x00
    if n > 1:
        q[1, :16] = 0xFF
        s[n - 1, -1] = 0.0
    s[0, 0] = 0.0625
    out32 = torch.empty((n, k), dtype=torch.float32, device="cuda")
    out16 = torch.empty((n, k), dtype=torch.float16, device="cuda")
    B.rawint4_decode(q.cuda(), s.cuda(), out32, out16)
    torch.cuda.synchronize()
    ref32 = orq.decode_f32(q.numpy(), bf16_bits(s))
    assert np.array_equal(out32.cpu().numpy().view(np.uint32), ref32.view(np.uint32))
    ref16 = ref32.astype(np.float16)  # exact here: every product fits fp16
    assert np.array_equal(ref16.astype(np.float32), ref32)
    assert np.array_equal(out16.cpu().numpy().view(np.uint16), ref16.view(np.uint16))


@pytest.mark.parametrize("case", ["cfg0", "cfg1", "cfg2", "cfg3", "cfg4", "bad_ids", "single"])
def test_permutation_bit_exact(B, case):
    if case.startswith("cfg"):
        cfg = CONFIGS[int(case[3:])]
        gen = torch.Generator().manual_seed(11)
        ids, _ = make_routing(cfg, gen)
        E = cfg.experts
    elif case == "bad_ids":
        gen = torch.Generator().manual_seed(5)
        E = 16
        ids = torch.randint(0, E, (777, 4), generator=gen)
        ids[3, 1] = E
        ids[100, 0] = -3
        ids[776, 3] = 1 << 40
    else:
        E = 1
        ids = torch.zeros((3, 1), dtype=torch.int64)
    Q, k = ids.shape
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(Q * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(Q * k, dtype=torch.int32, device="cuda")
    B.rawint4_moe_permute(ids.cuda(), E, offsets, perm, inv)
    torch.cuda.synchronize()
    counts, ref_off, ref_perm, ref_inv = omoe.stable_expert_permutation(ids.numpy(), E)
    assert offsets.cpu().numpy().tolist() == ref_off.tolist()
    p = perm.cpu().numpy()
    n_valid = int(ref_off[-1])
    assert p[:n_valid].tolist() == ref_perm.tolist()
    assert np.all(p[n_valid:] == -1)
    assert inv.cpu().numpy().tolist() == ref_inv.tolist()


@pytest.mark.parametrize("n,k", [(3, 64), (128, 7168), (33, 2048)])
def test_mxfp4_decode_bit_exact(B, n, k):
    """MXFP4 decode: fp32 output equals the oracle's E2M1 value times the
    UE8M0 scale bit for bit; the fp16 tensor-core operand equals its fp16
    rounding, which is exact for scale bytes in [104, 140] (all of them here,
    plus the zero scale byte)."""
    from oracle import mxfp4 as ofp4
    gen = torch.Generator().manual_seed(n * 7 + k)
    q = torch.randint(0, 256, (n, k // 2), generator=gen, dtype=torch.uint8)
    s = torch.randint(104, 141, (n, k // 32), generator=gen, dtype=torch.uint8)
    q[0, :16] = torch.arange(16, dtype=torch.uint8) * 17  # every code, in both nibbles
    s[0, 0] = 0
    out32 = torch.empty((n, k), dtype=torch.float32, device="cuda")
    out16 = torch.empty((n, k), dtype=torch.float16, device="cuda")
    B.rawint4_mxfp4_decode(q.cuda(), s.cuda(), out32, out16)
    torch.cuda.synchronize()
    ref = ofp4.dequantize_mxfp4(q.numpy(), s.numpy())
    assert np.array_equal(out32.cpu().double().numpy(), ref)
    ref16 = ref.astype(np.float16)
    assert np.array_equal(ref16.astype(np.float64), ref)
    assert np.array_equal(out16.cpu().numpy().view(np.uint16), ref16.view(np.uint16))
