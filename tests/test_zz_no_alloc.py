"""rawint4_moe_permute_static: the permutation for callers that cannot allocate.

Some callers cannot call cudaMalloc to hand the permutation its scratch
buffer (another component owns all device memory, or a device-synchronising
allocation is not acceptable mid-stream). rawint4_moe_permute_static keeps
that scratch in a fixed 1 MiB array inside the library. This test calls it
through the C ABI and checks that two calls in a row return exactly what the
caller-scratch entry point rawint4_moe_permute returns (integer outputs:
bit-exact), and that a problem larger than the fixed scratch is refused.
"""

import ctypes

import pytest
import torch

from workloads import CONFIGS, make_routing

pytestmark = pytest.mark.gpu


def _ids(case):
    if case == "largest":
        cfg = CONFIGS[4]
        ids, _ = make_routing(cfg, torch.Generator().manual_seed(3))
        return ids, cfg.experts
    if case == "zipf":
        cfg = CONFIGS[3]
        ids, _ = make_routing(cfg, torch.Generator().manual_seed(4))
        return ids, cfg.experts
    g = torch.Generator().manual_seed(5)
    ids = torch.randint(0, 16, (300, 4), generator=g)
    ids[7, 2] = 16  # out of range: dropped, inv = -1
    ids[299, 0] = -1
    return ids, 16


def _run(B, fn, ids, E):
    Q, k = ids.shape
    offsets = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    perm = torch.full((Q * k,), -7, dtype=torch.int32, device="cuda")
    inv = torch.full((Q * k,), -7, dtype=torch.int32, device="cuda")
    fn(ids.cuda(), E, offsets, perm, inv)
    torch.cuda.synchronize()
    return offsets.cpu(), perm.cpu(), inv.cpu()


def test_static_scratch_matches_caller_scratch_twice():
    from int4_quantised_moe_b200 import binding as B
    assert B.rawint4_moe_permute_static_max_bytes() == 1 << 20
    # two different problems back to back: the second call starts from the
    # state the first left in the shared array
    for case in ("largest", "bad_ids", "zipf"):
        ids, E = _ids(case)
        ref = _run(B, B.rawint4_moe_permute, ids, E)
        for _ in range(2):
            got = _run(B, B.rawint4_moe_permute_static, ids, E)
            for a, b in zip(got, ref):
                assert torch.equal(a, b), case


def test_static_scratch_refuses_oversized_problems():
    from int4_quantised_moe_b200 import binding as B
    cdll = B.library()
    # 2^20 slots over 4096 experts needs 1024 histograms of 16 KiB: far over 1 MiB.
    # The host rejects it before anything is enqueued, so the placeholder
    # pointers are never dereferenced.
    dummy = ctypes.c_void_p(256)
    rc = cdll.rawint4_moe_permute_static(dummy, 1 << 17, 8, 4096, dummy, dummy, dummy, None)
    assert rc == B.STATIC_SCRATCH_TOO_SMALL
    assert "fixed scratch" in B.strerror(rc)
