"""CPU oracle for the routed RAWINT4 MoE-LoRA layer (forward and backward).

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports, calls or links
this package; only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.

It is a plain, slow restatement of the method in float64 NumPy:

* ``oracle.rawint4``  - the RAWINT4 storage format: unpack, pack, dense
  dequantisation, the bit-exact fp32/bf16 decode, and the group-at-a-time
  transpose-free dX (page ``rawint4_sft_reference.py``).
* ``oracle.moe``      - the stable token->expert permutation, the routed
  MoE-LoRA forward (``routed_rawint4_lora``), the hand-derived backward, the
  clamped SwiGLU and its subgradient, and the authoritative gradient window of
  the contract test (``test_rawint4_sft_numerical.py``).
* ``oracle.metrics``  - relative L2 and cosine (``relative_l2_and_cosine``).

It shares no code with the CUDA path. Every function is pinned by the
``-m "not gpu"`` tests in ``tests/test_oracle_*.py`` (closed forms, page
fixtures, brute force, finite differences, autograd); see each module header.
"""

from . import metrics, moe, rawint4  # noqa: F401
