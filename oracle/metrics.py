"""Comparison metric of ``rawint4_sft_reference.py`` (``relative_l2_and_cosine``).

Test infrastructure only. Both numbers are taken over the whole flattened
tensor: relative L2 = |a - e| / max(|e|, 1e-12), cosine = a.e / max(|a||e|, 1e-20).
Pinned in tests/test_oracle_moe.py by closed-form cases (identical vectors,
orthogonal vectors, a known scaled perturbation).
"""

from __future__ import annotations

import numpy as np


def relative_l2_and_cosine(actual, expected):
    a = np.asarray(actual, dtype=np.float64).ravel()
    e = np.asarray(expected, dtype=np.float64).ravel()
    diff = np.linalg.norm(a - e)
    en = np.linalg.norm(e)
    an = np.linalg.norm(a)
    rel = float(diff / max(en, 1.0e-12))
    cos = float(np.dot(a, e) / max(an * en, 1.0e-20))
    return rel, cos
