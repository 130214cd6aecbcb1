"""fp64 oracle of the step-cache reuse decision: TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module; the product path never does.

Step caching (DBCache) reuses transformer work from the previous denoising
step when the residual produced by the first transformer blocks has changed
little, with a `residual diff threshold` (0.12 in the published setting) that
trades speed for quality (page "How to Scale Diffusion Inference Across AMD
RDNA 4 GPUs", section "Skip Transformer Work Only When the Model Has Enough
Steps").  The page gives no formula.  The plainest reading, used here, is the
relative L1 change of that residual between consecutive steps,

    diff = sum_i |r_i - r'_i| / sum_i |r'_i|,     reuse  <=>  diff < threshold,

with r the current step's residual and r' the previous step's (both the same
shape).  When the previous residual is all zero, diff is 0 if the current one
is too, else +inf (never reuse).
"""
from __future__ import annotations

import numpy as np


def residual_diff(cur, prev) -> float:
    """Relative L1 change of cur against prev, in fp64 (plain sums)."""
    cur = np.asarray(cur, dtype=np.float64).ravel()
    prev = np.asarray(prev, dtype=np.float64).ravel()
    if cur.shape != prev.shape:
        raise ValueError("cur and prev must have the same number of elements")
    num = float(np.abs(cur - prev).sum())
    den = float(np.abs(prev).sum())
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return num / den


def reuse(cur, prev, threshold: float) -> bool:
    """The cache decision: reuse the previous step's work when diff < threshold."""
    return residual_diff(cur, prev) < threshold
