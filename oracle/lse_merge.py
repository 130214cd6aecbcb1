"""fp64 oracle of the LSE merge of partial attentions: TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module; the product path never does.

Ring attention and USP (cited in the reference list of "xDiT: an Inference
Engine for Diffusion Transformers (DiTs) with Massive Parallelism"; the
`ring degree` setting of the 2-GPU script on the page "Accelerating Diffusers
and xDiT Image Generation with MXFP4 using AMD Quark on AMD Instinct MI350
GPUs") compute attention for a block of query rows one K/V chunk at a time and
combine the partial results.  The pages give no formula.  The plainest reading,
and the one that makes the combination exact, is the log-sum-exp rule: a
partial result over key chunk c is o_c = sum_{j in c} e^{s_j} v_j / l_c with
lse_c = log l_c, so over the union of the chunks

    lse = log sum_c exp(lse_c),      o = sum_c exp(lse_c - lse) o_c.

Written out below with the row max M = max_c lse_c subtracted first (exact in
real arithmetic).  A row whose parts all have lse = -inf (no keys at all) gives
o = 0 and lse = -inf.
"""
from __future__ import annotations

import numpy as np


def lse_merge(o_parts, lse_parts):
    """o_parts: sequence of [R, D] arrays; lse_parts: sequence of [R] arrays (natural log).

    Returns (o [R, D] float64, lse [R] float64)."""
    if len(o_parts) == 0 or len(o_parts) != len(lse_parts):
        raise ValueError("need one lse per partial output, at least one part")
    o_parts = [np.asarray(o, dtype=np.float64) for o in o_parts]
    lse_parts = [np.asarray(l, dtype=np.float64) for l in lse_parts]
    R, D = o_parts[0].shape
    lse_all = np.stack(lse_parts, axis=0)                   # [n, R]
    m = lse_all.max(axis=0)                                 # [R]
    o = np.zeros((R, D), dtype=np.float64)
    lse = np.full(R, -np.inf, dtype=np.float64)
    ok = np.isfinite(m)
    if ok.any():
        w = np.exp(lse_all[:, ok] - m[ok])                  # [n, R_ok], exp(-inf) = 0
        s = w.sum(axis=0)
        lse[ok] = m[ok] + np.log(s)
        acc = np.zeros((int(ok.sum()), D), dtype=np.float64)
        for c in range(len(o_parts)):
            acc += w[c][:, None] * o_parts[c][ok]
        o[ok] = acc / s[:, None]
    return o, lse
