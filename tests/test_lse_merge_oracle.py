"""Pins of the LSE-merge oracle (CPU only) against facts other than its own formula:
the attention oracle over the whole key range, a library attention on uneven key
splits, closed forms, and the algebra the merge must satisfy."""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle.lse_merge import lse_merge


def _f64_inputs(B, H, L, D, seed):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal((B, H, L, D)) for _ in range(3)]


def test_split_keys_equals_full_attention():
    """Ring-attention identity: query chunk r against each equal key chunk, merged,
    equals the attention oracle over all keys (independently pinned)."""
    B, H, Lc, D, n = 1, 2, 40, 16, 3
    q, k, v = _f64_inputs(B, H, n * Lc, D, 5)
    scale = 1 / math.sqrt(D)
    o_full, lse_full = oracle.attention(q, k, v, scale, dtype=oracle.F64)
    for r in range(n):
        qs = q[:, :, r * Lc:(r + 1) * Lc]
        parts = [oracle.attention(qs, k[:, :, c * Lc:(c + 1) * Lc], v[:, :, c * Lc:(c + 1) * Lc], scale,
                                  dtype=oracle.F64) for c in range(n)]
        o, lse = lse_merge([p[0].reshape(-1, D) for p in parts], [p[1].reshape(-1) for p in parts])
        np.testing.assert_allclose(o, o_full[:, :, r * Lc:(r + 1) * Lc].reshape(-1, D), rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, lse_full[:, :, r * Lc:(r + 1) * Lc].reshape(-1), rtol=0, atol=1e-12)


def test_uneven_split_with_library_partials():
    """Partials from torch's fp64 SDPA and logsumexp on uneven key chunks."""
    B, H, L, D = 1, 3, 97, 32
    q, k, v = _f64_inputs(B, H, L, D, 6)
    scale = 1 / math.sqrt(D)
    o_full, lse_full = oracle.attention(q, k, v, scale, dtype=oracle.F64)
    cuts = [0, 13, 14, 60, 97]
    tq = torch.from_numpy(q)
    parts_o, parts_l = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        kc, vc = torch.from_numpy(k[:, :, a:b]), torch.from_numpy(v[:, :, a:b])
        parts_o.append(torch.nn.functional.scaled_dot_product_attention(tq, kc, vc, scale=scale)
                       .numpy().reshape(-1, D))
        parts_l.append(torch.logsumexp(scale * tq @ kc.transpose(-1, -2), dim=-1).numpy().reshape(-1))
    o, lse = lse_merge(parts_o, parts_l)
    np.testing.assert_allclose(o, o_full.reshape(-1, D), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_full.reshape(-1), rtol=0, atol=1e-12)


def test_closed_form_two_parts_large_lse():
    """lse 1000 and 1001 (exp would overflow without the max): o = (o0 + e o1)/(1 + e)."""
    o0, o1 = np.array([[1.0, -2.0]]), np.array([[3.0, 5.0]])
    o, lse = lse_merge([o0, o1], [np.array([1000.0]), np.array([1001.0])])
    e = math.e
    np.testing.assert_allclose(o, (o0 + e * o1) / (1 + e), rtol=1e-15, atol=1e-15)
    assert abs(lse[0] - (1001.0 + math.log1p(math.exp(-1.0)))) < 1e-12


def test_equal_lse_is_mean_and_log_n():
    rng = np.random.default_rng(1)
    parts = [rng.standard_normal((5, 8)) for _ in range(4)]
    l0 = rng.standard_normal(5)
    o, lse = lse_merge(parts, [l0] * 4)
    np.testing.assert_allclose(o, np.mean(parts, axis=0), rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, l0 + math.log(4), rtol=0, atol=1e-15)


def test_empty_part_is_identity_and_all_empty_is_zero():
    rng = np.random.default_rng(2)
    o0, l0 = rng.standard_normal((6, 4)), rng.standard_normal(6)
    junk = rng.standard_normal((6, 4)) * 1e6
    o, lse = lse_merge([junk, o0], [np.full(6, -np.inf), l0])
    np.testing.assert_array_equal(o, o0)
    np.testing.assert_array_equal(lse, l0)
    o, lse = lse_merge([o0, junk], [np.full(6, -np.inf)] * 2)
    assert (o == 0).all() and np.isneginf(lse).all()


def test_order_independent_and_associative():
    rng = np.random.default_rng(3)
    parts = [(rng.standard_normal((7, 5)), rng.standard_normal(7) * 3) for _ in range(3)]
    o_abc, l_abc = lse_merge([p[0] for p in parts], [p[1] for p in parts])
    o_cab, l_cab = lse_merge([parts[2][0], parts[0][0], parts[1][0]], [parts[2][1], parts[0][1], parts[1][1]])
    np.testing.assert_allclose(o_cab, o_abc, rtol=0, atol=1e-14)
    np.testing.assert_allclose(l_cab, l_abc, rtol=0, atol=1e-14)
    o_ab, l_ab = lse_merge([parts[0][0], parts[1][0]], [parts[0][1], parts[1][1]])
    o_2, l_2 = lse_merge([o_ab, parts[2][0]], [l_ab, parts[2][1]])
    np.testing.assert_allclose(o_2, o_abc, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l_2, l_abc, rtol=0, atol=1e-13)


def test_rejects_mismatched_parts():
    with pytest.raises(ValueError):
        lse_merge([np.zeros((2, 2))], [])
