"""Pins of the low-precision GEMM oracle (oracle/lowp_gemm.py) to facts
outside it: an integer formulation written here from the formats' definitions
(E2M1 magnitudes are halves, e4m3 values are multiples of 2^-9, E8M0 is a
power of two), closed forms, the transpose identity, and the round trip
through the MXFP4 quantiser on values it represents exactly."""
from fractions import Fraction

import numpy as np
import pytest

from oracle import e4m3_payload, lowp_gemm, mxfp4

# Twice the E2M1 magnitude of codes 0..7: 0, 0.5, 1, 1.5, 2, 3, 4, 6 -> integers.
TWICE_E2M1 = [0, 1, 2, 3, 4, 6, 8, 12]


def _random_mxfp4(rng, rows, K, s_lo=-3, s_hi=3):
    codes = rng.integers(0, 16, size=(rows, K), dtype=np.uint8)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    scales = (rng.integers(s_lo, s_hi + 1, size=(rows, K // 32)) + 127).astype(np.uint8)
    return codes, packed, scales


def _exact_mxfp4(codes_a, scales_a, codes_w, scales_w):
    """Sum of (2 qa)(2 qw)/4 * 2^(sa + sw) over k, as exact Fractions."""
    M, K = codes_a.shape
    N = codes_w.shape[0]
    ia = [[(-1 if c & 8 else 1) * TWICE_E2M1[c & 7] for c in row] for row in codes_a.tolist()]
    iw = [[(-1 if c & 8 else 1) * TWICE_E2M1[c & 7] for c in row] for row in codes_w.tolist()]
    out = np.empty((M, N))
    for m in range(M):
        for n in range(N):
            acc = Fraction(0)
            for b in range(K // 32):
                dot = sum(ia[m][k] * iw[n][k] for k in range(32 * b, 32 * b + 32))
                acc += Fraction(dot, 4) * Fraction(2) ** (int(scales_a[m, b]) - 127 + int(scales_w[n, b]) - 127)
            out[m, n] = float(acc)
            assert Fraction(out[m, n]) == acc            # the exact value is an fp64 number
    return out


@pytest.mark.parametrize("M,N,K,seed", [(3, 5, 32, 1), (4, 6, 96, 2), (2, 3, 256, 3)])
def test_mxfp4_gemm_is_the_exact_block_scaled_sum(M, N, K, seed):
    rng = np.random.default_rng(seed)
    ca, pa, sa = _random_mxfp4(rng, M, K)
    cw, pw, sw = _random_mxfp4(rng, N, K)
    got = lowp_gemm.gemm_mxfp4(pa, sa, pw, sw)
    assert np.array_equal(got, _exact_mxfp4(ca, sa, cw, sw))


def test_mxfp4_gemm_transpose_identity_and_closed_form():
    rng = np.random.default_rng(4)
    _, pa, sa = _random_mxfp4(rng, 3, 64)
    _, pw, sw = _random_mxfp4(rng, 4, 64)
    assert np.array_equal(lowp_gemm.gemm_mxfp4(pa, sa, pw, sw), lowp_gemm.gemm_mxfp4(pw, sw, pa, sa).T)
    # A = all ones (code 2, scale 2^0); W row n = the constant 1.5 * 2^n (code 3, scale 2^n).
    K = 64
    ones = np.full((1, K // 2), 2 | (2 << 4), dtype=np.uint8)
    w = np.full((3, K // 2), 3 | (3 << 4), dtype=np.uint8)
    ws = (np.arange(3)[:, None] + 127 + np.zeros((1, K // 32), dtype=np.int64)).astype(np.uint8)
    got = lowp_gemm.gemm_mxfp4(ones, np.full((1, K // 32), 127, dtype=np.uint8), w, ws)
    assert list(got[0]) == [K * 1.5, K * 3.0, K * 6.0]


def test_mxfp4_gemm_of_exactly_representable_operands_equals_the_plain_product():
    rng = np.random.default_rng(5)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    # Blocks whose absmax is 6 * 2^s: the quantiser keeps every value exactly.
    def exact_block_values(rows, K):
        v = grid[rng.integers(0, 8, size=(rows, K))] * rng.choice([-1, 1], size=(rows, K))
        v[:, ::32] = 6.0
        return v * np.exp2(rng.integers(-2, 3, size=(rows, K // 32))).repeat(32, axis=1)
    a, w = exact_block_values(3, 64), exact_block_values(5, 64)
    pa, sa = mxfp4.quantize(a)
    pw, sw = mxfp4.quantize(w)
    assert np.array_equal(lowp_gemm.gemm_mxfp4(pa, sa, pw, sw), a @ w.T)


def test_e4m3_gemm_is_the_exact_scaled_integer_sum():
    rng = np.random.default_rng(6)
    table = e4m3_payload.decode_table()
    finite = np.array([c for c in range(256) if not np.isnan(table[c])], dtype=np.uint8)
    a = rng.choice(finite, size=(4, 80))
    w = rng.choice(finite, size=(3, 80))
    sa, sw = 0.0125, 3.5
    got = lowp_gemm.gemm_e4m3(a, sa, w, sw)
    # Every e4m3 value times 2^9 is an integer.
    ia = [[int(table[c] * 512) for c in row] for row in a.tolist()]
    iw = [[int(table[c] * 512) for c in row] for row in w.tolist()]
    for m in range(4):
        for n in range(3):
            exact = Fraction(sum(x * y for x, y in zip(ia[m], iw[n])), 512 * 512)
            assert got[m, n] == float(sa) * float(sw) * float(exact)


def test_e4m3_gemm_rejects_nan_codes():
    with pytest.raises(ValueError):
        lowp_gemm.gemm_e4m3(np.array([[0x7F]], dtype=np.uint8), 1.0, np.array([[0x38]], dtype=np.uint8), 1.0)
