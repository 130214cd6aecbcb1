"""CPU model of the kernel's FMA-pipe exp2 (same float32 steps): its error bound
against numpy's exp2, and the coefficients' provenance (re-fitted here)."""
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "attention_dit_attn_b200", "csrc")
sys.path.insert(0, CSRC)
import exp2_poly_fit  # noqa: E402


def kernel_coeffs():
    text = open(os.path.join(CSRC, "attn_common.cuh")).read()
    vals = {k: float(v) for k, v in re.findall(r"kPolyC(\d) = ([0-9.eE+-]+)f", text)}
    return np.array([vals["0"], vals["1"], vals["2"], vals["3"]], dtype=np.float32)


def exp2_poly_model(x: np.ndarray, c: np.ndarray) -> np.ndarray:
    """float32 replica of exp2_poly2: clamp to [-126, 127], rint via 1.5*2^23, cubic,
    exponent add."""
    x = np.minimum(np.maximum(x.astype(np.float32), np.float32(-126.0)), np.float32(127.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    q = exp2_poly_fit.horner32(c, f)
    bits = q.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.view(np.float32)


def test_coefficients_are_the_fit():
    assert np.allclose(kernel_coeffs(), exp2_poly_fit.fit(), rtol=0, atol=2e-6)


def test_relative_error_below_bf16_and_f16_half_ulp():
    # x above 0 occurs: a later key tile may exceed the running max of the first.
    x = np.linspace(-60.0, 126.0, 2_000_001, dtype=np.float32)
    got = exp2_poly_model(x, kernel_coeffs()).astype(np.float64)
    rel = np.abs(got / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() < 1e-4 < 2.0 ** -11     # f16 P half-ulp is 2^-11, bf16 2^-9


def test_clamped_tail_is_tiny_and_positive():
    x = np.array([-126.0, -200.0, -1e30], dtype=np.float32)
    got = exp2_poly_model(x, kernel_coeffs())
    assert np.all(got >= 0) and np.all(got < 1e-37)


def test_clamped_head_is_finite_and_caught_by_the_guard():
    """x past 127 gives 2^127: finite (no wrap of the exponent field) and far above
    both guards on the sum of p (2^15 for f16 P, 2^64 for bf16 P)."""
    x = np.array([127.0, 128.5, 300.0, 1e30], dtype=np.float32)
    got = exp2_poly_model(x, kernel_coeffs()).astype(np.float64)
    assert np.all(np.isfinite(got)) and np.all(got > 2.0 ** 126)
    assert np.all(got >= 2.0 ** 64)
