"""CPU model of the kernel's bf16 P packing (truncation of the f32 p to its high
half) and of the gain that makes it unbiased: the constants in attn_common.cuh
against their derivation, and the mean of trunc(p * gain) / p on a large sample."""
import math
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
COMMON = os.path.join(ROOT, "attention_dit_attn_b200", "csrc", "attn_common.cuh")


def kernel_constants():
    text = open(COMMON).read()
    gain = float(re.search(r"kTruncGain = ([0-9.eE+-]+)f", text).group(1))
    log2g = float(re.search(r"kTruncLog2 = ([0-9.eE+-]+)f", text).group(1))
    return gain, log2g


def trunc_bf16(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 by dropping the low 16 bits (what the byte permute keeps), as float64."""
    bits = x.astype(np.float32).view(np.uint32) & np.uint32(0xFFFF0000)
    return bits.view(np.float32).astype(np.float64)


def test_constants_follow_the_derivation():
    gain, log2g = kernel_constants()
    mu = 1.0 / (512.0 * math.log(2.0))          # mean relative loss for log-uniform significands
    assert abs(gain - 1.0 / (1.0 - mu)) < 2e-7
    assert abs(log2g - math.log2(gain)) < 2e-7


def test_truncated_p_times_gain_is_unbiased():
    gain, log2g = kernel_constants()
    rng = np.random.default_rng(7)
    x = rng.uniform(-40.0, 8.0, 4_000_000)       # exponents as the kernel sees them (<= kRescaleLog2)
    p = np.exp2(x)
    # the kernel folds the gain into the exponent: 2^(x + log2 gain)
    pg = np.exp2(x + log2g).astype(np.float32)
    ratio = trunc_bf16(pg) / p
    assert abs(ratio.mean() - 1.0) < 2e-5, ratio.mean()
    # same spread as round-to-nearest: one bf16 ulp wide
    assert ratio.std() < 2.5e-3
    # without the gain the truncation is biased low by about mu
    plain = trunc_bf16(p.astype(np.float32)) / p
    assert abs((1.0 - plain.mean()) - 1.0 / (512.0 * math.log(2.0))) < 3e-5


def test_normalised_rows_have_no_scale_bias():
    """O = sum(trunc(p g) v) * g / sum(p g): the kernel's normalisation, on many rows."""
    gain, log2g = kernel_constants()
    rng = np.random.default_rng(11)
    n_rows, n_keys = 2000, 512
    s = rng.standard_normal((n_rows, n_keys)) * 1.5
    v = rng.standard_normal((n_keys,)) + 2.0                # a mean away from 0 exposes a scale bias
    x = (s - s.max(axis=1, keepdims=True)) / math.log(2.0)
    p = np.exp2(x)
    pg = np.exp2(x + log2g).astype(np.float32).astype(np.float64)
    o = (trunc_bf16(pg) @ v) * gain / pg.sum(axis=1)
    ref = (p @ v) / p.sum(axis=1)
    rel = (o - ref) / ref
    assert abs(rel.mean()) < 1e-4, rel.mean()
