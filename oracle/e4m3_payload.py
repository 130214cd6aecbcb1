"""fp64 oracle of the Ulysses FP8 payload preparation: TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module; the product path never does.

The page "How to Scale Diffusion Inference Across AMD RDNA 4 GPUs" (section
"Balance Transformer Work and Communication") sends the all-to-all of Ulysses
sequence parallelism in FP8 (`--use fp8 comms`).  It does not say how values
are scaled; the reading used here is the per-head recipe the FP8 attention
inputs follow:

  * per row r (one (b, h) head of a shard): amax_r = max_i |x_ri|;
  * dequantisation scale s_r = amax_r / 448 rounded to fp32 (448 = the largest
    finite e4m3 value), and s_r = 1 for a row of zeros;
  * codes q_ri = e4m3(x_ri / s_r), the quotient rounded to fp32 first, then to
    the nearest e4m3 value, ties to the even code, magnitudes beyond 448
    saturating to 448; the sign bit is the sign of the quotient (negative values
    that round to 0 give -0);
  * the heads are then grouped by destination rank: a transpose of contiguous
    blocks, out[c][r] = in[r][c].

e4m3 is the OCP 8-bit float E4M3 ("fn" variant): 1 sign bit, 4 exponent bits
with bias 7, 3 mantissa bits, subnormals (exponent field 0: m/8 * 2^-6), no
infinities, codes 0x7F / 0xFF are NaN, so the largest finite value is
1.75 * 2^8 = 448.

The fp32 roundings are taken in fp64 and then rounded once to fp32.  For the
quotient of a bf16 value (8 significant bits) by an fp32 scale (and for
amax / 448) that equals the correctly rounded fp32 result: such a quotient is
never an fp32 rounding midpoint (those need 25 significant bits), and when it
is not one it lies at least about 2^-49 (relative) away from every midpoint,
far beyond the 2^-53 by which the fp64 rounding can move it.

Non-finite inputs are outside the contract (never generated).
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def decode_table() -> np.ndarray:
    """The 256 e4m3 codes as fp64 values (NaN for 0x7F and 0xFF)."""
    out = np.empty(256, dtype=np.float64)
    for c in range(256):
        sign = -1.0 if c & 0x80 else 1.0
        e = (c >> 3) & 0xF
        m = c & 0x7
        if e == 0xF and m == 0x7:
            out[c] = np.nan
        elif e == 0:
            out[c] = sign * (m / 8.0) * 2.0 ** -6
        else:
            out[c] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return out


_TABLE = decode_table()
_POS = _TABLE[:0x7F]                     # codes 0x00 .. 0x7E: 0 .. 448, increasing


def encode(v: np.ndarray) -> np.ndarray:
    """fp64 values -> e4m3 codes (uint8): nearest, ties to the even code,
    saturating at +-448, sign kept for results of magnitude 0."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    hi = np.clip(np.searchsorted(_POS, a, side="left"), 1, len(_POS) - 1)   # _POS[hi-1] < a <= _POS[hi]
    lo = hi - 1
    d_lo = a - _POS[lo]
    d_hi = _POS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(a >= E4M3_MAX, 0x7E, code)
    code = np.where(a == 0.0, 0, code)
    neg = np.signbit(v)
    return (code | np.where(neg, 0x80, 0)).astype(np.uint8)


def absmax_rows(x: np.ndarray, rows: int) -> np.ndarray:
    """max |x| over each of `rows` equal contiguous rows (exact)."""
    return np.abs(np.asarray(x, dtype=np.float64)).reshape(rows, -1).max(axis=1)


def row_scales(amax: np.ndarray) -> np.ndarray:
    """s = fp32(amax / 448), 1 where amax == 0."""
    amax = np.asarray(amax, dtype=np.float64)
    s = (amax / E4M3_MAX).astype(np.float32)
    return np.where(amax > 0, s, np.float32(1.0)).astype(np.float32)


def quantize_rows(x: np.ndarray, amax: np.ndarray):
    """Codes (uint8, the shape of x) and the fp32 scales of each row."""
    x = np.asarray(x, dtype=np.float64)
    rows = len(amax)
    s = row_scales(amax)
    v = (x.reshape(rows, -1) / s.astype(np.float64)[:, None]).astype(np.float32)
    return encode(v.astype(np.float64)).reshape(x.shape), s


def block_transpose(b: np.ndarray, R: int, C: int) -> np.ndarray:
    """Bytes of R x C contiguous equal blocks -> the C x R arrangement."""
    b = np.ascontiguousarray(b).view(np.uint8).reshape(R, C, -1)
    return np.ascontiguousarray(b.transpose(1, 0, 2)).reshape(-1)
