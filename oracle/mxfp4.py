"""fp64 oracle of the MXFP4 1x32 activation quantiser: TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module; the product path never does.

The page "Accelerating Diffusers and xDiT Image Generation with MXFP4 using
AMD Quark on AMD Instinct MI350 GPUs" (sections "MXFP4 Quantization" and
"MXFP4 Kernel") quantises the linear layers' activations on the fly to MXFP4,
the OCP Microscaling format it cites: blocks of 32 consecutive values along
the last axis share one E8M0 (power-of-two) scale, and each value is a 4-bit
E2M1 float.  The page does not restate the conversion rule; the plainest
reading is the OCP MX definition it points to:

  * shared exponent  s = floor(log2(max_i |v_i|)) - 2   (2 = the largest E2M1
    exponent), clamped to E8M0's range [-127, 127]; a block of zeros takes
    s = -127;
  * element codes    q_i = E2M1(v_i / 2^s), rounded to nearest, ties to even,
    magnitudes above 6 saturating to 6; the sign bit is the sign of v_i
    (negative values that round to 0 give -0);
  * E2M1 = 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit: magnitudes
    0, 0.5, 1, 1.5, 2, 3, 4, 6 for codes 0..7;
  * storage: the E8M0 byte s + 127 per block; two codes per byte, the block's
    first element of each pair in the low 4 bits.

Non-finite inputs are outside the contract (never generated).
"""
from __future__ import annotations

import numpy as np

E2M1_MAGNITUDES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)
BLOCK = 32
EMAX_ELEM = 2


def e2m1_round(y: np.ndarray) -> np.ndarray:
    """Round |y| to the E2M1 grid (nearest, ties to the code with an even
    mantissa bit, saturating at 6): returns codes 0..7 (magnitude only)."""
    a = np.abs(np.asarray(y, dtype=np.float64))
    grid = np.array(E2M1_MAGNITUDES)
    codes = np.empty(a.shape, dtype=np.uint8)
    flat, out = a.ravel(), codes.ravel()
    for idx, x in enumerate(flat):
        if x >= 6.0:
            out[idx] = 7
            continue
        hi = int(np.searchsorted(grid, x, side="left"))      # grid[hi-1] < x <= grid[hi]
        if grid[hi] == x:
            out[idx] = hi
            continue
        lo = hi - 1
        dlo, dhi = x - grid[lo], grid[hi] - x
        if dlo < dhi:
            out[idx] = lo
        elif dhi < dlo:
            out[idx] = hi
        else:                                                # tie: the even mantissa bit
            out[idx] = lo if lo % 2 == 0 else hi
    return codes


def shared_exponent(block_amax: np.ndarray) -> np.ndarray:
    """floor(log2(amax)) - 2 per block, clamped to [-127, 127]; -127 for amax = 0."""
    amax = np.asarray(block_amax, dtype=np.float64)
    s = np.full(amax.shape, -127, dtype=np.int64)
    nz = amax > 0
    _, e = np.frexp(amax[nz])                                # amax = f * 2^e, f in [0.5, 1)
    s[nz] = (e - 1) - EMAX_ELEM                              # floor(log2(amax)) = e - 1
    return np.clip(s, -127, 127)


def quantize(x) -> tuple[np.ndarray, np.ndarray]:
    """x: [rows, K] (K a multiple of 32).  Returns (packed codes uint8 [rows, K/2],
    E8M0 scales uint8 [rows, K/32])."""
    x = np.asarray(x, dtype=np.float64)
    rows, K = x.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 32")
    blocks = x.reshape(rows, K // BLOCK, BLOCK)
    s = shared_exponent(np.abs(blocks).max(axis=2))           # [rows, K/32]
    y = blocks / np.exp2(s.astype(np.float64))[:, :, None]    # exact: power-of-two scale
    codes = e2m1_round(y) | (np.signbit(blocks).astype(np.uint8) << 3)
    codes = codes.reshape(rows, K)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed, (s + 127).astype(np.uint8)


def dequantize(packed: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Inverse map: [rows, K/2] codes + [rows, K/32] E8M0 -> fp64 [rows, K]."""
    packed = np.asarray(packed, dtype=np.uint8)
    rows, half = packed.shape
    codes = np.empty((rows, 2 * half), dtype=np.uint8)
    codes[:, 0::2] = packed & 0xF
    codes[:, 1::2] = packed >> 4
    mag = np.array(E2M1_MAGNITUDES)[codes & 7]
    val = np.where(codes & 8, -mag, mag)
    s = np.asarray(scales, dtype=np.int64) - 127
    return val * np.repeat(np.exp2(s.astype(np.float64)), BLOCK, axis=1)
