"""fp64 oracle of the block-scaled low-precision linear layers: TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module; the product path never does.

The page "Accelerating Diffusers and xDiT Image Generation with MXFP4 using
AMD Quark on AMD Instinct MI350 GPUs" (sections "MXFP4 Quantization" and
"MXFP4 Kernel") runs the transformer's linear layers as FP4 x FP4 GEMMs on
MXFP4 operands: activations quantised on the fly in 1x32 blocks along K,
weights quantised the same way at load.  The page "How to Scale Diffusion
Inference Across AMD RDNA 4 GPUs" (section "Make the Model Fit Before Tuning
Latency") runs them in FP8 instead (`--gemm quantization fp8`).  Neither page
prints a formula; the plain reading is the GEMM of the dequantised operands,

    Y[m, n] = sum_k A[m, k] W[n, k]        (x @ W^T for activations A [M, K], weights W [N, K])

with
  * MXFP4: A and W the MXFP4 values, E2M1 code x 2^(E8M0 - 127) for each block
    of 32 consecutive k (oracle/mxfp4.py);
  * FP8: A and W the e4m3 values times one fp32 dequantisation scale per
    tensor (oracle/e4m3_payload.py decodes e4m3).

Every E2M1 value is a multiple of 1/2 below 8 and every e4m3 value a multiple
of 2^-9 below 2^9, so for the sizes and scale ranges the tests use, every
product and partial sum is exactly representable in fp64: the result below
is the exact one, in any summation order.
"""
from __future__ import annotations

import numpy as np

from . import e4m3_payload, mxfp4


def gemm_mxfp4(a_packed, a_scales, w_packed, w_scales) -> np.ndarray:
    """a_packed [M, K/2], a_scales [M, K/32], w_packed [N, K/2], w_scales [N, K/32]
    (the layout of oracle.mxfp4.quantize) -> fp64 [M, N]."""
    a = mxfp4.dequantize(a_packed, a_scales)
    w = mxfp4.dequantize(w_packed, w_scales)
    if a.shape[1] != w.shape[1]:
        raise ValueError("A and W must share K")
    return a @ w.T


def gemm_e4m3(a_codes, a_scale: float, w_codes, w_scale: float) -> np.ndarray:
    """a_codes [M, K], w_codes [N, K] (e4m3 bytes), per-tensor fp32 scales -> fp64 [M, N]
    = a_scale * w_scale * (A_hat @ W_hat^T)."""
    table = e4m3_payload.decode_table()
    a = table[np.asarray(a_codes, dtype=np.uint8)]
    w = table[np.asarray(w_codes, dtype=np.uint8)]
    if np.isnan(a).any() or np.isnan(w).any():
        raise ValueError("NaN codes are outside the contract")
    if a.shape[1] != w.shape[1]:
        raise ValueError("A and W must share K")
    return float(a_scale) * float(w_scale) * (a @ w.T)
