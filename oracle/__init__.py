"""fp64 CPU oracle for DiT joint attention: TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports it, and this package imports nothing from
the product path.

The arithmetic lives in ``oracle_attn.c`` (plain C, fp64, libm ``exp``/``log``,
no fast-math).  It computes the textbook scaled dot-product attention that the
xDiT pages' attention backend computes (page "How to Scale Diffusion Inference
Across AMD RDNA 4 GPUs", section "Select an Attention Backend and Compile the
Transformer"; the pages cite "Attention Is All You Need" and FlashAttention-2
in the reference list of "xDiT: an Inference Engine for Diffusion Transformers
(DiTs) with Massive Parallelism"):

    s_j = scale * q . k_j,   p_j = exp(s_j - max s),   o = sum_j p_j v_j / sum_j p_j,
    lse = max s + log(sum_j p_j)

This module only marshals arrays into that C code and builds it with gcc.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle_attn.c")
_LIB = os.path.join(_HERE, "liboracle_attn.so")

BF16, E4M3, F64 = 0, 1, 2

_lib = None


def build(force: bool = False) -> str:
    """Compile oracle_attn.c with gcc (-O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        lib.oracle_bf16_to_f64.restype = ctypes.c_double
        lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_e4m3_to_f64.restype = ctypes.c_double
        lib.oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        lib.oracle_decode_bf16.restype = None
        lib.oracle_decode_bf16.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64]
        lib.oracle_decode_e4m3.restype = None
        lib.oracle_decode_e4m3.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                           ctypes.c_double]
        lib.oracle_attention.restype = ctypes.c_int
        lib.oracle_attention.argtypes = [
            ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
            ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        lib.oracle_max_threads.restype = ctypes.c_int
        lib.oracle_max_threads.argtypes = []
        _lib = lib
    return _lib


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Decode uint16 bf16 bit patterns to fp64 (exact)."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(bits.shape, dtype=np.float64)
    _load().oracle_decode_bf16(_ptr(bits), _ptr(out), bits.size)
    return out


def e4m3_to_f64(codes: np.ndarray, scale: float = 1.0) -> np.ndarray:
    """Decode OCP FP8 E4M3 codes to fp64 and multiply by ``scale`` (exact)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(codes.shape, dtype=np.float64)
    _load().oracle_decode_e4m3(_ptr(codes), _ptr(out), codes.size, float(scale))
    return out


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float, *, dtype: int,
              q_scale: np.ndarray | None = None, k_scale: np.ndarray | None = None,
              v_scale: np.ndarray | None = None, rows: np.ndarray | None = None,
              nthreads: int = 0):
    """Run the fp64 oracle.

    q, k, v: [B, H, L, D] arrays holding bf16 bit patterns (uint16, dtype=BF16),
    E4M3 codes (uint8, dtype=E4M3, with [B*H] fp32 dequant scales) or fp64
    values (dtype=F64).  ``rows``: None for every query row, else an int64
    [B*H, R] array of query indices.  Returns (o [B, H, R, D], lse [B, H, R]).
    """
    want = {BF16: np.uint16, E4M3: np.uint8, F64: np.float64}[dtype]
    q = np.ascontiguousarray(q, dtype=want)
    k = np.ascontiguousarray(k, dtype=want)
    v = np.ascontiguousarray(v, dtype=want)
    if q.ndim != 4 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError(f"q/k/v must share one [B,H,L,D] shape, got {q.shape} {k.shape} {v.shape}")
    B, H, L, D = q.shape
    scales = [None, None, None]
    if dtype == E4M3:
        scales = [np.ascontiguousarray(s, dtype=np.float32).reshape(B * H)
                  for s in (q_scale, k_scale, v_scale)]
    if rows is None:
        nrows, rows_arr = L, None
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64).reshape(B * H, -1)
        nrows = rows_arr.shape[1]
    o = np.empty((B, H, nrows, D), dtype=np.float64)
    lse = np.empty((B, H, nrows), dtype=np.float64)
    rc = _load().oracle_attention(dtype, _ptr(q), _ptr(k), _ptr(v),
                                  _ptr(scales[0]), _ptr(scales[1]), _ptr(scales[2]),
                                  B, H, L, D, float(scale), _ptr(rows_arr), nrows,
                                  _ptr(o), _ptr(lse), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_attention failed with code {rc}")
    return o, lse
