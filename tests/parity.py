"""Helpers shared by the GPU parity tests: run the CUDA path and the fp64 oracle
on the same seeded inputs and compare them (tests only)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from attention_dit_attn_b200 import workloads as wl

# Bounds (from the stated targets): bf16 max|err| <= 2e-2 and relative
# Frobenius error <= 5e-3 for N(0,1) inputs; FP8 relative Frobenius <= 3e-2
# against the oracle on dequantised inputs.  LSE bounds are this build's own.
BF16_MAX_ABS = 2e-2
BF16_REL_F = 5e-3
FP8_REL_F = 3e-2
LSE_ABS = {"bf16": 1e-3, "e4m3": 5e-3}


def run_gpu(inp: wl.Inputs, scale: float, stream=None):
    import attention_dit_attn_b200 as dit
    dev = torch.device("cuda")
    q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
    kw = {}
    if inp.q_scale is not None:
        kw = dict(q_scale=inp.q_scale.to(dev).contiguous(), k_scale=inp.k_scale.to(dev).contiguous(),
                  v_scale=inp.v_scale.to(dev).contiguous())
    o, lse = dit.dit_attn_fwd(q, k, v, scale=scale, stream=stream, **kw)
    torch.cuda.synchronize()
    rc, word = dit.dit_attn_check_device_error()
    assert rc == 0, f"device error word {word:#x}"
    return o.cpu(), lse.cpu()


def run_oracle(inp: wl.Inputs, scale: float, rows: np.ndarray | None = None):
    if inp.q.dtype == torch.bfloat16:
        return oracle.attention(wl.as_bits(inp.q), wl.as_bits(inp.k), wl.as_bits(inp.v), scale,
                                dtype=oracle.BF16, rows=rows)
    return oracle.attention(wl.as_bits(inp.q), wl.as_bits(inp.k), wl.as_bits(inp.v), scale,
                            dtype=oracle.E4M3, q_scale=inp.q_scale.numpy(),
                            k_scale=inp.k_scale.numpy(), v_scale=inp.v_scale.numpy(), rows=rows)


def gather_rows(x: torch.Tensor, rows: np.ndarray | None) -> np.ndarray:
    """x: [B, H, L, ...] -> [B, H, R, ...] float64 at the given per-(b,h) rows."""
    a = x.to(torch.float64).numpy()
    if rows is None:
        return a
    B, H = a.shape[:2]
    out = np.empty((B, H, rows.shape[1]) + a.shape[3:], dtype=np.float64)
    for bh in range(B * H):
        b, h = divmod(bh, H)
        out[b, h] = a[b, h, rows[bh]]
    return out


def compare(o_gpu, lse_gpu, o_ref, lse_ref, rows=None):
    og = gather_rows(o_gpu, rows)
    lg = gather_rows(lse_gpu, rows)
    err = og - o_ref
    rel_f = float(np.linalg.norm(err) / np.linalg.norm(o_ref))
    per_head = np.linalg.norm(err.reshape(err.shape[0] * err.shape[1], -1), axis=1) / \
        np.linalg.norm(o_ref.reshape(err.shape[0] * err.shape[1], -1), axis=1)
    return {
        "rel_f": rel_f,
        "rel_f_worst_head": float(per_head.max()),
        "max_abs": float(np.abs(err).max()),
        "lse_max_abs": float(np.abs(lg - lse_ref).max()),
        "finite": bool(np.isfinite(og).all() and np.isfinite(lg).all()),
    }


def check(metrics: dict, dtype: str):
    assert metrics["finite"], metrics
    if dtype == "bf16":
        assert metrics["rel_f"] <= BF16_REL_F, metrics
        assert metrics["max_abs"] <= BF16_MAX_ABS, metrics
    else:
        assert metrics["rel_f"] <= FP8_REL_F, metrics
    assert metrics["lse_max_abs"] <= LSE_ABS[dtype], metrics
