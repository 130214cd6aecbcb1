"""Seeded synthetic inputs for DiT joint attention.

This module only draws and lays out input tensors.  It holds none of the
attention arithmetic, so both the CUDA path's tests/bench and the fp64 oracle
can take their inputs from it.

The five workloads mirror the DiT attention shapes the xDiT pages run
(FLUX, Stable Diffusion 3.5 and Wan video models on the page "How to Scale
Diffusion Inference Across AMD RDNA 4 GPUs", introduction; FLUX.1-dev at
1024x768 on the page "Accelerating Diffusers and xDiT Image Generation with
MXFP4 using AMD Quark on AMD Instinct MI350 GPUs", section "Benchmark
Script").  Only their shapes are used: no model weights, prompts or datasets.
Token counts are text tokens (prompt embedding) followed by image/video patch
tokens, concatenated into one joint sequence of length L.

Recipe (all draws on the CPU with ``torch.Generator().manual_seed(seed)``,
fp32, in the order q, k, v, then U, W when a low-rank component is asked for):
  * q, k, v ~ N(0, 1), shape [B, H, L, D];
  * ``text_rows`` > 0: rows [0, text_rows) of q and k (not v) are multiplied by
    ``text_scale`` (widens the logit range of the text tokens);
  * ``lowrank`` = r > 0: U ~ N(0,1) [B, L, r], W ~ N(0,1)/sqrt(r) [H, r, D],
    Z[b,h] = U[b] @ W[h] is added to q and k (the same Z to both), giving
    peaked softmax rows;
  * bf16 workloads round to bf16 (round-to-nearest-even, torch's cast);
  * e4m3 workloads quantise each (b, h) head of each tensor separately:
    s = max|x| / 448 (fp32), x_hat = e4m3(clamp(x / s, -448, 448)) with
    round-to-nearest-even; the dequantised value is s * x_hat.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

E4M3_MAX = 448.0


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    L: int
    D: int
    dtype: str            # "bf16" or "e4m3"
    seed: int
    text_rows: int = 0    # leading text tokens (part of L)
    text_scale: float = 1.0
    lowrank: int = 0
    sampled_rows: int = 0  # 0: parity compares every query row

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def flops(self) -> float:
        """Algorithmic FLOPs of one attention call: QK^T plus PV, 2 each per MAC."""
        return 4.0 * self.B * self.H * float(self.L) ** 2 * self.D


WORKLOADS = {
    "tiny_256": Workload("tiny_256", B=1, H=2, L=256, D=64, dtype="bf16", seed=1001),
    "flux_1024x768": Workload("flux_1024x768", B=1, H=24, L=512 + 3072, D=128, dtype="bf16",
                              seed=1002, text_rows=512),
    "flux_2048_cfg": Workload("flux_2048_cfg", B=2, H=24, L=512 + 16384, D=128, dtype="bf16",
                              seed=1003, text_rows=512, text_scale=2.0, sampled_rows=512),
    "sd35_1024_fp8": Workload("sd35_1024_fp8", B=2, H=38, L=154 + 4096, D=64, dtype="e4m3",
                              seed=1004, text_rows=154),
    "wan_720p_81f": Workload("wan_720p_81f", B=1, H=40, L=21 * 45 * 80, D=128, dtype="bf16",
                             seed=1005, lowrank=8, sampled_rows=512),
}
# Same five, in the order the workload list gives them.
ORDER = ["tiny_256", "flux_1024x768", "flux_2048_cfg", "sd35_1024_fp8", "wan_720p_81f"]

# Profiling-size slices of the workloads above (same L and D, fewer heads): inputs
# still larger than the 126 MB L2, small enough for a multi-pass ncu capture.
PROFILE_CASES = {
    "flux_2048_h16": Workload("flux_2048_h16", B=1, H=16, L=512 + 16384, D=128, dtype="bf16",
                              seed=1003, text_rows=512, text_scale=2.0),
}
ALL = {**WORKLOADS, **PROFILE_CASES}


@dataclass
class Inputs:
    q: torch.Tensor       # bf16 or float8_e4m3fn, [B, H, L, D], CPU
    k: torch.Tensor
    v: torch.Tensor
    q_scale: torch.Tensor | None  # fp32 [B, H] (e4m3 only)
    k_scale: torch.Tensor | None
    v_scale: torch.Tensor | None


def quantize_e4m3_per_head(x: torch.Tensor):
    """Per-(b,h) absmax quantisation to e4m3: returns (codes, fp32 scales [B,H])."""
    B, H = x.shape[:2]
    amax = x.abs().reshape(B, H, -1).amax(dim=-1).to(torch.float32)
    s = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    y = (x / s[:, :, None, None]).clamp(-E4M3_MAX, E4M3_MAX)
    return y.to(torch.float8_e4m3fn), s.contiguous()


def generate(B: int, H: int, L: int, D: int, dtype: str = "bf16", seed: int = 0,
             text_rows: int = 0, text_scale: float = 1.0, lowrank: int = 0) -> Inputs:
    """Draw one set of q/k/v following the recipe in the module docstring."""
    if dtype not in ("bf16", "e4m3"):
        raise ValueError(f"dtype must be bf16 or e4m3, got {dtype!r}")
    g = torch.Generator().manual_seed(int(seed))
    shape = (B, H, L, D)
    xs = []
    for _ in range(3):
        xs.append(torch.randn(shape, generator=g, dtype=torch.float32))
    q, k, v = xs
    if text_rows > 0 and text_scale != 1.0:
        q[:, :, :text_rows] *= text_scale
        k[:, :, :text_rows] *= text_scale
    if lowrank > 0:
        U = torch.randn((B, L, lowrank), generator=g, dtype=torch.float32)
        W = torch.randn((H, lowrank, D), generator=g, dtype=torch.float32) / math.sqrt(lowrank)
        for b in range(B):
            for h in range(H):
                z = U[b] @ W[h]
                q[b, h] += z
                k[b, h] += z
    if dtype == "bf16":
        return Inputs(q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16),
                      None, None, None)
    (qq, qs), (kq, ks), (vq, vs) = (quantize_e4m3_per_head(t) for t in (q, k, v))
    return Inputs(qq, kq, vq, qs, ks, vs)


def generate_workload(w: Workload) -> Inputs:
    return generate(w.B, w.H, w.L, w.D, w.dtype, w.seed, w.text_rows, w.text_scale, w.lowrank)


def sample_rows(B: int, H: int, L: int, n: int, seed: int) -> np.ndarray:
    """Per (b,h): n distinct query rows = {0, L-1} plus n-2 drawn without
    replacement from [1, L-1) with numpy PCG64(seed ^ (b*H + h)); sorted.
    Returns int64 [B*H, n].  n >= L gives every row."""
    if n >= L:
        return np.tile(np.arange(L, dtype=np.int64), (B * H, 1))
    out = np.empty((B * H, n), dtype=np.int64)
    for bh in range(B * H):
        rng = np.random.Generator(np.random.PCG64(seed ^ bh))
        mid = rng.choice(np.arange(1, L - 1, dtype=np.int64), size=n - 2, replace=False)
        out[bh] = np.sort(np.concatenate([[0, L - 1], mid]))
    return out


def as_bits(t: torch.Tensor) -> np.ndarray:
    """Raw storage of a bf16 (uint16) or e4m3 (uint8) tensor as a numpy array."""
    if t.dtype == torch.bfloat16:
        return t.contiguous().view(torch.uint16).numpy()
    if t.dtype == torch.float8_e4m3fn:
        return t.contiguous().view(torch.uint8).numpy()
    raise TypeError(f"unsupported dtype {t.dtype}")


# Linear-layer operands of the low-precision GEMMs: the DiT's QKV / output
# projection shapes, M = B * L tokens by K = N = H * D features (FLUX: 3072).
GEMM_SHAPES = {
    "flux_2048_cfg_proj": (2 * (512 + 16384), 3072, 3072),     # (M, N, K)
    "flux_1024x768_proj": (512 + 3072, 3072, 3072),
}


def gemm_operands_e4m3(M: int, N: int, K: int, seed: int = 0):
    """A [M, K] and W [N, K] drawn N(0,1) (W scaled by 1/sqrt(K), as a trained
    linear layer's weights are), each quantised per tensor to e4m3:
    s = max|x| / 448, codes = e4m3(x / s) (nearest-even, torch's cast).
    Returns (a codes, a_scale, w codes, w_scale); codes as torch.float8_e4m3fn."""
    g = torch.Generator().manual_seed(int(seed))
    a = torch.randn((M, K), generator=g, dtype=torch.float32)
    w = torch.randn((N, K), generator=g, dtype=torch.float32) / math.sqrt(K)
    out = []
    for x in (a, w):
        amax = float(x.abs().max())
        s = amax / E4M3_MAX if amax > 0 else 1.0
        s = float(torch.tensor(s, dtype=torch.float32))
        out += [(x / s).clamp(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn), s]
    return tuple(out)


def gemm_operands_mxfp4(M: int, N: int, K: int, seed: int = 0, scale_spread: int = 6):
    """MXFP4 operands drawn directly in their stored form (no conversion): packed
    E2M1 codes, two uniform random 4-bit codes per byte (every code is a valid
    E2M1 value, -0 included), and E8M0 block scales uniform in
    [127 - scale_spread, 127 + scale_spread] for A and [127 - scale_spread - 4,
    127 + scale_spread - 4] for W (smaller weights).  Layout as the quantiser
    writes it: A codes [M, K/2], A scales [M, K/32], W codes [N, K/2],
    W scales [N, K/32], all uint8."""
    if K % 32:
        raise ValueError("K must be a multiple of 32")
    g = torch.Generator().manual_seed(int(seed))
    a = torch.randint(0, 256, (M, K // 2), generator=g, dtype=torch.int32).to(torch.uint8)
    w = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.int32).to(torch.uint8)
    sa = torch.randint(127 - scale_spread, 127 + scale_spread + 1, (M, K // 32), generator=g,
                       dtype=torch.int32).to(torch.uint8)
    sw = torch.randint(123 - scale_spread, 123 + scale_spread + 1, (N, K // 32), generator=g,
                       dtype=torch.int32).to(torch.uint8)
    return a, sa, w, sw
