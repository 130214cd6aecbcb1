"""GPU parity of the FP8 linear-layer GEMM (dit_attn_gemm_fp8) against the exact
fp64 oracle (oracle/lowp_gemm.py), element by element.

Bound, from the arithmetic: the kernel forms every product exactly, sums the K
products in fp32 on the tensor cores (|error| <= K * 2^-24 * S for any order of
K fp32 additions, S = a_scale * w_scale * sum_k |a_k w_k|), applies the scale
in fp32 and rounds to bf16 (half an ulp: 2^-9 relative).  The test allows
2^-8 |y| + 2 K 2^-24 S per element, plus a relative Frobenius error of 2^-8 over
the whole output (bf16 rounding dominates)."""
import numpy as np
import pytest
import torch

from attention_dit_attn_b200 import workloads as wl
from oracle import lowp_gemm

pytestmark = pytest.mark.gpu


def _run(a, w, sa, sw):
    import attention_dit_attn_b200 as dit
    y = dit.dit_attn_gemm_fp8(a.cuda(), w.cuda(), sa, sw)
    torch.cuda.synchronize()
    rc, word = dit.dit_attn_gemm_check_device_error()
    assert rc == 0, f"device error word {word:#x}"
    return y.cpu()


def _check(y_gpu, a, w, sa, sw, rows=None):
    ac = a.view(torch.uint8).numpy()
    wc = w.view(torch.uint8).numpy()
    if rows is not None:
        ac = ac[rows]
        y_gpu = y_gpu[rows]
    ref = lowp_gemm.gemm_e4m3(ac, sa, wc, sw)
    table = np.abs(np.nan_to_num(lowp_gemm.e4m3_payload.decode_table()))
    S = sa * sw * (table[ac] @ table[wc].T)
    K = ac.shape[1]
    got = y_gpu.to(torch.float64).numpy()
    err = np.abs(got - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 2 * K * 2.0 ** -24 * S
    worst = float((err / np.maximum(bound, 1e-300)).max())
    assert np.isfinite(got).all()
    assert worst <= 1.0, f"error {worst:.3f} x the bound"
    rel_f = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    assert rel_f <= 2.0 ** -8, rel_f
    return rel_f


@pytest.mark.parametrize("M,N,K", [
    (1, 8, 16),            # one row, one partial tile, one partial K stage
    (300, 264, 208),       # ragged in M, N and K: tail tiles and a 80-byte last K stage
    (1000, 768, 512),      # several tiles in M and N, full K stages
    (256, 256, 3072),      # one pair tile, a long K
    (4099, 520, 96),       # many M tiles, N just past two tiles
])
def test_gemm_fp8_matches_the_oracle(cuda_lib, M, N, K):
    a, sa, w, sw = wl.gemm_operands_e4m3(M, N, K, seed=M + N + K)
    y = _run(a, w, sa, sw)
    assert y.shape == (M, N) and y.dtype == torch.bfloat16
    _check(y, a, w, sa, sw)


def test_gemm_fp8_full_projection_size_sampled_rows(cuda_lib):
    """flux_2048_cfg's projection shape (M = 2 x 16896 tokens, N = K = 3072) in the
    launch configuration the bench times; the oracle checks 96 sampled rows."""
    M, N, K = wl.GEMM_SHAPES["flux_2048_cfg_proj"]
    a, sa, w, sw = wl.gemm_operands_e4m3(M, N, K, seed=3)
    y = _run(a, w, sa, sw)
    rows = np.sort(np.random.default_rng(5).choice(M, 96, replace=False))
    rows[0], rows[-1] = 0, M - 1
    _check(y, a, w, sa, sw, rows)


def test_gemm_fp8_is_deterministic_and_writes_only_y(cuda_lib):
    import attention_dit_attn_b200 as dit
    M, N, K = 700, 392, 256
    a, sa, w, sw = wl.gemm_operands_e4m3(M, N, K, seed=11)
    ad, wd = a.cuda(), w.cuda()
    guard = torch.full((M * N + 4096,), 7.0, dtype=torch.bfloat16, device="cuda")
    y = guard[:M * N].view(M, N)
    dit.dit_attn_gemm_fp8(ad, wd, sa, sw, y=y)
    y1 = y.clone()
    dit.dit_attn_gemm_fp8(ad, wd, sa, sw, y=y)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y.view(torch.int16))
    assert bool((guard[M * N:] == 7.0).all())
    _check(y.cpu(), a, w, sa, sw)
