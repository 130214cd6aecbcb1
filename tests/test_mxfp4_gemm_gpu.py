"""GPU parity of the MXFP4 linear layer (dit_attn_gemm_mxfp4) and of its scale
tiling (dit_attn_mxfp4_tile_scales).

* The tiling is a byte permutation: checked bit for bit against the layout
  formula of include/dit_attn.h, written out here on the CPU.
* The GEMM is checked element by element against the exact fp64 oracle
  (oracle/lowp_gemm.py) on operands drawn directly as codes and scales.
  Bound, from the arithmetic: every scaled E2M1 x E2M1 product is exact in
  fp32; the K products are summed in fp32 on the tensor cores (|error| <=
  K 2^-24 S for any order of additions, S = sum_k |a_k w_k|); the result is
  rounded to bf16 (2^-9 relative).  Allowed: 2^-8 |y| + 2 K 2^-24 S per
  element, and a relative Frobenius error of 2^-8 over the output.
* End to end: bf16 activations quantised on the GPU (dit_attn_mxfp4_quantize),
  tiled, multiplied, against the oracle's own quantisation and GEMM."""
import numpy as np
import pytest
import torch

from attention_dit_attn_b200 import workloads as wl
from oracle import lowp_gemm, mxfp4

pytestmark = pytest.mark.gpu


def tile_cpu(plain: np.ndarray, K: int) -> np.ndarray:
    """The tiled layout, straight from its definition."""
    rows = plain.shape[0]
    kb = K // 32
    G = 2 * ((K + 255) // 256)
    out = np.zeros(((rows + 127) // 128) * G * 512, dtype=np.uint8)
    for r in range(rows):
        for b in range(kb):
            out[((r // 128) * G + b // 4) * 512 + 16 * (r % 32) + 4 * ((r % 128) // 32) + b % 4] = plain[r, b]
    return out


def _gemm_gpu(a, sa, w, sw, K):
    import attention_dit_attn_b200 as dit
    dev = torch.device("cuda")
    ta = dit.dit_attn_mxfp4_tile_scales(sa.to(dev), K)
    tw = dit.dit_attn_mxfp4_tile_scales(sw.to(dev), K)
    y = dit.dit_attn_gemm_mxfp4(a.to(dev), ta, w.to(dev), tw)
    torch.cuda.synchronize()
    rc, word = dit.dit_attn_gemm_check_device_error()
    assert rc == 0, f"device error word {word:#x}"
    return y.cpu()


def _check(y_gpu, a, sa, w, sw, rows=None):
    an, san = a.numpy(), sa.numpy()
    if rows is not None:
        an, san, y_gpu = an[rows], san[rows], y_gpu[rows]
    ref = lowp_gemm.gemm_mxfp4(an, san, w.numpy(), sw.numpy())
    S = np.abs(mxfp4.dequantize(an, san)) @ np.abs(mxfp4.dequantize(w.numpy(), sw.numpy())).T
    K = 2 * an.shape[1]
    got = y_gpu.to(torch.float64).numpy()
    assert np.isfinite(got).all()
    err = np.abs(got - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 2 * K * 2.0 ** -24 * S
    worst = float((err / np.maximum(bound, 1e-300)).max())
    assert worst <= 1.0, f"error {worst:.3f} x the bound"
    rel_f = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    assert rel_f <= 2.0 ** -8, rel_f


@pytest.mark.parametrize("rows,K", [(1, 32), (127, 96), (300, 288), (129, 3072)])
def test_tile_scales_is_the_layout(cuda_lib, rows, K):
    import attention_dit_attn_b200 as dit
    g = torch.Generator().manual_seed(rows + K)
    plain = torch.randint(0, 256, (rows, K // 32), generator=g, dtype=torch.int32).to(torch.uint8)
    tiled = dit.dit_attn_mxfp4_tile_scales(plain.cuda(), K)
    torch.cuda.synchronize()
    n = dit.dit_attn_mxfp4_tiled_scale_bytes(rows, K)
    assert np.array_equal(tiled.cpu().numpy()[:n], tile_cpu(plain.numpy(), K))


@pytest.mark.parametrize("M,N,K", [
    (1, 8, 32),            # one row, one partial tile, one partial K stage
    (200, 136, 288),       # ragged M, N past one 128-row scale block, a half-empty last K stage
    (300, 264, 512),       # two N tiles, the second with a single scale block
    (1000, 768, 1024),     # several tiles in M and N
    (128, 256, 3072),      # one tile, a long K
    (256, 256, 3584),      # K past what TMEM holds of W's scales: per-stage W scales
    (300, 19200, 64),      # more N tiles than CTA pairs: per-stage W scales
    (1100, 264, 3328),     # the longest K with resident W scales, pairs sharing an N tile
])
def test_gemm_mxfp4_matches_the_oracle(cuda_lib, M, N, K):
    a, sa, w, sw = wl.gemm_operands_mxfp4(M, N, K, seed=M + N + K)
    y = _gemm_gpu(a, sa, w, sw, K)
    assert y.shape == (M, N) and y.dtype == torch.bfloat16
    _check(y, a, sa, w, sw)


def test_gemm_mxfp4_full_projection_size_sampled_rows(cuda_lib):
    """flux_2048_cfg's projection shape (M = 2 x 16896 tokens, N = K = 3072); the oracle
    checks 96 sampled rows."""
    M, N, K = wl.GEMM_SHAPES["flux_2048_cfg_proj"]
    a, sa, w, sw = wl.gemm_operands_mxfp4(M, N, K, seed=5)
    y = _gemm_gpu(a, sa, w, sw, K)
    rows = np.sort(np.random.default_rng(6).choice(M, 96, replace=False))
    rows[0], rows[-1] = 0, M - 1
    _check(y, a, sa, w, sw, rows)


def test_quantise_tile_multiply_end_to_end(cuda_lib):
    """bf16 activations and weights through the GPU quantiser, tiling and GEMM, against
    the oracle's quantisation (oracle/mxfp4.py) and GEMM of the same bf16 values."""
    import attention_dit_attn_b200 as dit
    g = torch.Generator().manual_seed(21)
    M, N, K = 96, 72, 160
    x = (torch.randn((M, K), generator=g) * 3).to(torch.bfloat16)
    wt = (torch.randn((N, K), generator=g) / 8).to(torch.bfloat16)
    qa, sa = dit.dit_attn_mxfp4_quantize(x.cuda())
    qw, sw = dit.dit_attn_mxfp4_quantize(wt.cuda())
    y = dit.dit_attn_gemm_mxfp4(qa, dit.dit_attn_mxfp4_tile_scales(sa, K), qw, dit.dit_attn_mxfp4_tile_scales(sw, K))
    torch.cuda.synchronize()
    ra, rsa = mxfp4.quantize(x.to(torch.float64).numpy())
    rw, rsw = mxfp4.quantize(wt.to(torch.float64).numpy())
    _check(y.cpu(), torch.from_numpy(ra), torch.from_numpy(rsa), torch.from_numpy(rw), torch.from_numpy(rsw))


def test_gemm_mxfp4_is_deterministic_and_writes_only_y(cuda_lib):
    import attention_dit_attn_b200 as dit
    M, N, K = 700, 392, 512
    a, sa, w, sw = wl.gemm_operands_mxfp4(M, N, K, seed=12)
    ta = dit.dit_attn_mxfp4_tile_scales(sa.cuda(), K)
    tw = dit.dit_attn_mxfp4_tile_scales(sw.cuda(), K)
    ad, wd = a.cuda(), w.cuda()
    guard = torch.full((M * N + 4096,), 7.0, dtype=torch.bfloat16, device="cuda")
    y = guard[:M * N].view(M, N)
    dit.dit_attn_gemm_mxfp4(ad, ta, wd, tw, y=y)
    y1 = y.clone()
    dit.dit_attn_gemm_mxfp4(ad, ta, wd, tw, y=y)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y.view(torch.int16))
    assert bool((guard[M * N:] == 7.0).all())
    _check(y.cpu(), a, sa, w, sw)


def test_gemm_mxfp4_large_activation_takes_the_per_stage_path_sampled_rows(cuda_lib):
    """Four times the projection's tokens (M = 135168, 208 MB of codes, more than
    the 64 MB for which W's scales are kept in TMEM): the per-stage scale path on
    a full-size launch; the oracle checks 64 sampled rows."""
    M, N, K = 4 * wl.GEMM_SHAPES["flux_2048_cfg_proj"][0], 3072, 3072
    a, sa, w, sw = wl.gemm_operands_mxfp4(M, N, K, seed=8)
    y = _gemm_gpu(a, sa, w, sw, K)
    rows = np.sort(np.random.default_rng(9).choice(M, 64, replace=False))
    rows[0], rows[-1] = 0, M - 1
    _check(y, a, sa, w, sw, rows)
