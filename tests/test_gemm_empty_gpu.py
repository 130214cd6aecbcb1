"""Empty activations (M = 0 rows) through both linear-layer GEMMs and the scale
tiling: every call succeeds, launches nothing that writes, and leaves the
weight-side buffers as they were."""
import pytest
import torch

from attention_dit_attn_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def test_gemm_fp8_with_no_rows(cuda_lib):
    import attention_dit_attn_b200 as dit
    N, K = 264, 208
    _, _, w, sw = wl.gemm_operands_e4m3(8, N, K, seed=1)
    a = torch.empty((0, K), dtype=torch.float8_e4m3fn, device="cuda")
    y = dit.dit_attn_gemm_fp8(a, w.cuda(), 1.0, sw)
    torch.cuda.synchronize()
    assert y.shape == (0, N)
    rc, word = dit.dit_attn_gemm_check_device_error()
    assert rc == 0, f"device error word {word:#x}"


def test_gemm_mxfp4_and_tiling_with_no_rows(cuda_lib):
    import attention_dit_attn_b200 as dit
    N, K = 136, 288
    _, _, w, sw = wl.gemm_operands_mxfp4(8, N, K, seed=2)
    tw = dit.dit_attn_mxfp4_tile_scales(sw.cuda(), K)
    tw_before = tw.clone()
    a = torch.empty((0, K // 2), dtype=torch.uint8, device="cuda")
    sa = torch.empty((0, K // 32), dtype=torch.uint8, device="cuda")
    ta = dit.dit_attn_mxfp4_tile_scales(sa, K)
    assert dit.dit_attn_mxfp4_tiled_scale_bytes(0, K) == 0
    y = dit.dit_attn_gemm_mxfp4(a, ta, w.cuda(), tw)
    torch.cuda.synchronize()
    assert y.shape == (0, N)
    assert torch.equal(tw, tw_before)
    rc, word = dit.dit_attn_gemm_check_device_error()
    assert rc == 0, f"device error word {word:#x}"
