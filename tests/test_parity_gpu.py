"""GPU parity: the sm_100a kernel (through the C ABI) against the fp64 oracle.

Small shapes compare every output element; the five DiT workloads run at
their full sizes in the same launch configuration the bench times, comparing
every row (tiny_256, flux_1024x768) or 512 seeded sampled query rows per head
(flux_2048_cfg, sd35_1024_fp8, wan_720p_81f).
"""
import math

import numpy as np
import pytest
import torch

import parity
from attention_dit_attn_b200 import workloads as wl

pytestmark = pytest.mark.gpu

SMALL = [
    # B, H, L, D, dtype            (ragged tails, single key, L < tile, several tiles)
    (1, 1, 128, 128, "bf16"),
    (1, 1, 1, 128, "bf16"),
    (1, 2, 129, 128, "bf16"),
    (1, 1, 255, 128, "bf16"),
    (1, 1, 257, 128, "bf16"),
    (2, 3, 1000, 128, "bf16"),
    (1, 1, 2, 64, "bf16"),
    (1, 2, 700, 64, "bf16"),
    (3, 2, 385, 64, "bf16"),
    (1, 1, 33, 64, "bf16"),             # D = 64: four key splits, one key in the second
    (1, 2, 353, 64, "e4m3"),            # last tile: splits 0-2 valid, split 3 one key
    (1, 1, 1, 64, "e4m3"),
    (2, 2, 300, 64, "e4m3"),
    (1, 2, 1000, 64, "e4m3"),
    (1, 2, 1000, 128, "e4m3"),
    (1, 1, 77, 128, "e4m3"),
]


@pytest.mark.parametrize("B,H,L,D,dtype", SMALL)
def test_small_shapes_match_oracle(cuda_lib, B, H, L, D, dtype):
    inp = wl.generate(B, H, L, D, dtype, seed=L * 7 + D + B * 3 + H)
    scale = 1.0 / math.sqrt(D)
    o, lse = parity.run_gpu(inp, scale)
    o_ref, lse_ref = parity.run_oracle(inp, scale)
    parity.check(parity.compare(o, lse, o_ref, lse_ref), dtype)


def test_peaked_rows_with_lazy_rescale(cuda_lib):
    """Low-rank shared component (peaked rows, growing maxima) and text rows x2."""
    inp = wl.generate(1, 2, 1500, 128, "bf16", seed=11, text_rows=200, text_scale=2.0, lowrank=8)
    o, lse = parity.run_gpu(inp, 1 / math.sqrt(128))
    o_ref, lse_ref = parity.run_oracle(inp, 1 / math.sqrt(128))
    parity.check(parity.compare(o, lse, o_ref, lse_ref), "bf16")


def _jump_inputs(D: int, dtype: str, seed: int):
    """Rows whose running max jumps by far more than the lazy-rescale guard in
    later key tiles.  Every query has q[..., 0] = 8 (one head) or 2 (the other);
    key 300 (third tile) and key 650 (sixth tile) get k[..., 0] = 80 and 150, so
    their logits exceed the first tile's by tens to hundreds of log2 units: past
    the bf16 guard (2^64), past MUFU's and the cubic's range (2^128), and far
    past the f16 guard (2^15)."""
    g = torch.Generator().manual_seed(seed)
    B, H, L = 1, 2, 700
    q = torch.randn((B, H, L, D), generator=g) * 0.5
    k = torch.randn((B, H, L, D), generator=g) * 0.5
    v = torch.randn((B, H, L, D), generator=g)
    q[:, 0, :, 0] = 8.0
    q[:, 1, :, 0] = 2.0
    k[:, :, 300, 0] = 80.0
    k[:, :, 650, 0] = 150.0
    if dtype == "bf16":
        return wl.Inputs(q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16), None, None, None)
    (qq, qs), (kq, ks), (vq, vs) = (wl.quantize_e4m3_per_head(t) for t in (q, k, v))
    return wl.Inputs(qq, kq, vq, qs, ks, vs)


@pytest.mark.parametrize("D,dtype", [(128, "bf16"), (64, "bf16"), (64, "e4m3"), (128, "e4m3")])
def test_max_jumps_past_the_lazy_rescale_guard(cuda_lib, D, dtype):
    """The running max of a row is kept from its first key tile; later tiles are
    only checked through the sum of their p.  Jumps of tens to hundreds of log2
    units in later tiles must take the rescale path and still match the oracle."""
    inp = _jump_inputs(D, dtype, seed=40 + D)
    o, lse = parity.run_gpu(inp, 1 / math.sqrt(D))
    assert torch.isfinite(o.to(torch.float32)).all() and torch.isfinite(lse).all()
    o_ref, lse_ref = parity.run_oracle(inp, 1 / math.sqrt(D))
    parity.check(parity.compare(o, lse, o_ref, lse_ref), dtype)


def test_scale_zero_gives_mean_of_v(cuda_lib):
    inp = wl.generate(1, 2, 300, 128, "bf16", seed=12)
    o, lse = parity.run_gpu(inp, 0.0)
    mean = inp.v.to(torch.float64).mean(dim=2, keepdim=True).expand_as(o)
    assert torch.allclose(o.to(torch.float64), mean, atol=2e-2, rtol=0)
    assert torch.allclose(lse.to(torch.float64), torch.full_like(lse, math.log(300), dtype=torch.float64),
                          atol=1e-4, rtol=0)


def test_repeat_calls_are_bitwise_deterministic(cuda_lib):
    inp = wl.generate(1, 3, 777, 128, "bf16", seed=13)
    o1, l1 = parity.run_gpu(inp, 0.1)
    o2, l2 = parity.run_gpu(inp, 0.1)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_writes_stay_inside_o_and_lse(cuda_lib):
    """Rows >= L of the last query tile are not stored: guard words after O/LSE survive."""
    import attention_dit_attn_b200 as dit
    B, H, L, D = 1, 2, 200, 128
    inp = wl.generate(B, H, L, D, "bf16", seed=14)
    dev = torch.device("cuda")
    q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
    n, guard = B * H * L * D, 4096
    obuf = torch.full((n + guard,), 7.0, dtype=torch.bfloat16, device=dev)
    lbuf = torch.full((B * H * L + guard,), 7.0, dtype=torch.float32, device=dev)
    dit.dit_attn_fwd(q, k, v, obuf[:n].view(B, H, L, D), lbuf[:B * H * L], scale=0.1)
    torch.cuda.synchronize()
    assert torch.all(obuf[n:] == 7.0) and torch.all(lbuf[B * H * L:] == 7.0)
    o_ref, lse_ref = parity.run_oracle(inp, 0.1)
    parity.check(parity.compare(obuf[:n].view(B, H, L, D).cpu(), lbuf[:B * H * L].view(B, H, L).cpu(),
                                o_ref, lse_ref), "bf16")


def test_lse_may_be_null_and_side_stream(cuda_lib):
    import attention_dit_attn_b200 as dit
    inp = wl.generate(1, 2, 260, 64, "bf16", seed=15)
    dev = torch.device("cuda")
    q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o, lse = dit.dit_attn_fwd(q, k, v, scale=0.125, want_lse=False, stream=s)
    s.synchronize()
    assert lse is None
    o_ref, lse_ref = parity.run_oracle(inp, 0.125)
    m = parity.compare(o.cpu(), torch.from_numpy(lse_ref), o_ref, lse_ref)
    parity.check(m, "bf16")


def test_device_wait_timeout_is_reported_and_context_survives(cuda_lib):
    import attention_dit_attn_b200 as dit
    assert dit.dit_attn_check_device_error()[0] == 0
    assert dit.dit_attn_selftest_wait_timeout(2_000_000) == 0      # 2 ms limit, nothing arrives
    rc, word = dit.dit_attn_check_device_error()
    assert rc == 7 and (word & 0xFF) == 7 and (word >> 8) & 0xFF == 11
    assert dit.dit_attn_check_device_error()[0] == 0               # cleared
    test_small_shapes_match_oracle(cuda_lib, 1, 1, 300, 128, "bf16")


def test_argument_errors_on_gpu(cuda_lib):
    import attention_dit_attn_b200 as dit
    x = torch.zeros(1 * 1 * 64 * 128 + 8, dtype=torch.bfloat16, device="cuda")
    p = x.data_ptr()
    assert dit.dit_attn_fwd_ptr(p + 2, p, p, p, None, 1, 1, 64, 128, 0.1, 0) == 4      # misaligned q
    assert dit.dit_attn_fwd_ptr(p, p, p, p, None, 1, 1, 64, 96, 0.1, 0) == 2           # D=96
    assert dit.dit_attn_fwd_ptr(p, p, p, p, None, 1, 1, 64, 128, -1.0, 0) == 8         # scale<0
    assert dit.dit_attn_fwd_ptr(p, p, p, p, None, 1, 1, 64, 128, 0.1, 1) == 1          # fp8 no scales
    assert dit.dit_attn_fwd_ptr(p, p, p, p, None, 1, 1, 64, 128, 0.1, 0, p) == 3       # bf16 + scale
    assert dit.dit_attn_fwd_ptr(p, p, p, p, None, 1, 1, 0, 128, 0.1, 0) == 2           # L=0


# ------------------------------------------------------------------ the five DiT workloads

def _workload_case(name: str):
    w = wl.WORKLOADS[name]
    inp = wl.generate_workload(w)
    rows = None if w.sampled_rows == 0 else wl.sample_rows(w.B, w.H, w.L, w.sampled_rows, w.seed)
    o, lse = parity.run_gpu(inp, w.scale)
    o_ref, lse_ref = parity.run_oracle(inp, w.scale, rows=rows)
    m = parity.compare(o, lse, o_ref, lse_ref, rows)
    print(name, m)
    parity.check(m, w.dtype)


def test_workload_tiny_256(cuda_lib):
    _workload_case("tiny_256")


def test_workload_flux_1024x768(cuda_lib):
    _workload_case("flux_1024x768")


def test_workload_sd35_1024_fp8_sampled_rows(cuda_lib):
    w = wl.WORKLOADS["sd35_1024_fp8"]
    inp = wl.generate_workload(w)
    rows = wl.sample_rows(w.B, w.H, w.L, 512, w.seed)
    o, lse = parity.run_gpu(inp, w.scale)
    o_ref, lse_ref = parity.run_oracle(inp, w.scale, rows=rows)
    m = parity.compare(o, lse, o_ref, lse_ref, rows)
    print("sd35_1024_fp8", m)
    parity.check(m, w.dtype)


def test_workload_flux_2048_cfg(cuda_lib):
    _workload_case("flux_2048_cfg")


def test_workload_wan_720p_81f(cuda_lib):
    _workload_case("wan_720p_81f")
