"""GPU parity of the fused Ulysses attention (dit_attn_fwd_ulysses).

The N ranks are emulated on one GPU: N shard tensors per input, and one call
per rank, in sequence (a call waits on nothing but its own stream, so no call
waits for another).  The shards' O and LSE, put back together, must equal
dit_attn_fwd on the whole sequence bit for bit (same tiles, same arithmetic),
and one case is also held against the fp64 oracle.  Shard sizes that are not
multiples of 128 make K/V/Q tiles straddle two shards."""
import math

import pytest
import torch

import parity
from attention_dit_attn_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _shards(x, n):
    Ls = x.shape[2] // n
    return [x[:, :, c * Ls:(c + 1) * Ls].contiguous() for c in range(n)]


def _run_fused(inp, n, scale, ranks=None):
    import attention_dit_attn_b200 as dit
    dev = torch.device("cuda")
    B, H, L, D = inp.q.shape
    q, k, v = (_shards(t.to(dev), n) for t in (inp.q, inp.k, inp.v))
    o = [torch.full((B, H, L // n, D), float("nan"), dtype=torch.bfloat16, device=dev) for _ in range(n)]
    lse = [torch.full((B, H, L // n), float("nan"), dtype=torch.float32, device=dev) for _ in range(n)]
    kw = {}
    if inp.q_scale is not None:
        kw = dict(q_scale=inp.q_scale.to(dev).contiguous(), k_scale=inp.k_scale.to(dev).contiguous(),
                  v_scale=inp.v_scale.to(dev).contiguous())
    for r in (range(n) if ranks is None else ranks):
        dit.dit_attn_fwd_ulysses(q, k, v, o, lse, rank=r, scale=scale, **kw)
    torch.cuda.synchronize()
    rc, word = dit.dit_attn_ulysses_check_device_error()
    assert rc == 0, f"device error word {word:#x}"
    return torch.cat([t.cpu() for t in o], dim=2), torch.cat([t.cpu() for t in lse], dim=2)


@pytest.mark.parametrize("n,B,H,Ls,D,dtype", [
    (1, 1, 2, 320, 128, "bf16"),
    (2, 1, 4, 256, 128, "bf16"),
    (4, 2, 8, 192, 64, "bf16"),        # 192-row shards: tiles straddle shards
    (3, 1, 6, 320, 128, "e4m3"),       # last key tile 64 keys, last query tile partly past L
    (8, 1, 8, 64, 128, "bf16"),        # eight 64-row shards
    (2, 2, 2, 448, 64, "e4m3"),
])
def test_fused_equals_attention_on_the_whole_sequence(cuda_lib, n, B, H, Ls, D, dtype):
    inp = wl.generate(B, H, n * Ls, D, dtype, seed=100 * n + Ls + D)
    scale = 1.0 / math.sqrt(D)
    o, lse = _run_fused(inp, n, scale)
    o_ref, lse_ref = parity.run_gpu(inp, scale)
    assert torch.equal(o.view(torch.int16), o_ref.view(torch.int16))
    assert torch.equal(lse, lse_ref)


def test_fused_matches_the_oracle(cuda_lib):
    inp = wl.generate(1, 4, 4 * 192, 128, "bf16", seed=7, text_rows=100, text_scale=2.0)
    scale = 1.0 / math.sqrt(128)
    o, lse = _run_fused(inp, 4, scale)
    o_ref, lse_ref = parity.run_oracle(inp, scale)
    parity.check(parity.compare(o, lse, o_ref, lse_ref), "bf16")


@pytest.mark.parametrize("n,B,H,Ls,D", [
    (3, 1, 6, 320, 64),     # 320-row shards split 128-row tiles; last query tile partly past L
    (3, 1, 3, 320, 128),
    (2, 2, 4, 192, 64),
])
def test_fused_fp8_matches_the_oracle(cuda_lib, n, B, H, Ls, D):
    """The FP8 fused path against the fp64 oracle on the dequantised inputs, at the
    FP8 bound (relative Frobenius 3e-2, LSE 5e-3)."""
    inp = wl.generate(B, H, n * Ls, D, "e4m3", seed=31 * n + Ls + D, text_rows=77, text_scale=2.0)
    scale = 1.0 / math.sqrt(D)
    o, lse = _run_fused(inp, n, scale)
    o_ref, lse_ref = parity.run_oracle(inp, scale)
    m = parity.compare(o, lse, o_ref, lse_ref)
    parity.check(m, "e4m3")


def test_one_rank_writes_only_its_head_group(cuda_lib):
    inp = wl.generate(1, 8, 4 * 128, 64, "bf16", seed=9)
    o, lse = _run_fused(inp, 4, 0.125, ranks=[1])          # heads 2 and 3
    written = torch.zeros(8, dtype=torch.bool)
    written[2:4] = True
    assert not torch.isnan(o[0, written].float()).any() and not torch.isnan(lse[0, written]).any()
    assert torch.isnan(o[0, ~written].float()).all() and torch.isnan(lse[0, ~written]).all()
