"""GPU steps of Ulysses sequence parallelism, each bit for bit against the reference
op the multi-rank CPU tests use (so the N-rank GPU path is the checked exchange
logic composed of checked steps), and a one-rank NCCL run of ulysses_attention
against dit_attn_fwd."""
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, os.path.join(ROOT, "tests"))
import parity  # noqa: E402
from oracle import e4m3_payload  # noqa: E402
from ulysses_ref import RefOps  # noqa: E402
from attention_dit_attn_b200 import workloads as wl  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape,R,C,dtype", [((2, 4, 96, 128), 2, 4, torch.bfloat16),
                                             ((4, 2, 2, 300, 64), 4, 4, torch.bfloat16),
                                             ((3, 8, 50), 3, 8, torch.float32),        # 200-byte blocks: 4-byte path
                                             ((2, 6, 33, 64), 2, 6, torch.float8_e4m3fn)])
def test_block_transpose(cuda_lib, shape, R, C, dtype):
    import attention_dit_attn_b200 as dit
    g = torch.Generator().manual_seed(1)
    x = torch.randn(shape, generator=g).to(dtype)
    got = dit.dit_attn_block_transpose(x.cuda(), R, C).cpu()
    ref = RefOps().block_transpose(x, R, C)
    assert torch.equal(got.view(torch.uint8), ref.view(torch.uint8))


def test_absmax_rows(cuda_lib):
    import attention_dit_attn_b200 as dit
    g = torch.Generator().manual_seed(2)
    x = (torch.randn((2, 6, 100, 64), generator=g) * torch.exp2(torch.randint(-5, 5, (2, 6, 1, 1), generator=g)))
    x = x.to(torch.bfloat16)
    x[0, 0] = 0
    got = dit.dit_attn_absmax_rows(x.cuda(), 12).cpu()
    assert torch.equal(got, RefOps().absmax_rows(x, 12))


def test_quantize_e4m3_rows_matches_the_recipe(cuda_lib):
    import attention_dit_attn_b200 as dit
    g = torch.Generator().manual_seed(3)
    x = (torch.randn((2, 6, 96, 64), generator=g) * 3.0).to(torch.bfloat16)
    x[0, 1] = 0                                          # a zero row: scale 1
    ops = RefOps()
    amax = ops.absmax_rows(x, 12)
    amax[5] *= 0.5                                       # half the true max: values saturate at 448
    q, s = dit.dit_attn_quantize_e4m3_rows(x.cuda(), amax.cuda())
    rq, rs = ops.quantize_e4m3_rows(x, amax)
    assert torch.equal(s.cpu(), rs)
    assert torch.equal(q.cpu().view(torch.uint8), rq.view(torch.uint8))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture
def nccl_single(cuda_lib):
    import torch.distributed as dist
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1)
    yield
    dist.destroy_process_group()


def test_one_rank_ulysses_equals_direct_attention(nccl_single):
    import attention_dit_attn_b200 as dit
    from attention_dit_attn_b200.ulysses import ulysses_attention
    g = torch.Generator().manual_seed(4)
    B, H, L, D = 1, 4, 1000, 128
    q, k, v = (torch.randn((B, H, L, D), generator=g).to(torch.bfloat16).cuda() for _ in range(3))
    o, lse = ulysses_attention(q, k, v)
    o_ref, lse_ref = dit.dit_attn_fwd(q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
    # FP8 payload: the received tensors are the FP8 attention's inputs with the global scales
    o8, lse8 = ulysses_attention(q, k, v, fp8_comm=True)
    qq, ss = [], []
    for t in (q, k, v):
        a = dit.dit_attn_absmax_rows(t, B * H)
        qt, st = dit.dit_attn_quantize_e4m3_rows(t, a)
        qq.append(qt)
        ss.append(st)
    o8_ref, lse8_ref = dit.dit_attn_fwd(*qq, q_scale=ss[0], k_scale=ss[1], v_scale=ss[2], scale=1 / math.sqrt(D))
    torch.cuda.synchronize()
    assert torch.equal(o8, o8_ref) and torch.equal(lse8, lse8_ref)
    assert dit.dit_attn_check_device_error()[0] == 0


def test_one_rank_ulysses_matches_the_oracle(nccl_single):
    """ulysses_attention against the fp64 oracle, independently of dit_attn_fwd:
    bf16 at the bf16 bounds; with the FP8 payload, against the oracle attending
    over the payload oracle's own quantisation of the same bf16 inputs (per-head
    absmax, s = amax / 448, nearest-even e4m3), at the FP8 bound."""
    from attention_dit_attn_b200.ulysses import ulysses_attention
    B, H, L, D = 1, 4, 777, 64
    inp = wl.generate(B, H, L, D, "bf16", seed=44, text_rows=60, text_scale=2.0)
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    scale = 1 / math.sqrt(D)
    o, lse = ulysses_attention(q, k, v, scale=scale)
    o8, lse8 = ulysses_attention(q, k, v, scale=scale, fp8_comm=True)
    torch.cuda.synchronize()
    o_ref, lse_ref = parity.run_oracle(inp, scale)
    parity.check(parity.compare(o.cpu(), lse.cpu(), o_ref, lse_ref), "bf16")
    codes, scales = [], []
    for t in (inp.q, inp.k, inp.v):
        x = t.to(torch.float64).numpy()
        c, s = e4m3_payload.quantize_rows(x, e4m3_payload.absmax_rows(x, B * H))
        codes.append(torch.from_numpy(np.ascontiguousarray(c)).view(torch.float8_e4m3fn))
        scales.append(torch.from_numpy(s.reshape(B, H).copy()))
    inp8 = wl.Inputs(*codes, *scales)
    o8_ref, lse8_ref = parity.run_oracle(inp8, scale)
    parity.check(parity.compare(o8.cpu(), lse8.cpu(), o8_ref, lse8_ref), "e4m3")
