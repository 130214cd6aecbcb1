"""The fused Ulysses path across processes: two ranks as two processes on one
GPU, their shards shared through CUDA IPC, coordinated by a gloo process group
(host barriers only: no kernel waits on another process's kernel).  The ranks'
O and LSE shards, put together, must equal dit_attn_fwd on the whole sequence
bit for bit, and meet the fp64 oracle within the bf16 / FP8 bounds."""
import datetime
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import parity
from attention_dit_attn_b200 import workloads as wl

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CASES = [(1, 4, 2 * 192, 128, "bf16"), (2, 2, 2 * 320, 64, "e4m3")]


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, case, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from attention_dit_attn_b200.ulysses import ulysses_attention_fused
        B, H, L, D, dtype = case
        inp = wl.generate(B, H, L, D, dtype, seed=L + D)
        Ls = L // world
        part = lambda t: t[:, :, rank * Ls:(rank + 1) * Ls].contiguous().cuda()
        kw = {}
        if inp.q_scale is not None:
            kw = dict(q_scale=inp.q_scale.cuda().contiguous(), k_scale=inp.k_scale.cuda().contiguous(),
                      v_scale=inp.v_scale.cuda().contiguous())
        o, lse = ulysses_attention_fused(part(inp.q), part(inp.k), part(inp.v), scale=1 / math.sqrt(D), **kw)
        out.put((rank, o.cpu().view(torch.int16).numpy(), lse.cpu().numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", CASES)
def test_two_processes_share_shards_through_ipc(cuda_lib, case):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        rank, o, lse = q.get(timeout=90)
        got[rank] = (o, lse)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    o = torch.from_numpy(np.concatenate([got[r][0] for r in range(world)], axis=2)).view(torch.bfloat16)
    lse = torch.from_numpy(np.concatenate([got[r][1] for r in range(world)], axis=2))
    B, H, L, D, dtype = case
    inp = wl.generate(B, H, L, D, dtype, seed=L + D)
    o_ref, lse_ref = parity.run_gpu(inp, 1 / math.sqrt(D))
    assert torch.equal(o.view(torch.int16), o_ref.view(torch.int16))
    assert torch.equal(lse, lse_ref)
    o_or, lse_or = parity.run_oracle(inp, 1 / math.sqrt(D))
    parity.check(parity.compare(o, lse, o_or, lse_or), dtype)
