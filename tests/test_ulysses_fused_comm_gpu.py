"""The per-layer fused Ulysses call (FusedUlysses) across processes: two ranks as
two processes on one GPU, set up once and then called for several successive
layers with new inputs each time (no handle exchange per call; the persistent
peer mappings are reused).  Each layer's O and LSE shards, put together, must
equal dit_attn_fwd on the whole sequence bit for bit; the first layer is also
held against the fp64 oracle.  No kernel waits on another process's kernel:
the ranks are ordered by host barriers and interprocess events only."""
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
LAYERS = 3


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer_inputs(case, layer):
    B, H, L, D, dtype = case
    return wl.generate(B, H, L, D, dtype, seed=1000 * layer + L + D, text_rows=40, text_scale=2.0)


def _rank_main(rank, world, port, case, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from attention_dit_attn_b200.ulysses import FusedUlysses
        B, H, L, D, dtype = case
        Ls = L // world
        comm = FusedUlysses(B=B, H=H, Ls=Ls, D=D, dtype=torch.bfloat16 if dtype == "bf16" else torch.float8_e4m3fn)
        peer_ptrs = [[t.data_ptr() for t in bufs] for bufs in comm._bufs]
        res = []
        for layer in range(LAYERS):
            inp = _layer_inputs(case, layer)
            part = lambda t: t[:, :, rank * Ls:(rank + 1) * Ls].contiguous().cuda()
            kw = {}
            if inp.q_scale is not None:
                kw = dict(q_scale=inp.q_scale.cuda(), k_scale=inp.k_scale.cuda(), v_scale=inp.v_scale.cuda())
            o, lse = comm(part(inp.q), part(inp.k), part(inp.v), scale=1 / math.sqrt(D), **kw)
            res.append((o.cpu().view(torch.int16).numpy(), lse.cpu().numpy()))
        comm.check()
        same = peer_ptrs == [[t.data_ptr() for t in bufs] for bufs in comm._bufs]
        comm.close()
        out.put((rank, res, same))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", [(1, 4, 2 * 192, 128, "bf16"), (2, 2, 2 * 320, 64, "e4m3")])
def test_successive_layers_reuse_the_mappings(cuda_lib, case):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        rank, res, same = q.get(timeout=120)
        got[rank] = res
        assert same, "the peer mappings changed between layers"
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    B, H, L, D, dtype = case
    for layer in range(LAYERS):
        o = torch.from_numpy(np.concatenate([got[r][layer][0] for r in range(world)], axis=2)).view(torch.bfloat16)
        lse = torch.from_numpy(np.concatenate([got[r][layer][1] for r in range(world)], axis=2))
        inp = _layer_inputs(case, layer)
        o_ref, lse_ref = parity.run_gpu(inp, 1 / math.sqrt(D))
        assert torch.equal(o.view(torch.int16), o_ref.view(torch.int16)), f"layer {layer}"
        assert torch.equal(lse, lse_ref), f"layer {layer}"
        if layer == 0:
            o_or, lse_or = parity.run_oracle(inp, 1 / math.sqrt(D))
            parity.check(parity.compare(o, lse, o_or, lse_or), dtype)
