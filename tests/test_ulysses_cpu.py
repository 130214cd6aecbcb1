"""Ulysses exchange logic on gloo ranks (CPU): N = 2 and 4 ranks, each holding a
sequence shard, must reproduce attention over the whole sequence bit for bit
(the per-GPU steps replaced by reference ops; attention from the fp64 oracle),
with and without the FP8 payload."""
import math
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(B, H, L, D, seed):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn((B, H, L, D), generator=g).to(torch.bfloat16) for _ in range(3)]


def _rank_main(rank, world, port, B, H, L, D, fp8, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch.distributed as dist
    from attention_dit_attn_b200.ulysses import ulysses_attention
    from ulysses_ref import RefOps
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v = _inputs(B, H, L, D, 5)
        Ls = L // world
        shard = lambda t: t[:, :, rank * Ls:(rank + 1) * Ls].contiguous()
        o, lse = ulysses_attention(shard(q), shard(k), shard(v), fp8_comm=fp8, ops=RefOps())
        out.put((rank, o.view(torch.int16).clone(), lse.clone()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,fp8", [(2, False), (4, False), (2, True), (4, True)])
def test_sharded_ulysses_equals_full_attention(world, fp8):
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from ulysses_ref import RefOps
    B, H, L, D = 1, 4, 48 * world, 64
    ctx = mp.get_context("spawn")
    q_ = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, B, H, L, D, fp8, q_)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted((q_.get(timeout=240) for _ in range(world)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    o = torch.cat([g[1] for g in got], dim=2).view(torch.bfloat16)
    lse = torch.cat([g[2] for g in got], dim=2)
    # single-process reference over the whole sequence, same ops
    ops = RefOps()
    q, k, v = _inputs(B, H, L, D, 5)
    scales = [None] * 3
    if fp8:
        qq = []
        scales = []
        for t in (q, k, v):
            a = ops.absmax_rows(t, B * H)
            qt, st = ops.quantize_e4m3_rows(t, a)
            qq.append(qt)
            scales.append(st.view(B, H).contiguous())
        q, k, v = qq
    o_ref, lse_ref = ops.attention(q, k, v, 1 / math.sqrt(D), *scales)
    assert torch.equal(o.view(torch.int16), o_ref.view(torch.int16))
    assert torch.equal(lse, lse_ref)


def _fused_bad_shape_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist
    from attention_dit_attn_b200.ulysses import ulysses_attention_fused
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    try:
        x = torch.zeros((1, 3, 64, 64), dtype=torch.bfloat16)          # 3 heads over 2 ranks
        try:
            ulysses_attention_fused(x, x, x)
            out.put((rank, "returned"))
        except ValueError:
            out.put((rank, "ValueError"))
        dist.barrier()                                                  # both ranks are still in step
    finally:
        dist.destroy_process_group()


def test_fused_path_rejects_bad_shapes_on_every_rank_before_any_collective():
    world = 2
    ctx = mp.get_context("spawn")
    q_ = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_fused_bad_shape_main, args=(r, world, port, q_)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted(q_.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == [(0, "ValueError"), (1, "ValueError")]
