"""The shared-memory host barrier of the per-layer fused Ulysses call, on gloo
ranks (CPU): every rank learns every rank's status at each epoch, a fast rank's
next epoch never overwrites a status a slow rank has not read, and a rank that
never arrives makes the others raise instead of hanging (failure made on the
host: a rank that leaves)."""
import datetime
import os
import socket
import sys
import time

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, scenario, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from attention_dit_attn_b200.ulysses import HostBarrier
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bar = HostBarrier(timeout_s=3.0)
        res = []
        if scenario == "status":
            for epoch in range(1, 41):
                if rank == epoch % world:
                    time.sleep(0.002)                   # a slow rank each epoch
                # rank r is unhealthy at the epochs divisible by (r + 2)
                res.append(bar.wait(ok=epoch % (rank + 2) != 0))
            out.put((rank, res))
        elif scenario == "leave":
            bar.wait()
            if rank == world - 1:
                out.put((rank, "left"))             # leaves between steps: never arrives again
            else:
                try:
                    bar.wait()
                    out.put((rank, "passed"))
                except TimeoutError as e:
                    out.put((rank, f"timeout: {e}"))
        bar.close()
    finally:
        dist.destroy_process_group()


def _run(world, scenario):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, scenario, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return got


@pytest.mark.parametrize("world", [2, 3])
def test_every_rank_sees_every_status(world):
    got = _run(world, "status")
    want = [[epoch % (r + 2) != 0 for r in range(world)] for epoch in range(1, 41)]
    for r in range(world):
        assert got[r] == want


def test_a_rank_that_leaves_makes_the_others_time_out():
    got = _run(3, "leave")
    assert got[2] == "left"
    for r in (0, 1):
        assert got[r].startswith("timeout") and "[2]" in got[r], got[r]
