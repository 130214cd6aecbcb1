"""Host logic of the bench across ranks (gloo, world_size 2, CPU only) and the
reference arm's JSON contract."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist(world, backend="gloo")
    try:
        d.barrier()
        # rank r "took" 1.0 + r seconds: the job time is the slowest rank's.
        t = d.max(1.0 + rank)
        v = bench.aggregate(per_rank_flops=2e12, steps=10, world=d.world, max_seconds=t)
        out.put((rank, t, v))
    finally:
        d.close()


def test_max_over_ranks_and_whole_job_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, t, v in got:
        assert t == 2.0                      # max over ranks
        assert v == pytest.approx(2e12 * 10 * 2 / 2.0 / 1e12)   # all ranks' work / slowest time


def test_reference_arm_prints_one_json_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny_256",
                        "--steps", "3", "--warmup", "3"], cwd=ROOT, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["config"]["workload"] == "tiny_256"


def test_reference_arm_on_other_ranks_exits_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny_256",
                        "--steps", "3", "--warmup", "3"], cwd=ROOT, capture_output=True, text=True,
                       env=env, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_bench_rejects_too_few_warmup_steps():
    r = subprocess.run([sys.executable, "bench.py", "--warmup", "2"], cwd=ROOT, capture_output=True,
                       text=True, timeout=120)
    assert r.returncode != 0


@pytest.mark.parametrize("op,unit", [("lse_merge", "GB/s"), ("residual_diff", "GB/s"), ("mxfp4_quant", "GB/s"),
                                     ("ulysses_fp8_payload", "GB/s")])
def test_reference_arm_of_each_op_prints_one_json_line(op, unit):
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--op", op, "--workload", "tiny_256",
                        "--steps", "3", "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == unit and d["value"] > 0
    assert d["config"]["op"] == op and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0


def test_payload_byte_count_and_ulysses_degree():
    import bench
    assert [bench.ulysses_degree(h) for h in (24, 38, 40, 2, 3)] == [8, 2, 8, 2, 1]
    # absmax 2n + quantiser 3n + head grouping 2n, plus 12 bytes per row of maxima and scales.
    assert bench.payload_bytes(1000, 4) == 7000 + 48
