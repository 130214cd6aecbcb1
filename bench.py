#!/usr/bin/env python
"""Bench of the DiT joint-attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one dit_attn_fwd call over one batch of synthetic inputs (the whole
hot path is one kernel launch).  Prints ONE JSON line on rank 0.

* value: attention TFLOP/s (4*B*H*L^2*D per call) over all ranks, inputs
  resident in HBM, timed with CUDA events between barriers; max over ranks.
* e2e: the same metric through the public API with the step's q/k/v copied
  from pinned host memory and o/lse copied back, inside the timed region.
* roofline: the attention kernel against the measured bf16 (or derived fp8)
  tensor peak.
* per_workload (N=1): the other configurations (flux_1024x768, sd35_1024_fp8,
  wan_720p_81f), each device-timed for about a second with its own clock
  record, TFLOP/s, % of nominal peak and roofline fraction.
* cpu_baseline: the fp64 oracle on this host's cores over a bounded sample of
  the workload's query rows, plus a one-thread run, the host's CPU model and
  the extrapolated time of a full call (rank 0, N=1 only).
* --impl reference: the oracle alone, as the reference arm, on the same
  workload and metric.
* --op lse_merge: instead of the forward, the LSE merge of --parts partial
  attentions (ring attention's combine step) over the workload's rows; the
  parts are real partial results (each query chunk against each key chunk,
  computed once before timing).  Metric: GB/s of algorithmic HBM traffic,
  roofline against the measured copy bandwidth.
* --op residual_diff: the step-cache reuse decision (relative L1 change of a
  hidden-state-sized bf16 residual, B*L*H*D elements of the workload, against
  the previous step's); GB/s of algorithmic HBM traffic.
* --op mxfp4_quant: the MXFP4 1x32 activation quantiser on a (B*L) x (H*D)
  bf16 activation of the workload; GB/s of algorithmic HBM traffic.
* --op gemm_fp8: the FP8 linear layer Y = A W^T of the workload's projection
  (M = B*L tokens, N = K = H*D features), e4m3 in, bf16 out; TFLOP/s,
  roofline against the fp8 dense peak (2 x the measured bf16 peak).
* --op gemm_mxfp4: the same projection in MXFP4 (E2M1 codes, one E8M0 scale per
  32 K elements), roofline against the fp4 dense peak (4 x the measured bf16
  peak).
* --op ulysses_fp8_payload: the per-GPU preparation of Ulysses' FP8 all-to-all
  payload for one [B, H, L, D] bf16 tensor of the workload: per-head absmax,
  e4m3 quantisation, heads grouped by destination rank; GB/s of algorithmic
  HBM traffic (roofline: the quantiser, the step's largest kernel).
Multi-GPU (torchrun): every rank runs its own replica (no data exchange:
heads and batches are independent), scaling "weak".
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention TFLOP/s and % of B200 tensor-core peak at 1 GPU"
MERGE_METRIC = "LSE merge of partial attentions: GB/s of algorithmic HBM traffic at 1 GPU"
DIFF_METRIC = "step-cache residual-change decision: GB/s of algorithmic HBM traffic at 1 GPU"
MXFP4_METRIC = "MXFP4 1x32 activation quantiser: GB/s of algorithmic HBM traffic at 1 GPU"
GEMM_FP8_METRIC = "FP8 linear layer Y = A W^T (e4m3 in, bf16 out): TFLOP/s at 1 GPU"
GEMM_MXFP4_METRIC = "MXFP4 linear layer Y = A W^T (block-scaled E2M1 in, bf16 out): TFLOP/s at 1 GPU"
PAYLOAD_METRIC = ("Ulysses FP8 payload preparation (absmax, e4m3 quantise, head grouping): "
                  "GB/s of algorithmic HBM traffic at 1 GPU")
DEFAULT_WORKLOAD = "flux_2048_cfg"      # the first workload with L >= 16k (the stated target)
NOMINAL_TFLOPS = {"bf16": 2250.0, "e4m3": 4500.0, "e2m1": 9000.0}
# Dense tensor rate of each input type relative to bf16 (nominal B200 figures: 2.25 / 4.5 / 9 PFLOP/s).
RATE_VS_BF16 = {"bf16": 1.0, "e4m3": 2.0, "e2m1": 4.0}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
L2_BYTES = 126 * 1024 * 1024


# ------------------------------------------------------------------ small helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# Source files of each kernel: a committed ncu summary is used only while these match.
KERNEL_SOURCES = {
    "attn_fwd": ["attn_common.cuh", "attn_fwd_sm100.cuh", "dit_attn.cu", "exp2_poly_fit.py", "sm100_ptx.cuh"],
    "lse_merge": ["lse_merge.cu"],
    "residual_diff": ["residual_diff.cu"],
    "mxfp4_quant": ["mxfp4_quant.cu"],
    "ulysses_ops": ["ulysses_ops.cu"],
    "lowp_gemm_fp8": ["gemm_sm100.cuh", "lowp_gemm.cu", "sm100_ptx.cuh"],
    "lowp_gemm_mxfp4": ["gemm_sm100.cuh", "lowp_gemm.cu", "sm100_ptx.cuh"],
}


# Spin-kernel cycles queued ahead of each per-launch start event (about 100 us at
# 2 GHz, several times the host cost of one wrapper call).
GATE_CYCLES = 200_000


def host_gate(stream):
    """Keep ``stream`` busy while the host prepares the next timed launch: a short
    spin kernel queued before the launch's start event, so the wrapper's host-side
    work (argument checks, marshalling, the C entry's pointer checks) falls
    outside the launch's CUDA-event interval instead of showing up as idle GPU
    time inside it."""
    import torch
    with torch.cuda.stream(stream):
        torch.cuda._sleep(GATE_CYCLES)


def kernel_source_hash(kind: str = "attn_fwd") -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "attention_dit_attn_b200", "csrc")
    for name in sorted(KERNEL_SOURCES[kind]):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, kind: str = "attn_fwd"):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source (its source hash matches); else None."""
    path = os.path.join(ROOT, "profiles", f"{kind}_{workload}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    m_hash = re.search(r"kernel_source_hash:\s*([0-9a-f]+)", text)
    m_bytes = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not m_hash or not m_bytes or m_hash.group(1) != kernel_source_hash(kind):
        return None
    return float(m_bytes.group(1))


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self):
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self, gpu_index: int | None):
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                idx = int(parts[0])
                if gpu_index is not None and idx != gpu_index:
                    continue
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


def physical_gpu_index(local_rank: int):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local_rank < len(ids) and ids[local_rank].isdigit():
            return int(ids[local_rank])
        return None
    return local_rank


# ------------------------------------------------------------------ distributed plumbing

class Dist:
    def __init__(self, n_gpus: int, backend: str | None = None):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            dist.init_process_group(backend=backend or "nccl",
                                    timeout=datetime.timedelta(seconds=120))
            self.pg = dist
        if n_gpus != self.world and self.world > 1:
            print(f"warning: --gpus {n_gpus} but WORLD_SIZE {self.world}", file=sys.stderr)

    @classmethod
    def single(cls):
        d = cls.__new__(cls)
        d.world, d.rank, d.local_rank, d.pg = 1, 0, 0, None
        return d

    def barrier(self):
        if self.pg is not None:
            self.pg.barrier()

    def max(self, x: float, device=None) -> float:
        if self.pg is None:
            return x
        import torch
        t = torch.tensor([x], dtype=torch.float64, device=device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


def aggregate(per_rank_flops: float, steps: int, world: int, max_seconds: float) -> float:
    """Whole-job TFLOP/s: the work of every rank over the slowest rank's time."""
    return per_rank_flops * steps * world / max_seconds / 1e12


# ------------------------------------------------------------------ CPU (oracle) timing

def oracle_sample_time(w, inp, n_rows: int, n_heads: int = 1, nthreads: int = 0):
    """Time the fp64 oracle on n_rows sampled query rows of each of the first n_heads
    heads of batch entry 0 (all L keys each); returns (seconds, flops)."""
    import oracle
    from attention_dit_attn_b200 import workloads as wl
    n_heads = max(1, min(n_heads, w.H))
    q = wl.as_bits(inp.q[:1, :n_heads])
    k = wl.as_bits(inp.k[:1, :n_heads])
    v = wl.as_bits(inp.v[:1, :n_heads])
    rows = wl.sample_rows(1, n_heads, w.L, min(n_rows, w.L), w.seed)
    kw = {}
    dtype = oracle.BF16
    if inp.q_scale is not None:
        dtype = oracle.E4M3
        kw = dict(q_scale=inp.q_scale[:1, :n_heads].numpy(), k_scale=inp.k_scale[:1, :n_heads].numpy(),
                  v_scale=inp.v_scale[:1, :n_heads].numpy())
    t0 = time.perf_counter()
    oracle.attention(q, k, v, w.scale, dtype=dtype, rows=rows, nthreads=nthreads, **kw)
    dt = time.perf_counter() - t0
    return dt, 4.0 * w.L * w.D * rows.size


def plan_sample(w, inp, seconds: float):
    """(rows per head, heads) so that the oracle runs for about `seconds`."""
    probe = min(w.L, 256)
    dt, _ = oracle_sample_time(w, inp, probe)
    per_row = max(dt / probe, 1e-7)
    total = max(16, int(seconds / per_row))
    if total <= w.L:
        return total, 1
    heads = min(w.H, -(-total // w.L))
    return w.L, heads


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_baseline(w, inp, seconds: float = 15.0):
    """The oracle on all host threads (about `seconds`), then on one thread (about a
    fifth of that), each on sampled query rows; the full call's time on this host is
    extrapolated from the all-threads rate (4*L*D FLOPs per row, B*H*L rows)."""
    import oracle
    threads = oracle.max_threads()          # read before the one-thread run changes it
    rows, heads = plan_sample(w, inp, seconds)
    dt, flops = oracle_sample_time(w, inp, rows, heads, nthreads=threads)
    rate = flops / dt
    rows1 = max(16, min(w.L, int(rows * heads * 0.2 / threads) or 16))
    dt1, flops1 = oracle_sample_time(w, inp, rows1, 1, nthreads=1)
    return {"value": rate / 1e12, "unit": "TFLOP/s", "cores": threads,
            "kind": "oracle",
            "sample": f"fp64 oracle on {rows} sampled query rows x {heads} head(s) of batch 0 of "
                      f"{w.name} (all {w.L} keys per row): {dt:.1f} s on {threads} threads",
            "single_thread": {"value": flops1 / dt1 / 1e12, "unit": "TFLOP/s",
                              "sample": f"{rows1} sampled query rows of head 0: {dt1:.2f} s on 1 thread"},
            "host_cpus": os.cpu_count(), "cpu_model": cpu_model(),
            "full_call_seconds_extrapolated": w.flops / rate,
            "full_call_note": f"all {w.B * w.H * w.L} query rows of one call at the sampled all-threads rate"}


# ------------------------------------------------------------------ arms

def run_reference(args, dist: Dist):
    """Reference arm: the fp64 CPU oracle as it stands (no GPU)."""
    if dist.rank != 0:
        return
    import oracle
    from attention_dit_attn_b200 import workloads as wl
    w = wl.ALL[args.workload]
    inp = wl.generate_workload(w)
    total_budget = 120.0
    rows, heads = plan_sample(w, inp, total_budget / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample_time(w, inp, rows, heads)
    t_total, f_total = 0.0, 0.0
    for _ in range(args.steps):
        dt, fl = oracle_sample_time(w, inp, rows, heads)
        t_total += dt
        f_total += fl
    value = f_total / t_total / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.max_threads(),
                         "kind": "oracle",
                         "sample": f"each step: fp64 oracle on {rows} sampled query rows x {heads} "
                                   f"head(s) of batch 0 of {w.name} (all {w.L} keys per row)"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def workload_config(w):
    in_bytes = 3 * w.B * w.H * w.L * w.D * (1 if w.dtype == "e4m3" else 2)
    return {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "D": w.D, "text_tokens": w.text_rows,
            "input_dtype": w.dtype, "output_dtype": "bf16", "causal": False,
            "inputs_bytes": in_bytes,
            "l2": ("inputs larger than L2 (%.0f MB > 126 MB)" % (in_bytes / 1e6)) if in_bytes > L2_BYTES
            else "L2 flushed between timed steps (256 MB write)",
            "parallelism": "replicas"}


# ------------------------------------------------------------------ LSE merge (ring-attention combine)

def merge_bytes(rows: int, D: int, n: int) -> int:
    """Algorithmic bytes of one merge: n parts of bf16 o + fp32 lse read, one written."""
    return rows * (n * (2 * D + 4) + 2 * D + 4)


def make_merge_parts(w, inp, dev, n: int):
    """Ring degree n over the workload's sequence: part c holds, for every query
    chunk r, dit_attn_fwd(Q_r, K_c, V_c); rows ordered (r, b, h, l)."""
    import torch
    import attention_dit_attn_b200 as dit
    if w.L % n:
        raise ValueError(f"L={w.L} does not split into {n} equal chunks")
    Lc = w.L // n
    q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
    kw = {}
    if inp.q_scale is not None:
        kw = dict(q_scale=inp.q_scale.to(dev).contiguous(), k_scale=inp.k_scale.to(dev).contiguous(),
                  v_scale=inp.v_scale.to(dev).contiguous())
    chunk = lambda t, i: t[:, :, i * Lc:(i + 1) * Lc].contiguous()
    parts = []
    for c in range(n):
        outs = [dit.dit_attn_fwd(chunk(q, r), chunk(k, c), chunk(v, c), scale=w.scale, **kw) for r in range(n)]
        parts.append((torch.stack([o for o, _ in outs]).reshape(-1, w.D).contiguous(),
                      torch.stack([l for _, l in outs]).reshape(-1).contiguous()))
    torch.cuda.synchronize(dev)
    return parts


def merge_oracle_rate(parts_cpu, seconds: float):
    """The fp64 merge oracle on a bounded sample of rows: (GB/s algorithmic, rows, s)."""
    from oracle.lse_merge import lse_merge
    rows_total, D = parts_cpu[0][0].shape
    n = len(parts_cpu)
    rows = min(rows_total, 4096)
    while True:
        t0 = time.perf_counter()
        lse_merge([o[:rows].double().numpy() for o, _ in parts_cpu], [l[:rows].double().numpy() for _, l in parts_cpu])
        dt = time.perf_counter() - t0
        if dt >= seconds / 4 or rows >= rows_total:
            break
        rows = min(rows_total, rows * 4)
    return merge_bytes(rows, D, n) / dt / 1e9, rows, dt


def merge_config(w, n, rows):
    return {"workload": w.name, "op": "lse_merge", "parts": n, "rows": rows, "D": w.D,
            "B": w.B, "H": w.H, "L": w.L, "ring_degree": n, "input_dtype": "bf16 o + fp32 lse",
            "output_dtype": "bf16 o + fp32 lse", "bytes_per_call": merge_bytes(rows, w.D, n),
            "l2": "inputs larger than L2" if merge_bytes(rows, w.D, n) > L2_BYTES
            else "L2 flushed between timed steps (256 MB write)",
            "parallelism": "replicas"}


def run_merge_reference(args, dist: Dist):
    if dist.rank != 0:
        return
    import torch
    from attention_dit_attn_b200 import workloads as wl
    w = wl.ALL[args.workload]
    n = args.parts
    rows = w.B * w.H * w.L
    g = torch.Generator().manual_seed(w.seed)
    sample = min(rows, 1 << 16)
    parts = [(torch.randn((sample, w.D), generator=g).to(torch.bfloat16), torch.randn((sample,), generator=g))
             for _ in range(n)]
    per = 60.0 / max(1, args.steps + args.warmup)
    for _ in range(args.warmup):
        merge_oracle_rate(parts, per)
    rates = [merge_oracle_rate(parts, per) for _ in range(args.steps)]
    value = statistics.median(r[0] for r in rates)
    cores = 1
    line = {
        "impl": "reference", "metric": MERGE_METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * merge_bytes(rows, w.D, n) / (value * 1e9),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": merge_config(w, n, rows),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step: fp64 numpy merge oracle on {rates[0][1]} rows of {n} parts"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def run_merge(args, dist: Dist):
    import torch
    import attention_dit_attn_b200 as dit
    from attention_dit_attn_b200 import workloads as wl

    dit.ensure_built()
    torch.cuda.set_device(dist.local_rank)
    dev = torch.device("cuda", dist.local_rank)
    w = wl.ALL[args.workload]
    n = args.parts
    parts = make_merge_parts(w, wl.generate_workload(w), dev, n)
    rows = parts[0][0].shape[0]
    nbytes = merge_bytes(rows, w.D, n)
    o = torch.empty_like(parts[0][0])
    lse = torch.empty_like(parts[0][1])
    flush = None
    if nbytes <= L2_BYTES:
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        dit.dit_attn_lse_merge(parts, o, lse, stream=stream)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler()
    if dist.rank == 0:
        sampler.start()
        time.sleep(0.3)
    dist.barrier()
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for a, b in evs:
        if flush is not None:
            flush.fill_(1)
        host_gate(stream)
        a.record(stream)
        dit.dit_attn_lse_merge(parts, o, lse, stream=stream)
        b.record(stream)
    torch.cuda.synchronize(dev)
    seconds = sum(a.elapsed_time(b) for a, b in evs) / 1e3
    dist.barrier()
    if dist.rank == 0:
        time.sleep(0.2)
        sampler.stop()
    max_seconds = dist.max(seconds, dev)
    value = nbytes * args.steps * dist.world / max_seconds / 1e9
    achieved = nbytes / (seconds / args.steps) / 1e9

    # end to end: parts from pinned host memory, merged result back to the host
    e2e_steps = max(3, min(args.steps, 10))
    hparts = [(po.cpu().pin_memory(), pl.cpu().pin_memory()) for po, pl in parts]
    dparts = [(torch.empty_like(po), torch.empty_like(pl)) for po, pl in parts]
    ho = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    hl = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()

    def e2e_step():
        for (ho_, hl_), (do_, dl_) in zip(hparts, dparts):
            do_.copy_(ho_, non_blocking=True)
            dl_.copy_(hl_, non_blocking=True)
        dit.dit_attn_lse_merge(dparts, o, lse, stream=stream)
        ho.copy_(o, non_blocking=True)
        hl.copy_(lse, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(dev)
    dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize(dev)
    e2e_s = dist.max(a.elapsed_time(b) / 1e3, dev)
    h2d = sum(po.numel() * 2 + pl.numel() * 4 for po, pl in hparts)
    d2h = ho.numel() * 2 + hl.numel() * 4

    peaks, peaks_kind = load_peaks()
    peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    traffic = profiled_traffic(w.name, kind="lse_merge")
    clocks = sampler.summary(physical_gpu_index(dist.local_rank)) if dist.rank == 0 else {}
    line = {
        "metric": MERGE_METRIC, "value": value, "unit": "GB/s", "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * max_seconds / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic", "config": merge_config(w, n, rows),
        "e2e": {"value": nbytes * e2e_steps * dist.world / e2e_s / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "result_matches_device": torch.equal(ho, o.cpu())},
        "gpu_launches": args.steps,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": f"HBM copy, {peaks_kind}", "traffic": traffic,
                     "kernel": "lse_merge_kernel", "bytes_per_launch": nbytes},
        "clocks": clocks,
    }
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        parts_cpu = [(po[: 1 << 16].cpu(), pl[: 1 << 16].cpu()) for po, pl in parts]
        rate, srows, dt = merge_oracle_rate(parts_cpu, args.cpu_seconds)
        line["cpu_baseline"] = {"value": rate, "unit": "GB/s", "cores": 1, "kind": "oracle",
                                "sample": f"fp64 numpy merge oracle on the first {srows} rows of the "
                                          f"{n} parts: {dt:.2f} s"}
    if dist.rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ step-cache decision (DBCache)

def diff_inputs(w, dev):
    """Seeded residuals of the workload's hidden-state size: prev ~ N(0,1), cur = prev
    + 0.05 N(0,1) (a step whose work is reused at the published threshold 0.12)."""
    import torch
    n = w.B * w.L * w.H * w.D
    g = torch.Generator(device=dev).manual_seed(w.seed)
    prev = torch.randn(n, generator=g, device=dev)
    cur = (prev + 0.05 * torch.randn(n, generator=g, device=dev)).to(torch.bfloat16)
    return cur, prev.to(torch.bfloat16)


def diff_config(w, n):
    return {"workload": w.name, "op": "residual_diff", "elements": n, "B": w.B, "L": w.L,
            "hidden": w.H * w.D, "input_dtype": "bf16", "threshold": 0.12, "bytes_per_call": 4 * n + 8,
            "l2": "inputs larger than L2" if 4 * n > L2_BYTES else "L2 flushed between timed steps (256 MB write)",
            "parallelism": "replicas"}


def diff_oracle_rate(cur_cpu, prev_cpu, seconds: float):
    from oracle.residual_diff import residual_diff
    n = min(cur_cpu.numel(), 1 << 20)
    while True:
        c, pv = cur_cpu[:n].double().numpy(), prev_cpu[:n].double().numpy()
        t0 = time.perf_counter()
        residual_diff(c, pv)
        dt = time.perf_counter() - t0
        if dt >= seconds / 4 or n >= cur_cpu.numel():
            return 4 * n / dt / 1e9, n, dt
        n = min(cur_cpu.numel(), n * 4)


def run_diff_reference(args, dist: Dist):
    if dist.rank != 0:
        return
    import torch
    from attention_dit_attn_b200 import workloads as wl
    w = wl.ALL[args.workload]
    n = w.B * w.L * w.H * w.D
    g = torch.Generator().manual_seed(w.seed)
    m = min(n, 1 << 24)
    prev = torch.randn(m, generator=g)
    cur = (prev + 0.05 * torch.randn(m, generator=g)).to(torch.bfloat16)
    prev = prev.to(torch.bfloat16)
    per = 60.0 / max(1, args.steps + args.warmup)
    for _ in range(args.warmup):
        diff_oracle_rate(cur, prev, per)
    rates = [diff_oracle_rate(cur, prev, per) for _ in range(args.steps)]
    value = statistics.median(r[0] for r in rates)
    line = {
        "impl": "reference", "metric": DIFF_METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * 4 * n / (value * 1e9),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": diff_config(w, n),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"each step: fp64 numpy oracle on {rates[0][1]} elements"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def run_diff(args, dist: Dist):
    import torch
    import attention_dit_attn_b200 as dit
    from attention_dit_attn_b200 import workloads as wl

    dit.ensure_built()
    torch.cuda.set_device(dist.local_rank)
    dev = torch.device("cuda", dist.local_rank)
    w = wl.ALL[args.workload]
    cur, prev = diff_inputs(w, dev)
    n = cur.numel()
    nbytes = 4 * n + 8
    ws = torch.zeros(dit.dit_attn_residual_diff_workspace_bytes(n), dtype=torch.uint8, device=dev)
    d = torch.empty(1, dtype=torch.float32, device=dev)
    r = torch.empty(1, dtype=torch.int32, device=dev)
    flush = None
    if 4 * n <= L2_BYTES:
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    call = lambda c, p: dit.dit_attn_residual_diff(c, p, 0.12, workspace=ws, diff=d, reuse=r, stream=stream)
    for _ in range(args.warmup):
        call(cur, prev)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler()
    if dist.rank == 0:
        sampler.start()
        time.sleep(0.3)
    dist.barrier()
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for a, b in evs:
        if flush is not None:
            flush.fill_(1)
        host_gate(stream)
        a.record(stream)
        call(cur, prev)
        b.record(stream)
    torch.cuda.synchronize(dev)
    seconds = sum(a.elapsed_time(b) for a, b in evs) / 1e3
    dist.barrier()
    if dist.rank == 0:
        time.sleep(0.2)
        sampler.stop()
    max_seconds = dist.max(seconds, dev)
    value = nbytes * args.steps * dist.world / max_seconds / 1e9
    achieved = nbytes / (seconds / args.steps) / 1e9

    # end to end: both residuals from pinned host memory, the decision back to the host
    e2e_steps = max(3, min(args.steps, 10))
    hc, hp = cur.cpu().pin_memory(), prev.cpu().pin_memory()
    dc, dp = torch.empty_like(cur), torch.empty_like(prev)
    hd = torch.empty(1, dtype=torch.float32).pin_memory()
    hr = torch.empty(1, dtype=torch.int32).pin_memory()

    def e2e_step():
        dc.copy_(hc, non_blocking=True)
        dp.copy_(hp, non_blocking=True)
        call(dc, dp)
        hd.copy_(d, non_blocking=True)
        hr.copy_(r, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(dev)
    dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize(dev)
    e2e_s = dist.max(a.elapsed_time(b) / 1e3, dev)

    peaks, peaks_kind = load_peaks()
    peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    traffic = profiled_traffic(w.name, kind="residual_diff")
    clocks = sampler.summary(physical_gpu_index(dist.local_rank)) if dist.rank == 0 else {}
    line = {
        "metric": DIFF_METRIC, "value": value, "unit": "GB/s", "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * max_seconds / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic", "config": diff_config(w, n),
        "e2e": {"value": nbytes * e2e_steps * dist.world / e2e_s / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": 4 * n, "d2h_bytes_per_step": 8, "steps": e2e_steps,
                "result_matches_device": bool(float(hd.item()) == float(d.item()) and int(hr.item()) == int(r.item())),
                "diff": float(hd.item()), "reuse": int(hr.item())},
        "gpu_launches": args.steps,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": f"HBM copy, {peaks_kind}", "traffic": traffic,
                     "kernel": "residual_diff_kernel", "bytes_per_launch": nbytes},
        "clocks": clocks,
    }
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        rate, sn, dt = diff_oracle_rate(cur.cpu(), prev.cpu(), args.cpu_seconds)
        line["cpu_baseline"] = {"value": rate, "unit": "GB/s", "cores": 1, "kind": "oracle",
                                "sample": f"fp64 numpy oracle on the first {sn} elements: {dt:.2f} s"}
    if dist.rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ MXFP4 activation quantiser

def mxfp4_bytes(rows: int, K: int) -> int:
    return rows * (2 * K + K // 2 + K // 32)


def mxfp4_config(w, rows, K):
    return {"workload": w.name, "op": "mxfp4_quant", "rows": rows, "K": K, "input_dtype": "bf16",
            "output": "E2M1 codes (K/2 bytes per row) + E8M0 scales (K/32 bytes per row)",
            "bytes_per_call": mxfp4_bytes(rows, K),
            "l2": "inputs larger than L2" if 2 * rows * K > L2_BYTES else "L2 flushed between timed steps (256 MB write)",
            "parallelism": "replicas"}


def mxfp4_oracle_rate(x_cpu, seconds: float):
    from oracle import mxfp4
    rows = 8
    K = x_cpu.shape[1]
    while True:
        xs = x_cpu[:rows].double().numpy()
        t0 = time.perf_counter()
        mxfp4.quantize(xs)
        dt = time.perf_counter() - t0
        if dt >= seconds / 4 or rows >= x_cpu.shape[0]:
            return mxfp4_bytes(rows, K) / dt / 1e9, rows, dt
        rows = min(x_cpu.shape[0], rows * 4)


def run_mxfp4_reference(args, dist: Dist):
    if dist.rank != 0:
        return
    import torch
    from attention_dit_attn_b200 import workloads as wl
    w = wl.ALL[args.workload]
    rows, K = w.B * w.L, w.H * w.D
    g = torch.Generator().manual_seed(w.seed)
    x = torch.randn((min(rows, 4096), K), generator=g).to(torch.bfloat16)
    per = 60.0 / max(1, args.steps + args.warmup)
    for _ in range(args.warmup):
        mxfp4_oracle_rate(x, per)
    rates = [mxfp4_oracle_rate(x, per) for _ in range(args.steps)]
    value = statistics.median(r[0] for r in rates)
    line = {
        "impl": "reference", "metric": MXFP4_METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * mxfp4_bytes(rows, K) / (value * 1e9),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": mxfp4_config(w, rows, K),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"each step: fp64 numpy oracle on {rates[0][1]} rows of {K}"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def run_mxfp4(args, dist: Dist):
    import torch
    import attention_dit_attn_b200 as dit
    from attention_dit_attn_b200 import workloads as wl

    dit.ensure_built()
    torch.cuda.set_device(dist.local_rank)
    dev = torch.device("cuda", dist.local_rank)
    w = wl.ALL[args.workload]
    rows, K = w.B * w.L, w.H * w.D
    g = torch.Generator(device=dev).manual_seed(w.seed)
    x = torch.randn((rows, K), generator=g, device=dev).to(torch.bfloat16)
    q = torch.empty((rows, K // 2), dtype=torch.uint8, device=dev)
    sc = torch.empty((rows, K // 32), dtype=torch.uint8, device=dev)
    nbytes = mxfp4_bytes(rows, K)
    flush = None
    if 2 * rows * K <= L2_BYTES:
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    call = lambda xx: dit.dit_attn_mxfp4_quantize(xx, q, sc, stream=stream)
    for _ in range(args.warmup):
        call(x)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler()
    if dist.rank == 0:
        sampler.start()
        time.sleep(0.3)
    dist.barrier()
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for a, b in evs:
        if flush is not None:
            flush.fill_(1)
        host_gate(stream)
        a.record(stream)
        call(x)
        b.record(stream)
    torch.cuda.synchronize(dev)
    seconds = sum(a.elapsed_time(b) for a, b in evs) / 1e3
    dist.barrier()
    if dist.rank == 0:
        time.sleep(0.2)
        sampler.stop()
    max_seconds = dist.max(seconds, dev)
    value = nbytes * args.steps * dist.world / max_seconds / 1e9
    achieved = nbytes / (seconds / args.steps) / 1e9

    e2e_steps = max(3, min(args.steps, 10))
    hx = x.cpu().pin_memory()
    dx = torch.empty_like(x)
    hq = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    hs = torch.empty(sc.shape, dtype=sc.dtype).pin_memory()

    def e2e_step():
        dx.copy_(hx, non_blocking=True)
        call(dx)
        hq.copy_(q, non_blocking=True)
        hs.copy_(sc, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(dev)
    dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize(dev)
    e2e_s = dist.max(a.elapsed_time(b) / 1e3, dev)

    peaks, peaks_kind = load_peaks()
    peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    traffic = profiled_traffic(w.name, kind="mxfp4_quant")
    clocks = sampler.summary(physical_gpu_index(dist.local_rank)) if dist.rank == 0 else {}
    line = {
        "metric": MXFP4_METRIC, "value": value, "unit": "GB/s", "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * max_seconds / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic", "config": mxfp4_config(w, rows, K),
        "e2e": {"value": nbytes * e2e_steps * dist.world / e2e_s / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": 2 * rows * K, "d2h_bytes_per_step": rows * (K // 2 + K // 32),
                "steps": e2e_steps, "result_matches_device": bool(torch.equal(hq, q.cpu()) and torch.equal(hs, sc.cpu()))},
        "gpu_launches": args.steps,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": f"HBM copy, {peaks_kind}", "traffic": traffic,
                     "kernel": "mxfp4_quant_kernel", "bytes_per_launch": nbytes},
        "clocks": clocks,
    }
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        rate, srows, dt = mxfp4_oracle_rate(x[:4096].cpu(), args.cpu_seconds)
        line["cpu_baseline"] = {"value": rate, "unit": "GB/s", "cores": 1, "kind": "oracle",
                                "sample": f"fp64 numpy oracle on the first {srows} rows of {K}: {dt:.2f} s"}
    if dist.rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ FP8 linear-layer GEMM (NEXT-3)

def gemm_shape(w):
    """The DiT block's projection on this workload: M = B*L tokens, N = K = H*D features."""
    return w.B * w.L, w.H * w.D, w.H * w.D


def gemm_config(w, M, N, K, kind="fp8"):
    if kind == "fp8":
        in_bytes = M * K + N * K
    else:
        in_bytes = (M + N) * (K // 2 + K // 32)
    return {"workload": w.name, "op": "gemm_" + kind, "M": M, "N": N, "K": K,
            "input_dtype": "e4m3" if kind == "fp8" else "MXFP4 (E2M1 + E8M0 per 32)",
            "output_dtype": "bf16", "flops_per_call": 2.0 * M * N * K,
            "bytes_per_call": in_bytes + 2 * M * N,
            "l2": "inputs and output larger than L2" if in_bytes + 2 * M * N > L2_BYTES
            else "L2 flushed between timed steps (256 MB write)",
            "parallelism": "replicas"}


def gemm_oracle_rate(a, sa, w_, sw, seconds: float, kind="fp8"):
    """fp64 oracle (oracle/lowp_gemm.py) on the first rows of A: (TFLOP/s, rows, s)."""
    import torch
    from oracle import lowp_gemm
    ac, wc = a.view(torch.uint8).numpy(), w_.view(torch.uint8).numpy()
    K = wc.shape[1] if kind == "fp8" else 2 * wc.shape[1]
    rows = 4
    while True:
        t0 = time.perf_counter()
        if kind == "fp8":
            lowp_gemm.gemm_e4m3(ac[:rows], sa, wc, sw)
        else:
            lowp_gemm.gemm_mxfp4(ac[:rows], sa[:rows].numpy(), wc, sw.numpy())
        dt = time.perf_counter() - t0
        if dt >= seconds / 4 or rows >= ac.shape[0]:
            return 2.0 * rows * wc.shape[0] * K / dt / 1e12, rows, dt
        rows = min(ac.shape[0], rows * 4)


def gemm_operands(w, M, N, K, kind):
    from attention_dit_attn_b200 import workloads as wl
    if kind == "fp8":
        return wl.gemm_operands_e4m3(M, N, K, seed=w.seed)
    return wl.gemm_operands_mxfp4(M, N, K, seed=w.seed)


def run_gemm_reference(args, dist: Dist):
    if dist.rank != 0:
        return
    from attention_dit_attn_b200 import workloads as wl
    kind = args.op.split("_")[1]
    w = wl.ALL[args.workload]
    M, N, K = gemm_shape(w)
    a, sa, w_, sw = gemm_operands(w, min(M, 1024), N, K, kind)
    per = 60.0 / max(1, args.steps + args.warmup)
    for _ in range(args.warmup):
        gemm_oracle_rate(a, sa, w_, sw, per, kind)
    rates = [gemm_oracle_rate(a, sa, w_, sw, per, kind) for _ in range(args.steps)]
    value = statistics.median(r[0] for r in rates)
    line = {
        "impl": "reference", "metric": GEMM_FP8_METRIC if kind == "fp8" else GEMM_MXFP4_METRIC, "value": value,
        "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * 2.0 * M * N * K / (value * 1e12),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": gemm_config(w, M, N, K, kind),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
                         "sample": f"each step: fp64 numpy oracle (BLAS) on {rates[0][1]} rows of A x [{N}, {K}]"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def run_gemm(args, dist: Dist):
    import torch
    import attention_dit_attn_b200 as dit
    from attention_dit_attn_b200 import workloads as wl

    dit.ensure_built()
    torch.cuda.set_device(dist.local_rank)
    dev = torch.device("cuda", dist.local_rank)
    kind = args.op.split("_")[1]                       # fp8 | mxfp4
    w = wl.ALL[args.workload]
    M, N, K = gemm_shape(w)
    a_cpu, sa, w_cpu, sw = gemm_operands(w, M, N, K, kind)
    a, wt = a_cpu.to(dev), w_cpu.to(dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    if kind == "fp8":
        call = lambda aa, yy: dit.dit_attn_gemm_fp8(aa, wt, sa, sw, y=yy, stream=stream)
        dtype, kern = "e4m3", "dit_gemm::gemm_kernel<Fp8Kind> (CTA pair, persistent)"
    else:
        # Scales in the tiled layout the tensor cores read: the weight's once,
        # the activation's as part of each end-to-end step.
        ta = dit.dit_attn_mxfp4_tile_scales(sa.to(dev), K)
        tw = dit.dit_attn_mxfp4_tile_scales(sw.to(dev), K)
        call = lambda aa, yy: dit.dit_attn_gemm_mxfp4(aa, ta, wt, tw, y=yy, stream=stream)
        dtype, kern = "e2m1", "dit_gemm::gemm_mxf4_kernel (one CTA per SM, persistent)"
    cfg = gemm_config(w, M, N, K, kind)
    flops = cfg["flops_per_call"]
    flush = None
    if cfg["bytes_per_call"] <= L2_BYTES:
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        call(a, y)
    torch.cuda.synchronize(dev)
    rc, word = dit.dit_attn_gemm_check_device_error(stream)
    if rc != 0:
        raise RuntimeError(f"device error during warm-up: {word:#x}")
    sampler = ClockSampler()
    if dist.rank == 0:
        sampler.start()
        time.sleep(0.3)
    dist.barrier()
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for e0, e1 in evs:
        if flush is not None:
            flush.fill_(1)
        host_gate(stream)
        e0.record(stream)
        call(a, y)
        e1.record(stream)
    torch.cuda.synchronize(dev)
    seconds = sum(e0.elapsed_time(e1) for e0, e1 in evs) / 1e3
    dist.barrier()
    if dist.rank == 0:
        time.sleep(0.2)
        sampler.stop()
    rc, word = dit.dit_attn_gemm_check_device_error(stream)
    if rc != 0:
        raise RuntimeError(f"device error during the timed region: {word:#x}")
    max_seconds = dist.max(seconds, dev)
    value = flops * args.steps * dist.world / max_seconds / 1e12
    achieved = flops / (seconds / args.steps) / 1e12

    # End to end: the activations (and MXFP4 scales) in from pinned host memory, Y back
    # out, every step.
    e2e_steps = max(3, min(args.steps, 10))
    ha = a_cpu.view(torch.uint8).pin_memory()
    da = torch.empty_like(a)
    hy = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    if kind == "mxfp4":
        hs = sa.pin_memory()
        ds = torch.empty_like(hs, device=dev)
        dta = torch.empty_like(ta)

    def e2e_step():
        da.view(torch.uint8).copy_(ha, non_blocking=True)
        if kind == "fp8":
            call(da, y)
        else:
            ds.copy_(hs, non_blocking=True)
            dit.dit_attn_mxfp4_tile_scales(ds, K, tiled=dta, stream=stream)
            dit.dit_attn_gemm_mxfp4(da, dta, wt, tw, y=y, stream=stream)
        hy.copy_(y, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(dev)
    dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_s = dist.max(e0.elapsed_time(e1) / 1e3, dev)
    h2d = ha.numel() + (hs.numel() if kind == "mxfp4" else 0)

    peaks, peaks_kind = load_peaks()
    peak = RATE_VS_BF16[dtype] * float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    clocks = sampler.summary(physical_gpu_index(dist.local_rank)) if dist.rank == 0 else {}
    line = {
        "metric": GEMM_FP8_METRIC if kind == "fp8" else GEMM_MXFP4_METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * max_seconds / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": dtype, "data": "synthetic", "config": cfg,
        "pct_of_peak": {"nominal_dense": 100.0 * value / dist.world / NOMINAL_TFLOPS[dtype],
                        "nominal_tflops": NOMINAL_TFLOPS[dtype]},
        "e2e": {"value": flops * e2e_steps * dist.world / e2e_s / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": 2 * M * N, "steps": e2e_steps,
                "result_matches_device": bool(torch.equal(hy, y.cpu()))},
        "gpu_launches": args.steps,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak,
                     "peak_source": f"{dtype} dense = {RATE_VS_BF16[dtype]:g} x bf16 {peaks_kind} (burst), "
                                    "the nominal dense-rate ratio",
                     "traffic": profiled_traffic(w.name, kind="lowp_gemm_" + kind),
                     "kernel": kern, "flops_per_launch": flops},
        "clocks": clocks,
    }
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        rate, srows, dt = gemm_oracle_rate(a_cpu[:2048], sa if kind == "fp8" else sa[:2048], w_cpu, sw,
                                           args.cpu_seconds, kind)
        line["cpu_baseline"] = {"value": rate, "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
                                "sample": f"fp64 numpy oracle (BLAS threads) on the first {srows} rows of A "
                                          f"x [{N}, {K}]: {dt:.2f} s"}
    if dist.rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ Ulysses FP8 payload

def ulysses_degree(H: int) -> int:
    """The largest of 8, 4, 2, 1 ranks that the heads split over evenly."""
    return next(n for n in (8, 4, 2, 1) if H % n == 0)


def payload_bytes(n: int, rows: int) -> int:
    """absmax reads 2n bytes and writes the row maxima; the quantiser reads 2n
    and the maxima, writes n and the scales; the head grouping reads and
    writes n."""
    return 7 * n + 12 * rows


def payload_config(w, N):
    n = w.B * w.H * w.L * w.D
    return {"workload": w.name, "op": "ulysses_fp8_payload", "shape": [w.B, w.H, w.L, w.D],
            "ranks": N, "input_dtype": "bf16", "payload": "e4m3 + fp32 per-head scales",
            "bytes_per_call": payload_bytes(n, w.B * w.H),
            "kernels": ["absmax_rows_kernel", "quantize_rows_kernel", "block_transpose_kernel"],
            "note": "one rank's tensor; the all-reduce of the head maxima and the all-to-all are "
                    "collectives across GPUs, not part of this single-GPU step",
            "l2": "inputs larger than L2" if 2 * n > L2_BYTES else "L2 flushed between timed steps (256 MB write)",
            "parallelism": "replicas"}


def payload_oracle_rate(x_cpu, rows: int, N: int, B: int, seconds: float):
    """Oracle rate over whole heads (rows) of x_cpu [rows, row_len], as many as
    fit in about seconds/4 (the head grouping over the quantised sample)."""
    from oracle import e4m3_payload as ep
    r = 1
    while True:
        xs = x_cpu[:r].double().numpy()
        t0 = time.perf_counter()
        amax = ep.absmax_rows(xs, r)
        qc, _ = ep.quantize_rows(xs, amax)
        if r % N == 0:
            ep.block_transpose(qc, r // N, N)
        dt = time.perf_counter() - t0
        if dt >= seconds / 4 or r >= rows:
            return payload_bytes(xs.size, r) / dt / 1e9, r, dt
        r = min(rows, r * 2)


def payload_input(w, dev):
    import torch
    g = torch.Generator(device=dev).manual_seed(w.seed)
    return torch.randn((w.B, w.H, w.L, w.D), generator=g, device=dev).to(torch.bfloat16)


def run_payload_reference(args, dist: Dist):
    if dist.rank != 0:
        return
    import torch
    from attention_dit_attn_b200 import workloads as wl
    w = wl.ALL[args.workload]
    N = ulysses_degree(w.H)
    rows, row_len = w.B * w.H, w.L * w.D
    g = torch.Generator().manual_seed(w.seed)
    x = torch.randn((min(rows, 8), row_len), generator=g).to(torch.bfloat16)
    per = 60.0 / max(1, args.steps + args.warmup)
    for _ in range(args.warmup):
        payload_oracle_rate(x, x.shape[0], N, w.B, per)
    rates = [payload_oracle_rate(x, x.shape[0], N, w.B, per) for _ in range(args.steps)]
    value = statistics.median(r[0] for r in rates)
    nbytes = payload_bytes(rows * row_len, rows)
    line = {
        "impl": "reference", "metric": PAYLOAD_METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * nbytes / (value * 1e9),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": payload_config(w, N),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"each step: fp64 numpy oracle on {rates[0][1]} head(s) of {row_len} values"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def run_payload(args, dist: Dist):
    import torch
    import attention_dit_attn_b200 as dit
    from attention_dit_attn_b200 import workloads as wl

    dit.ensure_built()
    torch.cuda.set_device(dist.local_rank)
    dev = torch.device("cuda", dist.local_rank)
    w = wl.ALL[args.workload]
    N = ulysses_degree(w.H)
    rows = w.B * w.H
    x = payload_input(w, dev)
    n = x.numel()
    amax = torch.empty(rows, dtype=torch.float32, device=dev)
    q8 = torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=dev)
    sc = torch.empty(rows, dtype=torch.float32, device=dev)
    out = torch.empty_like(q8)
    nbytes = payload_bytes(n, rows)
    flush = None
    if 2 * n <= L2_BYTES:
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(xx, evq=None):
        dit.dit_attn_absmax_rows(xx, rows, amax, stream=stream)
        if evq is not None:
            evq[0].record(stream)
        dit.dit_attn_quantize_e4m3_rows(xx, amax, q8, sc, stream=stream)
        if evq is not None:
            evq[1].record(stream)
        dit.dit_attn_block_transpose(q8, w.B, N, out, stream=stream)   # [B, N, H/N, ...] -> [N, B, H/N, ...]

    for _ in range(args.warmup):
        step(x)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler()
    if dist.rank == 0:
        sampler.start()
        time.sleep(0.3)
    dist.barrier()
    torch.cuda.synchronize(dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    evs = [(ev(), ev(), (ev(), ev())) for _ in range(args.steps)]
    for a, b, evq in evs:
        if flush is not None:
            flush.fill_(1)
        host_gate(stream)
        a.record(stream)
        step(x, evq)
        b.record(stream)
    torch.cuda.synchronize(dev)
    seconds = sum(a.elapsed_time(b) for a, b, _ in evs) / 1e3
    q_seconds = sum(e0.elapsed_time(e1) for _, _, (e0, e1) in evs) / 1e3
    dist.barrier()
    if dist.rank == 0:
        time.sleep(0.2)
        sampler.stop()
    max_seconds = dist.max(seconds, dev)
    value = nbytes * args.steps * dist.world / max_seconds / 1e9
    q_bytes = 3 * n + 4 * rows + 4 * rows
    achieved = q_bytes / (q_seconds / args.steps) / 1e9

    e2e_steps = max(3, min(args.steps, 10))
    hx = x.cpu().pin_memory()
    dx = torch.empty_like(x)
    hout = torch.empty(out.shape, dtype=torch.uint8).pin_memory()
    hs = torch.empty(sc.shape, dtype=sc.dtype).pin_memory()

    def e2e_step():
        dx.copy_(hx, non_blocking=True)
        step(dx)
        hout.copy_(out.view(torch.uint8), non_blocking=True)
        hs.copy_(sc, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(dev)
    dist.barrier()
    a, b = ev(), ev()
    a.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize(dev)
    e2e_s = dist.max(a.elapsed_time(b) / 1e3, dev)

    peaks, peaks_kind = load_peaks()
    peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    traffic = profiled_traffic(w.name, kind="ulysses_ops")
    clocks = sampler.summary(physical_gpu_index(dist.local_rank)) if dist.rank == 0 else {}
    line = {
        "metric": PAYLOAD_METRIC, "value": value, "unit": "GB/s", "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * max_seconds / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic", "config": payload_config(w, N),
        "e2e": {"value": nbytes * e2e_steps * dist.world / e2e_s / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": 2 * n, "d2h_bytes_per_step": n + 4 * rows,
                "steps": e2e_steps,
                "result_matches_device": bool(torch.equal(hout, out.view(torch.uint8).cpu()) and torch.equal(hs, sc.cpu()))},
        "gpu_launches": 3 * args.steps,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": f"HBM copy, {peaks_kind}", "traffic": traffic,
                     "kernel": "quantize_rows_kernel", "bytes_per_launch": q_bytes},
        "clocks": clocks,
    }
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        xr = x.reshape(rows, -1)[:8].cpu()
        rate, sr, dt = payload_oracle_rate(xr, xr.shape[0], N, w.B, args.cpu_seconds)
        line["cpu_baseline"] = {"value": rate, "unit": "GB/s", "cores": 1, "kind": "oracle",
                                "sample": f"fp64 numpy oracle on the first {sr} head(s) of {xr.shape[1]} values: {dt:.2f} s"}
    if dist.rank == 0:
        print(json.dumps(line), flush=True)


PER_WORKLOAD = ["flux_1024x768", "sd35_1024_fp8", "wan_720p_81f"]


def time_workload(w, dev, min_seconds: float = 1.0, warmup: int = 3):
    """Device-timed attention on one workload (inputs resident, L2 flushed between
    launches when the inputs fit in it), with its own clock record: a dict for the
    per_workload key of the bench line."""
    import torch
    import attention_dit_attn_b200 as dit
    from attention_dit_attn_b200 import workloads as wl
    inp = wl.generate_workload(w)
    q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
    kw = {}
    if inp.q_scale is not None:
        kw = dict(q_scale=inp.q_scale.to(dev).contiguous(), k_scale=inp.k_scale.to(dev).contiguous(),
                  v_scale=inp.v_scale.to(dev).contiguous())
    del inp
    o = torch.empty((w.B, w.H, w.L, w.D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.H, w.L), dtype=torch.float32, device=dev)
    cfg = workload_config(w)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev) if cfg["inputs_bytes"] <= L2_BYTES \
        else None
    stream = torch.cuda.current_stream(dev)
    call = lambda: dit.dit_attn_fwd(q, k, v, o, lse, scale=w.scale, stream=stream, **kw)
    for _ in range(warmup):
        call()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    call()
    b.record(stream)
    torch.cuda.synchronize(dev)
    steps = max(5, min(2000, int(min_seconds / max(a.elapsed_time(b) / 1e3, 1e-6))))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    sampler = ClockSampler()
    sampler.start()
    time.sleep(0.3)
    for e0, e1 in evs:
        if flush is not None:
            flush.fill_(1)
        host_gate(stream)
        e0.record(stream)
        call()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    time.sleep(0.2)
    sampler.stop()
    rc, word = dit.dit_attn_check_device_error(stream)
    if rc != 0:
        raise RuntimeError(f"device error while timing {w.name}: {word:#x}")
    sec = sum(e0.elapsed_time(e1) for e0, e1 in evs) / 1e3 / steps
    tflops = w.flops / sec / 1e12
    peaks, kind = load_peaks()
    bf16_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak = bf16_peak if w.dtype == "bf16" else 2.0 * bf16_peak
    return {"tflops": tflops, "ms_per_call": 1e3 * sec, "steps": steps, "dtype": w.dtype,
            "pct_of_nominal_dense": 100.0 * tflops / NOMINAL_TFLOPS[w.dtype],
            "frac": tflops / peak,
            "peak_source": f"bf16 {kind} (burst)" if w.dtype == "bf16" else f"fp8 = 2 x bf16 {kind} (burst)",
            "l2": cfg["l2"], "clocks": sampler.summary(None)}


def run_ours(args, dist: Dist):
    import torch
    import attention_dit_attn_b200 as dit
    from attention_dit_attn_b200 import workloads as wl

    dit.ensure_built()
    torch.cuda.set_device(dist.local_rank)
    dev = torch.device("cuda", dist.local_rank)
    w = wl.ALL[args.workload]
    inp = wl.generate_workload(w)
    q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
    kw = {}
    if inp.q_scale is not None:
        kw = dict(q_scale=inp.q_scale.to(dev).contiguous(), k_scale=inp.k_scale.to(dev).contiguous(),
                  v_scale=inp.v_scale.to(dev).contiguous())
    o = torch.empty((w.B, w.H, w.L, w.D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.H, w.L), dtype=torch.float32, device=dev)
    cfg = workload_config(w)
    flush = None
    if cfg["inputs_bytes"] <= L2_BYTES:
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        if flush is not None:
            flush.fill_(1)
        dit.dit_attn_fwd(q, k, v, o, lse, scale=w.scale, stream=stream, **kw)

    # ---- device-resident timing
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    rc, word = dit.dit_attn_check_device_error(stream)
    if rc != 0:
        raise RuntimeError(f"device error during warm-up: {word:#x}")
    sampler = ClockSampler()
    if dist.rank == 0:
        sampler.start()
        time.sleep(0.3)
    dist.barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if flush is None:
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        kernel_ms_total = e0.elapsed_time(e1)
        seconds = kernel_ms_total / 1e3
    else:
        # Flush between steps; time only the attention launches (per-launch events).
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        e0.record(stream)
        for a, b in evs:
            flush.fill_(1)
            host_gate(stream)
            a.record(stream)
            dit.dit_attn_fwd(q, k, v, o, lse, scale=w.scale, stream=stream, **kw)
            b.record(stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        kernel_ms_total = sum(a.elapsed_time(b) for a, b in evs)
        seconds = kernel_ms_total / 1e3
    dist.barrier()
    if dist.rank == 0:
        time.sleep(0.2)
        sampler.stop()
    rc, word = dit.dit_attn_check_device_error(stream)
    if rc != 0:
        raise RuntimeError(f"device error during the timed region: {word:#x}")
    max_seconds = dist.max(seconds, dev)
    value = aggregate(w.flops, args.steps, dist.world, max_seconds)
    kernel_avg_s = kernel_ms_total / 1e3 / args.steps
    launches = args.steps * dit.dit_attn_launches_per_call(w.B, w.H, w.L, w.D, 0 if w.dtype == "bf16" else 1)

    # ---- end to end through the public API, host buffers, copies in the timed region.
    # Every step copies its q/k/v in from pinned host memory and its o/lse back
    # out.  Two device buffer sets and three streams let the copies of one step
    # overlap the attention of the neighbouring step, as a serving loop would.
    e2e_steps = max(3, min(args.steps, 10))
    hq, hk, hv = (t.pin_memory() for t in (inp.q, inp.k, inp.v))
    ho = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    hl = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    bufs = [dict(q=torch.empty_like(q), k=torch.empty_like(k), v=torch.empty_like(v), o=torch.empty_like(o),
                 lse=torch.empty_like(lse)) for _ in range(2)]
    s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    in_done, cmp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def e2e_run(n_steps, start=None, end=None):
        if start is not None:
            start.record(s_in)
        for i in range(n_steps):
            b = i % 2
            buf = bufs[b]
            if i >= 2:
                s_in.wait_event(cmp_done[b])         # step i-2's attention has read this buffer set
            with torch.cuda.stream(s_in):
                buf["q"].copy_(hq, non_blocking=True)
                buf["k"].copy_(hk, non_blocking=True)
                buf["v"].copy_(hv, non_blocking=True)
            in_done[b].record(s_in)
            s_cmp.wait_event(in_done[b])
            if i >= 2:
                s_cmp.wait_event(out_done[b])        # step i-2's o/lse have been copied out
            dit.dit_attn_fwd(buf["q"], buf["k"], buf["v"], buf["o"], buf["lse"], scale=w.scale, stream=s_cmp,
                             **kw)
            cmp_done[b].record(s_cmp)
            s_out.wait_event(cmp_done[b])
            with torch.cuda.stream(s_out):
                ho.copy_(buf["o"], non_blocking=True)
                hl.copy_(buf["lse"], non_blocking=True)
            out_done[b].record(s_out)
        if end is not None:
            end.record(s_out)

    e2e_run(2)
    torch.cuda.synchronize(dev)
    dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_run(e2e_steps, a, b)
    torch.cuda.synchronize(dev)
    e2e_s = dist.max(a.elapsed_time(b) / 1e3, dev)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
    d2h = ho.numel() * ho.element_size() + hl.numel() * hl.element_size()
    last = bufs[(e2e_steps - 1) % 2]
    e2e_ok = bool(torch.equal(ho, last["o"].cpu()) and torch.equal(hl, last["lse"].cpu()) and torch.equal(ho, o.cpu()))

    peaks, peaks_kind = load_peaks()
    if w.dtype == "bf16":
        peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        peak_note = f"bf16 dense, {peaks_kind} (burst)"
    else:
        # FP8 contraction: measured bf16 peak x the nominal fp8/bf16 ratio (2x).
        peak = 2.0 * float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        peak_note = f"fp8 dense = 2 x bf16 {peaks_kind} (burst)"
    achieved = w.flops / kernel_avg_s / 1e12
    traffic = profiled_traffic(w.name)
    clocks = sampler.summary(physical_gpu_index(dist.local_rank)) if dist.rank == 0 else {}

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * max_seconds / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": w.dtype, "data": "synthetic",
        "config": cfg,
        "pct_of_peak": {"nominal_dense": 100.0 * value / dist.world / NOMINAL_TFLOPS[w.dtype],
                        "nominal_tflops": NOMINAL_TFLOPS[w.dtype]},
        "e2e": {"value": aggregate(w.flops, e2e_steps, dist.world, e2e_s), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "result_matches_device": e2e_ok},
        "gpu_launches": launches,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "peak_source": peak_note, "traffic": traffic,
                     "kernel": "dit::attn_fwd_kernel (CTA pair)", "flops_per_launch": w.flops},
        "clocks": clocks,
    }
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, inp, args.cpu_seconds)
    if dist.world == 1 and not args.no_per_workload:
        # The other configurations, each device-timed on its own (parity cases
        # too; reported beside the headline, not folded into it).
        del q, k, v, o, lse, bufs, hq, hk, hv, ho, hl, inp
        torch.cuda.empty_cache()
        line["per_workload"] = {name: time_workload(wl.ALL[name], dev) for name in PER_WORKLOAD
                                if name != w.name}
    if dist.rank == 0:
        print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="attention: skip the device timing of the other workloads (per_workload key)")
    ap.add_argument("--op", choices=["attention", "lse_merge", "residual_diff", "mxfp4_quant", "ulysses_fp8_payload",
                                     "gemm_fp8", "gemm_mxfp4"],
                    default="attention")
    ap.add_argument("--parts", type=int, default=2, help="lse_merge: number of partial results (ring degree)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    from attention_dit_attn_b200 import workloads as wl
    if args.workload not in wl.ALL:
        ap.error(f"--workload must be one of {list(wl.ALL)}")
    if not 1 <= args.parts <= 8:
        ap.error("--parts must be 1..8")
    if args.impl == "reference":
        # The oracle runs on rank 0's host cores only; other ranks exit at once.
        if int(os.environ.get("RANK", "0")) == 0:
            {"lse_merge": run_merge_reference, "residual_diff": run_diff_reference,
             "mxfp4_quant": run_mxfp4_reference, "ulysses_fp8_payload": run_payload_reference,
             "gemm_fp8": run_gemm_reference, "gemm_mxfp4": run_gemm_reference}.get(
                args.op, run_reference)(args, Dist.single())
        return
    dist = Dist(args.gpus)
    try:
        {"lse_merge": run_merge, "residual_diff": run_diff, "mxfp4_quant": run_mxfp4,
         "ulysses_fp8_payload": run_payload, "gemm_fp8": run_gemm, "gemm_mxfp4": run_gemm}.get(
            args.op, run_ours)(args, dist)
    finally:
        dist.close()


if __name__ == "__main__":
    main()
