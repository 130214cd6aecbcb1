"""Ulysses sequence parallelism around the DiT attention (optional FP8 payload).

Page "How to Scale Diffusion Inference Across AMD RDNA 4 GPUs", section
"Balance Transformer Work and Communication": Ulysses divides the tokens that
attention processes across GPUs, every attention layer exchanges data between
them with an all-to-all, and `--use fp8 comms` sends that exchange in FP8.

Each of the N ranks of ``group`` holds a sequence shard of q, k, v: all H heads
of Ls = L / N consecutive tokens, [B, H, Ls, D].  Per attention layer:

  1. (FP8) per-(b, h) absmax of each shard, all-reduced (max) over the group, so
     every rank quantises its shard with the same per-head scale s = amax / 448;
  2. group heads by destination (block transpose), all-to-all: each rank now
     holds all L tokens of H / N heads, [B, H/N, L, D] (block transpose back);
  3. attention over the full sequence on those heads (dit_attn_fwd; in FP8 the
     received e4m3 tensors and the global scales are exactly its FP8 inputs);
  4. the inverse exchange of O (and the LSE) back to sequence shards.

The exchange is torch.distributed (NCCL between GPUs).  The per-GPU steps go
through ``ops``: by default this library's kernels (dit_attn_block_transpose,
dit_attn_absmax_rows, dit_attn_quantize_e4m3_rows, dit_attn_fwd); tests on CPU
pass reference ops to check the exchange logic with gloo ranks.

dit_attn_fwd_ulysses is the fused alternative: given every rank's shard
pointers (peers' memory mapped into this context), one kernel per rank reads
the tiles from the shards and writes O and the LSE back into them, with no
all-to-all and no gathered copy.
"""
from __future__ import annotations

import math


class KernelOps:
    """The per-GPU steps, on this library's CUDA kernels."""

    def block_transpose(self, x, R, C):
        from . import dit_attn_block_transpose
        return dit_attn_block_transpose(x, R, C)

    def absmax_rows(self, x, rows):
        from . import dit_attn_absmax_rows
        return dit_attn_absmax_rows(x, rows)

    def quantize_e4m3_rows(self, x, amax):
        from . import dit_attn_quantize_e4m3_rows
        return dit_attn_quantize_e4m3_rows(x, amax)

    def attention(self, q, k, v, scale, q_scale=None, k_scale=None, v_scale=None):
        from . import dit_attn_fwd
        return dit_attn_fwd(q, k, v, scale=scale, q_scale=q_scale, k_scale=k_scale, v_scale=v_scale)


def _all_to_all(x, group):
    """Equal-split all-to-all of a contiguous tensor's bytes (FP8 travels as uint8)."""
    import torch
    import torch.distributed as dist
    send = x.view(torch.uint8) if x.dtype == torch.float8_e4m3fn else x
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv.reshape(-1), send.reshape(-1), group=group)
    return recv.view(x.dtype) if x.dtype == torch.float8_e4m3fn else recv


def ulysses_attention(q, k, v, *, group=None, scale: float | None = None, fp8_comm: bool = False, ops=None):
    """q, k, v: this rank's shard [B, H, Ls, D] (bf16; tokens rank*Ls .. rank*Ls + Ls of
    the joint sequence, all heads).  Returns (o [B, H, Ls, D] bf16, lse [B, H, Ls] fp32),
    this rank's shard of attention over the whole sequence."""
    import torch
    import torch.distributed as dist
    ops = ops or KernelOps()
    N = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, H, Ls, D = q.shape
    if H % N:
        raise ValueError(f"{H} heads do not split over {N} ranks")
    Hn = H // N
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    scales = [None, None, None]
    payload = [q, k, v]
    if fp8_comm:
        amax = torch.stack([ops.absmax_rows(t, B * H) for t in (q, k, v)])      # [3, B*H]
        dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
        payload, scales = [], []
        for t, a in zip((q, k, v), amax):
            qt, st = ops.quantize_e4m3_rows(t, a.contiguous())
            payload.append(qt)
            # this rank's heads after the exchange: [B, Hn]
            scales.append(st.view(B, H)[:, rank * Hn:(rank + 1) * Hn].contiguous())
    full = []
    for t in payload:
        # [B, N, Hn, Ls, D] -> [N, B, Hn, Ls, D]: heads grouped by destination rank
        send = ops.block_transpose(t.contiguous(), B, N)
        recv = _all_to_all(send, group)
        # [N(src), B*Hn, Ls, D] -> [B*Hn, N(src), Ls, D] = [B, Hn, L, D]
        full.append(ops.block_transpose(recv, N, B * Hn).view(B, Hn, N * Ls, D))
    o, lse = ops.attention(full[0], full[1], full[2], scale, *scales)
    # O back: [B*Hn, N(dst), Ls, D] -> [N(dst), B*Hn, Ls, D] -> exchange -> [N(src), B, Hn, Ls, D]
    # -> [B, N(src), Hn, Ls, D] = [B, H, Ls, D]
    o_recv = _all_to_all(ops.block_transpose(o.contiguous(), B * Hn, N), group)
    o_out = ops.block_transpose(o_recv, N, B).view(B, H, Ls, D)
    l_recv = _all_to_all(ops.block_transpose(lse.contiguous(), B * Hn, N), group)
    l_out = ops.block_transpose(l_recv, N, B).view(B, H, Ls)
    return o_out, l_out


class HostBarrier:
    """Barrier of the ranks of one node over a small POSIX shared-memory block,
    which also tells every rank whether all ranks arrived healthy.

    Rank r writes ``epoch << 1 | ok`` into its own 8-byte slot of row
    ``epoch % 2`` and spins until every slot of that row has reached the epoch.
    Each slot has one writer and one aligned 8-byte store, so no atomics are
    needed.  Two rows keep a fast rank's next epoch from overwriting a status a
    slow rank has not read yet: no rank can reach epoch + 2 before every rank
    has left epoch.  A rank that does not arrive within ``timeout_s`` (it died
    or raised) makes the others raise TimeoutError instead of hanging.
    Latency is a few microseconds, against about a hundred for a gloo barrier."""

    def __init__(self, group=None, timeout_s: float = 60.0):
        import numpy as np
        import torch.distributed as dist
        from multiprocessing import resource_tracker, shared_memory
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.timeout_s = float(timeout_s)
        nbytes = 2 * self.world * 8
        name = [None]
        if self.rank == 0:
            self._shm = shared_memory.SharedMemory(create=True, size=nbytes)
            self._shm.buf[:nbytes] = bytes(nbytes)
            name[0] = self._shm.name
        dist.broadcast_object_list(name, src=dist.get_global_rank(group, 0) if group is not None else 0,
                                   group=group)
        if self.rank != 0:
            self._shm = shared_memory.SharedMemory(name=name[0])
            # Attaching registers the block with this process's resource tracker,
            # which would unlink it at exit under the owner's feet.
            resource_tracker.unregister(self._shm._name, "shared_memory")
        dist.barrier(group=group)
        if self.rank == 0:
            self._shm.unlink()          # every rank has it mapped; the name is no longer needed
        self._slots = np.ndarray((2, self.world), dtype=np.int64, buffer=self._shm.buf)
        self.epoch = 0

    def wait(self, ok: bool = True) -> list[bool]:
        """Arrive with this rank's status; returns every rank's status."""
        import time
        self.epoch += 1
        row = self._slots[self.epoch % 2]
        row[self.rank] = (self.epoch << 1) | int(bool(ok))
        t0 = time.monotonic()
        while True:
            vals = row.copy()
            if ((vals >> 1) >= self.epoch).all():
                return [bool(x & 1) for x in vals]
            if time.monotonic() - t0 > self.timeout_s:
                late = [c for c in range(self.world) if (vals[c] >> 1) < self.epoch]
                raise TimeoutError(f"host barrier {self.epoch}: ranks {late} did not arrive in {self.timeout_s} s")
            time.sleep(0)

    def close(self):
        if self._shm is not None:
            self._slots = None
            self._shm.close()
            self._shm = None


class UlyssesFusedError(RuntimeError):
    """Raised on every rank when any rank's part of a fused Ulysses call failed."""


def _fused_device_status(stream) -> tuple[bool, int]:
    """Read (and clear) the fused kernel's device error word: (ok, word)."""
    from . import dit_attn_ulysses_check_device_error
    rc, word = dit_attn_ulysses_check_device_error(stream)
    return rc == 0, word


class FusedUlysses:
    """Fused Ulysses attention as a per-layer call, for the ranks of one node (one
    process per GPU, or several processes sharing a GPU).

    Set-up, once: every rank allocates persistent shard buffers for the largest
    shape it will run (q, k, v in the input dtype, O bf16, LSE fp32), the ranks
    exchange their CUDA IPC memory and event handles over ``group``, and each
    maps the others' buffers.  Each call then:

      1. copies this rank's q/k/v shard into its buffers on its stream (the
         stream already waited, at the end of the previous call, for every
         rank's kernel that read them);
      2. records an interprocess event, meets the other ranks at a host barrier
         that also carries each rank's status, and makes its stream wait on
         every rank's event (GPU-side ordering across processes);
      3. launches dit_attn_fwd_ulysses, which reads every rank's q/k/v tiles and
         writes O and the LSE into the shard each row belongs to;
      4. records a second event, meets the ranks at a second barrier and waits
         on their second events, so this rank's O/LSE buffers are complete in
         stream order when the call returns.

    The only host synchronisation is the two barriers (shared memory, a few
    microseconds): no device-wide synchronise, no handle exchange per call.
    A failure on one rank (an argument error, a launch error) is seen by all
    ranks at the next barrier, and all raise UlyssesFusedError together.
    Device-side wait timeouts of the kernel are read by ``check()``, which
    synchronises this rank's stream; call it at a step boundary (once per
    denoising step, say) and every rank raises if any rank's kernel gave up.

    All ranks call in the same order with the same shape.  Plain peer loads and
    stores only: the kernel's tensor maps cover peers' memory without cluster
    multicast."""

    def __init__(self, group=None, *, B: int, H: int, Ls: int, D: int, dtype=None, device=None,
                 timeout_s: float = 60.0):
        import torch
        import torch.distributed as dist
        from torch.multiprocessing.reductions import reduce_tensor
        self.group = group
        self.N = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        dtype = torch.bfloat16 if dtype is None else dtype
        if dtype not in (torch.bfloat16, torch.float8_e4m3fn):
            raise TypeError(f"unsupported dtype {dtype}")
        # Checked before any collective, so every rank fails the same way.
        if H % self.N or Ls % 64 or Ls < 64 or self.N > 8 or D not in (64, 128) or B < 1:
            raise ValueError(f"need H % ranks == 0, Ls a multiple of 64, at most 8 ranks and D in (64, 128) "
                             f"(H={H}, Ls={Ls}, ranks={self.N}, D={D})")
        self.B, self.H, self.Ls_max, self.D, self.dtype = B, H, Ls, D, dtype
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.stream = torch.cuda.Stream(self.device)
        n_in = B * H * Ls * D
        with torch.cuda.device(self.device):
            bufs = [torch.empty(n_in, dtype=torch.uint8 if dtype == torch.float8_e4m3fn else dtype,
                                device=self.device) for _ in range(3)]
            bufs.append(torch.empty(n_in, dtype=torch.bfloat16, device=self.device))
            bufs.append(torch.empty(B * H * Ls, dtype=torch.float32, device=self.device))
            self._ev_in = torch.cuda.Event(interprocess=True)
            self._ev_out = torch.cuda.Event(interprocess=True)
        self.barrier = HostBarrier(group, timeout_s)
        handles = [None] * self.N
        dist.all_gather_object(handles, ([reduce_tensor(t) for t in bufs],
                                         self._ev_in.ipc_handle(), self._ev_out.ipc_handle()), group=group)
        self._bufs = []
        self._peer_in, self._peer_out = [], []
        for c in range(self.N):
            if c == self.rank:
                self._bufs.append(bufs)
                self._peer_in.append(self._ev_in)
                self._peer_out.append(self._ev_out)
            else:
                tens, h_in, h_out = handles[c]
                self._bufs.append([fn(*args) for fn, args in tens])
                self._peer_in.append(torch.cuda.Event.from_ipc_handle(self.device, h_in))
                self._peer_out.append(torch.cuda.Event.from_ipc_handle(self.device, h_out))
        self.barrier.wait()            # every rank has mapped every other rank's buffers
        self.closed = False

    def _views(self, c: int, Ls: int):
        import torch
        q, k, v, o, lse = self._bufs[c]
        n = self.B * self.H * Ls * self.D
        shape = (self.B, self.H, Ls, self.D)
        cast = (lambda t: t.view(torch.float8_e4m3fn)) if self.dtype == torch.float8_e4m3fn else (lambda t: t)
        return ([cast(t[:n]).view(shape) for t in (q, k, v)] + [o[:n].view(shape),
                                                                 lse[:self.B * self.H * Ls].view(self.B, self.H, Ls)])

    def __call__(self, q, k, v, *, scale: float | None = None, q_scale=None, k_scale=None, v_scale=None,
                 copy_out: bool = True):
        """This rank's shard [B, H, Ls, D] of q, k, v (Ls <= the set-up Ls, a multiple
        of 64, the same on every rank); FP8 with [B, H] per-head scales agreed by all
        ranks.  Returns (o [B, H, Ls, D] bf16, lse [B, H, Ls] fp32), this rank's shard
        of attention over the whole sequence, complete in the order of torch's
        current stream.  With copy_out=False they are views of the persistent
        buffers, overwritten by the next call."""
        import torch
        from . import dit_attn_fwd_ulysses
        if self.closed:
            raise RuntimeError("FusedUlysses is closed")
        err = None
        try:
            B, H, Ls, D = q.shape
            if (B, H, D) != (self.B, self.H, self.D) or Ls > self.Ls_max or Ls % 64 or Ls < 64:
                raise ValueError(f"shard shape {tuple(q.shape)} does not fit the set-up "
                                 f"[{self.B}, {self.H}, <= {self.Ls_max}, {self.D}] (Ls a multiple of 64)")
            if not (q.dtype == k.dtype == v.dtype == self.dtype) or not (q.shape == k.shape == v.shape):
                raise ValueError("q, k, v must share the set-up dtype and one shape")
            views = [self._views(c, Ls) for c in range(self.N)]
            cur = torch.cuda.current_stream(self.device)
            self.stream.wait_stream(cur)              # the caller's q/k/v are written
            with torch.cuda.stream(self.stream):
                for dst, src in zip(views[self.rank][:3], (q, k, v)):
                    dst.copy_(src)
                self._ev_in.record(self.stream)
        except Exception as e:  # noqa: BLE001 - reported to every rank below
            err = e
        if not all(self.barrier.wait(err is None)):
            raise UlyssesFusedError(f"rank {self.rank}: a rank failed before the fused attention") from err
        try:
            for c in range(self.N):
                if c != self.rank:
                    self.stream.wait_event(self._peer_in[c])
            dit_attn_fwd_ulysses([w[0] for w in views], [w[1] for w in views], [w[2] for w in views],
                                 [w[3] for w in views], [w[4] for w in views], rank=self.rank, scale=scale,
                                 q_scale=q_scale, k_scale=k_scale, v_scale=v_scale, stream=self.stream)
            self._ev_out.record(self.stream)
        except Exception as e:  # noqa: BLE001
            err = e
            self._ev_out.record(self.stream)          # peers still wait on this event
        if not all(self.barrier.wait(err is None)):
            raise UlyssesFusedError(f"rank {self.rank}: a rank's fused attention failed to launch") from err
        for c in range(self.N):
            if c != self.rank:
                self.stream.wait_event(self._peer_out[c])
        cur.wait_stream(self.stream)
        o, lse = views[self.rank][3], views[self.rank][4]
        if copy_out:
            o, lse = o.clone(), lse.clone()
        return o, lse

    def check(self):
        """Synchronise this rank's stream and read the fused kernel's device error
        word; every rank raises UlyssesFusedError if any rank's kernel gave up a wait
        (its outputs since the last check are then not to be trusted)."""
        ok, word = _fused_device_status(self.stream)
        if not all(self.barrier.wait(ok)):
            raise UlyssesFusedError(f"rank {self.rank}: a fused attention kernel timed out "
                                    f"(this rank's error word {word:#x})")

    def close(self):
        """Release the peers' mappings once no rank's kernel uses them (collective)."""
        if self.closed:
            return
        import torch
        self.stream.synchronize()
        self.barrier.wait()
        self._bufs = [self._bufs[self.rank]]
        self._peer_in = self._peer_out = []
        torch.cuda.synchronize(self.device)
        self.barrier.wait()
        self.barrier.close()
        self.closed = True


def ulysses_attention_fused(q, k, v, *, group=None, scale: float | None = None, q_scale=None, k_scale=None,
                            v_scale=None):
    """The fused path of ulysses_attention as a one-off call: the same inputs (this
    rank's shard [B, H, Ls, D] of q, k, v; FP8 with [B, H] per-head scales agreed by
    all ranks) and the same result (this rank's shard of O and the LSE over the whole
    sequence), computed by dit_attn_fwd_ulysses with every rank's own tensors mapped
    into this process through CUDA IPC.  All ranks of ``group`` run on one node;
    ``group`` may be any backend (it carries the IPC handles and statuses).
    Ls must be a multiple of 64 and H a multiple of the group size.

    Each call exchanges handles, synchronises and reads the kernel's device error
    word, and every rank raises UlyssesFusedError if any rank failed.  For one call
    per transformer layer use FusedUlysses, which does the set-up once."""
    import torch
    import torch.distributed as dist
    from torch.multiprocessing.reductions import reduce_tensor

    from . import dit_attn_fwd_ulysses
    N = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, H, Ls, D = q.shape
    # Checked before any collective, so every rank fails the same way.
    if H % N or Ls % 64 or N > 8:
        raise ValueError(f"need H % ranks == 0, Ls % 64 == 0 and at most 8 ranks (H={H}, Ls={Ls}, ranks={N})")
    o = torch.empty((B, H, Ls, D), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, H, Ls), dtype=torch.float32, device=q.device)
    local = [t.contiguous() for t in (q, k, v)] + [o, lse]
    handles = [None] * N
    dist.all_gather_object(handles, [reduce_tensor(t) for t in local], group=group)

    def exchange(status):
        got = [None] * N
        dist.all_gather_object(got, status, group=group)
        return got

    err, word, shards = None, 0, None
    try:
        shards = [local if c == rank else [fn(*args) for fn, args in handles[c]] for c in range(N)]
        torch.cuda.synchronize(q.device)
    except Exception as e:  # noqa: BLE001 - reported to every rank below
        err = e
    # every rank's q/k/v are written and mapped (the exchange is the barrier)
    if all(ok for ok, _ in exchange((err is None, 0))):
        try:
            dit_attn_fwd_ulysses([s[0] for s in shards], [s[1] for s in shards], [s[2] for s in shards],
                                 [s[3] for s in shards], [s[4] for s in shards], rank=rank, scale=scale,
                                 q_scale=q_scale, k_scale=k_scale, v_scale=v_scale)
            ok, word = _fused_device_status(torch.cuda.current_stream(q.device))
            if not ok:
                err = UlyssesFusedError(f"device error word {word:#x}")
        except Exception as e:  # noqa: BLE001
            err = e
        statuses = exchange((err is None, word))   # every rank's writes into this rank's o/lse are done
    else:
        statuses = [(False, 0)]
    del shards, handles
    dist.barrier(group=group)                     # no rank still maps another's memory
    if not all(ok for ok, _ in statuses):
        bad = [c for c, (ok, _) in enumerate(statuses) if not ok]
        raise UlyssesFusedError(f"rank {rank}: fused Ulysses attention failed on ranks {bad} "
                                f"(error words {[hex(w) for _, w in statuses]})") from err
    return o, lse
