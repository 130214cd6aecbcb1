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


def ulysses_attention_fused(q, k, v, *, group=None, scale: float | None = None, q_scale=None, k_scale=None,
                            v_scale=None):
    """The fused path of ulysses_attention: the same inputs (this rank's shard
    [B, H, Ls, D] of q, k, v; FP8 with [B, H] per-head scales agreed by all ranks)
    and the same result (this rank's shard of O and the LSE over the whole
    sequence), computed by dit_attn_fwd_ulysses with every rank's shards mapped
    into this process through CUDA IPC.  All ranks of ``group`` run on one node;
    ``group`` may be any backend (it carries only the IPC handles and barriers).
    Ls must be a multiple of 64 and H a multiple of the group size."""
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
    shards = [local if c == rank else [fn(*args) for fn, args in handles[c]] for c in range(N)]
    torch.cuda.synchronize(q.device)
    dist.barrier(group=group)            # every rank's q/k/v are written and mapped
    dit_attn_fwd_ulysses([s[0] for s in shards], [s[1] for s in shards], [s[2] for s in shards],
                         [s[3] for s in shards], [s[4] for s in shards], rank=rank, scale=scale,
                         q_scale=q_scale, k_scale=k_scale, v_scale=v_scale)
    torch.cuda.synchronize(q.device)
    dist.barrier(group=group)            # every rank's writes into this rank's o/lse are done
    del shards, handles
    dist.barrier(group=group)            # no rank still maps another's memory
    return o, lse
