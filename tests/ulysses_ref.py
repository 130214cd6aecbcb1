"""Reference implementations of the per-GPU Ulysses steps, for CPU tests of the
exchange logic with gloo ranks (tests only): layout moves with torch, the
quantisation recipe of the seeded generator, attention from the fp64 oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle

E4M3_MAX = 448.0


class RefOps:
    def block_transpose(self, x, R, C):
        b = x.contiguous().view(torch.uint8).reshape(R, C, -1)
        return b.permute(1, 0, 2).contiguous().view(x.dtype).reshape(x.shape)

    def absmax_rows(self, x, rows):
        return x.float().abs().reshape(rows, -1).amax(dim=1)

    def quantize_e4m3_rows(self, x, amax):
        rows = amax.numel()
        s = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
        y = (x.float().reshape(rows, -1) / s[:, None]).clamp(-E4M3_MAX, E4M3_MAX)
        return y.to(torch.float8_e4m3fn).reshape(x.shape), s

    def attention(self, q, k, v, scale, q_scale=None, k_scale=None, v_scale=None):
        if q.dtype == torch.bfloat16:
            bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
            o, lse = oracle.attention(bits(q), bits(k), bits(v), scale, dtype=oracle.BF16)
        else:
            codes = lambda t: t.contiguous().view(torch.uint8).numpy()
            o, lse = oracle.attention(codes(q), codes(k), codes(v), scale, dtype=oracle.E4M3,
                                      q_scale=q_scale.numpy(), k_scale=k_scale.numpy(), v_scale=v_scale.numpy())
        return torch.from_numpy(o).to(torch.bfloat16), torch.from_numpy(lse).to(torch.float32)
