"""GPU parity of dit_attn_lse_merge against the fp64 merge oracle, and of the
ring-attention composition (forward per key chunk, then merge) against the
full-attention oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle.lse_merge import lse_merge
from attention_dit_attn_b200 import workloads as wl
import parity

pytestmark = pytest.mark.gpu

# bf16 output rounding (round to nearest: relative 2^-8 at most) plus fp32
# accumulation and the MUFU exp2 on the weights.
O_REL = 2.0 ** -8
O_ABS = 1e-6
LSE_TOL = 2e-5


def _parts(rows, D, n, seed, empty=()):
    g = torch.Generator().manual_seed(seed)
    parts = []
    for c in range(n):
        o = torch.randn((rows, D), generator=g).to(torch.bfloat16)
        lse = (torch.randn((rows,), generator=g) * 3.0).float()
        if c in empty:
            lse[: rows // 2] = -math.inf          # the first half of the rows saw no key in this chunk
        parts.append((o, lse))
    return parts


def _check(o_gpu, lse_gpu, parts):
    o_ref, lse_ref = lse_merge([p[0].double().numpy() for p in parts], [p[1].double().numpy() for p in parts])
    og = o_gpu.double().cpu().numpy()
    err = np.abs(og - o_ref)
    assert (err <= O_REL * np.abs(o_ref) + O_ABS).all(), float((err - O_REL * np.abs(o_ref)).max())
    if lse_gpu is not None:
        lg = lse_gpu.double().cpu().numpy()
        assert np.allclose(lg, lse_ref, rtol=LSE_TOL, atol=LSE_TOL, equal_nan=False)


@pytest.mark.parametrize("rows,D,n", [(1, 128, 1), (7, 64, 2), (1000, 128, 2), (4097, 64, 3),
                                      (513, 128, 8), (333, 128, 5)])
def test_merge_matches_oracle(cuda_lib, rows, D, n):
    import attention_dit_attn_b200 as dit
    parts = _parts(rows, D, n, seed=rows * 31 + n)
    dev = [(o.cuda(), l.cuda()) for o, l in parts]
    o, lse = dit.dit_attn_lse_merge(dev)
    torch.cuda.synchronize()
    _check(o, lse, parts)


def test_merge_with_empty_chunks_and_all_empty_rows(cuda_lib):
    import attention_dit_attn_b200 as dit
    rows, D = 600, 128
    parts = _parts(rows, D, 3, seed=9, empty=(0, 2))
    # rows 0..9: no keys in any chunk -> o = 0, lse = -inf
    for o_, l_ in parts:
        l_[:10] = -math.inf
    o, lse = dit.dit_attn_lse_merge([(o_.cuda(), l_.cuda()) for o_, l_ in parts])
    torch.cuda.synchronize()
    assert (o[:10].float() == 0).all() and torch.isneginf(lse[:10]).all()
    _check(o[10:], lse[10:], [(o_[10:], l_[10:]) for o_, l_ in parts])


def test_merge_in_place_over_part_zero(cuda_lib):
    import attention_dit_attn_b200 as dit
    rows, D = 2049, 64
    parts = _parts(rows, D, 2, seed=4)
    dev = [(o.cuda(), l.cuda()) for o, l in parts]
    ref_o, ref_l = dit.dit_attn_lse_merge(dev)
    o, lse = dit.dit_attn_lse_merge(dev, o=dev[0][0], lse=dev[0][1])
    torch.cuda.synchronize()
    assert o.data_ptr() == dev[0][0].data_ptr()
    assert torch.equal(o, ref_o) and torch.equal(lse, ref_l)


def test_merge_without_lse_and_zero_rows(cuda_lib):
    import attention_dit_attn_b200 as dit
    parts = _parts(300, 128, 2, seed=5)
    dev = [(o.cuda(), l.cuda()) for o, l in parts]
    o, lse = dit.dit_attn_lse_merge(dev, want_lse=False)
    torch.cuda.synchronize()
    assert lse is None
    _check(o, None, parts)
    empty = [(torch.empty((0, 64), dtype=torch.bfloat16, device="cuda"),
              torch.empty((0,), dtype=torch.float32, device="cuda"))] * 2
    o0, l0 = dit.dit_attn_lse_merge(empty)
    assert o0.numel() == 0 and l0.numel() == 0


@pytest.mark.parametrize("B,H,Lc,D,dt,n", [(1, 2, 1000, 128, "bf16", 2), (2, 2, 300, 64, "bf16", 3),
                                           (1, 2, 700, 128, "e4m3", 2)])
def test_ring_attention_composition(cuda_lib, B, H, Lc, D, dt, n):
    """Each query chunk meets the n key chunks through dit_attn_fwd (equal lengths, as
    in ring attention); the merged result must match the oracle's attention over all keys."""
    import attention_dit_attn_b200 as dit
    L = n * Lc
    inp = wl.generate(B, H, L, D, dt, seed=77 + n)
    sc = 1 / math.sqrt(D)
    o_ref, lse_ref = parity.run_oracle(inp, sc)
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    kw = {}
    if inp.q_scale is not None:
        kw = dict(q_scale=inp.q_scale.cuda().contiguous(), k_scale=inp.k_scale.cuda().contiguous(),
                  v_scale=inp.v_scale.cuda().contiguous())
    o_all = torch.empty((B, H, L, D), dtype=torch.bfloat16)
    lse_all = torch.empty((B, H, L), dtype=torch.float32)
    for r in range(n):
        qs = q[:, :, r * Lc:(r + 1) * Lc].contiguous()
        parts = [dit.dit_attn_fwd(qs, k[:, :, c * Lc:(c + 1) * Lc].contiguous(),
                                  v[:, :, c * Lc:(c + 1) * Lc].contiguous(), scale=sc, **kw)
                 for c in range(n)]
        o, lse = dit.dit_attn_lse_merge(parts)
        torch.cuda.synchronize()
        o_all[:, :, r * Lc:(r + 1) * Lc] = o.cpu()
        lse_all[:, :, r * Lc:(r + 1) * Lc] = lse.cpu()
    assert dit.dit_attn_check_device_error()[0] == 0
    m = parity.compare(o_all, lse_all, o_ref, lse_ref)
    parity.check(m, dt)


def test_merge_full_size_sampled_rows(cuda_lib):
    """The bench's merge workload (2 parts of flux_2048_cfg's shape), 4096 sampled rows."""
    import attention_dit_attn_b200 as dit
    rows, D = 2 * 24 * 16896, 128
    g = torch.Generator(device="cuda").manual_seed(12)
    dev = [(torch.randn((rows, D), generator=g, device="cuda").to(torch.bfloat16),
            torch.randn((rows,), generator=g, device="cuda") * 3.0) for _ in range(2)]
    o, lse = dit.dit_attn_lse_merge(dev)
    torch.cuda.synchronize()
    idx = torch.from_numpy(np.random.default_rng(3).choice(rows, 4096, replace=False)).cuda()
    idx[0], idx[1] = 0, rows - 1
    parts = [(p[0][idx].cpu(), p[1][idx].cpu()) for p in dev]
    _check(o[idx].cpu(), lse[idx].cpu(), parts)
