"""GPU parity of dit_attn_residual_diff (the step-cache reuse decision) against the
fp64 oracle: ragged sizes, exact boundary cases, zero residuals, determinism and
the workspace being left zeroed, and the bench's full size."""
import math

import numpy as np
import pytest
import torch

from oracle.residual_diff import residual_diff

pytestmark = pytest.mark.gpu

# fp32 sums over a few hundred elements per thread, fp64 beyond.
REL_TOL = 2e-6


def _residuals(n, change, seed):
    g = torch.Generator().manual_seed(seed)
    prev = torch.randn(n, generator=g)
    cur = prev + change * torch.randn(n, generator=g)
    return cur.to(torch.bfloat16), prev.to(torch.bfloat16)


def _run(cur, prev, thr, workspace=None):
    import attention_dit_attn_b200 as dit
    d, r = dit.dit_attn_residual_diff(cur.cuda(), prev.cuda(), thr, workspace=workspace)
    torch.cuda.synchronize()
    return float(d.item()), int(r.item())


@pytest.mark.parametrize("n", [1, 7, 8, 9, 1000, 4097, 65539, 3_000_001])
def test_matches_oracle(cuda_lib, n):
    cur, prev = _residuals(n, 0.08, seed=n)
    ref = residual_diff(cur.double().numpy(), prev.double().numpy())
    d, r = _run(cur, prev, 0.12)
    assert abs(d - ref) <= REL_TOL * ref + 1e-7, (d, ref)
    if abs(ref - 0.12) > 1e-4:
        assert r == int(ref < 0.12)


def test_exact_boundary_is_strict(cuda_lib):
    """1.125 against 1.0 everywhere: diff is exactly 0.125 in every precision."""
    n = 1 << 20
    prev = torch.ones(n, dtype=torch.bfloat16)
    cur = torch.full((n,), 1.125, dtype=torch.bfloat16)
    d, r = _run(cur, prev, 0.125)
    assert d == 0.125 and r == 0
    d, r = _run(cur, prev, 0.12500001)
    assert r == 1


def test_zero_residuals(cuda_lib):
    z = torch.zeros(4096, dtype=torch.bfloat16)
    d, r = _run(z, z, 0.12)
    assert d == 0.0 and r == 1
    d, r = _run(torch.ones(4096, dtype=torch.bfloat16), z, 1e30)
    assert math.isinf(d) and r == 0


def test_deterministic_and_workspace_left_zero(cuda_lib):
    import attention_dit_attn_b200 as dit
    cur, prev = _residuals(5_000_003, 0.2, seed=1)
    ws = torch.zeros(dit.dit_attn_residual_diff_workspace_bytes(cur.numel()), dtype=torch.uint8, device="cuda")
    a = _run(cur, prev, 0.12, workspace=ws)
    assert int(ws[:4].view(torch.int32).item()) == 0
    b = _run(cur, prev, 0.12, workspace=ws)
    assert a == b


@pytest.mark.parametrize("change,expect_reuse", [(0.02, 1), (0.05, 1), (0.3, 0), (1.0, 0)])
def test_decision_follows_the_change(cuda_lib, change, expect_reuse):
    cur, prev = _residuals(1 << 18, change, seed=int(change * 100))
    ref = residual_diff(cur.double().numpy(), prev.double().numpy())
    d, r = _run(cur, prev, 0.12)
    assert r == expect_reuse == int(ref < 0.12)


def test_full_size_bench_workload(cuda_lib):
    """flux_2048_cfg's hidden-state size: B * L * H * D = 2 * 16896 * 24 * 128 elements."""
    n = 2 * 16896 * 24 * 128
    g = torch.Generator(device="cuda").manual_seed(5)
    prev = torch.randn(n, generator=g, device="cuda")
    cur = (prev + 0.05 * torch.randn(n, generator=g, device="cuda")).to(torch.bfloat16)
    prev = prev.to(torch.bfloat16)
    ref = residual_diff(cur.cpu().double().numpy(), prev.cpu().double().numpy())
    d, r = _run(cur, prev, 0.12)
    assert abs(d - ref) <= REL_TOL * ref, (d, ref)
    assert r == 1
