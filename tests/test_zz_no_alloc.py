"""dit_attn_residual_diff_noalloc (the library's fixed device scratch, no workspace,
no allocation) against dit_attn_residual_diff with a caller workspace, on two calls
in a row: the second call checks that the first left the shared scratch ready."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def _residuals(n, change, seed):
    g = torch.Generator().manual_seed(seed)
    prev = torch.randn(n, generator=g)
    cur = prev + change * torch.randn(n, generator=g)
    return cur.to(torch.bfloat16).cuda(), prev.to(torch.bfloat16).cuda()


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row(cuda_lib):
    import attention_dit_attn_b200 as dit
    cases = [(_residuals(10_000_019, 0.08, 1), 0.12),     # many blocks, ragged tail
             (_residuals(4_099, 0.3, 2), 0.12)]            # then a grid of a few blocks
    for (cur, prev), thr in cases:
        ws = torch.zeros(dit.dit_attn_residual_diff_workspace_bytes(cur.numel()), dtype=torch.uint8,
                         device="cuda")
        d_ref, r_ref = dit.dit_attn_residual_diff(cur, prev, thr, workspace=ws)
        d_na, r_na = dit.dit_attn_residual_diff_noalloc(cur, prev, thr)
        torch.cuda.synchronize()
        assert torch.equal(d_na, d_ref) and torch.equal(r_na, r_ref), (d_na, d_ref, r_na, r_ref)
    # and the same inputs twice more: identical bits each time
    (cur, prev), thr = cases[0]
    a = dit.dit_attn_residual_diff_noalloc(cur, prev, thr)
    b = dit.dit_attn_residual_diff_noalloc(cur, prev, thr)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
