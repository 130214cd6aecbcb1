"""GPU parity of the Ulysses FP8 payload kernels against the fp64 payload oracle,
bit for bit: rows split over many CTAs (ragged last chunk, more rows than one
grid dimension holds, zero and saturated rows), and the bench's full-size
tensor (flux_2048_cfg's [2, 24, 16896, 128]) with every head maximum, three
heads' codes and scales, and the whole head grouping for 8 ranks compared."""
import numpy as np
import pytest
import torch

from oracle import e4m3_payload as ep

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,row_len", [(3, 300016), (1, 16), (5, 16 * 1024 + 32), (70000, 16)])
def test_chunked_rows_match_oracle(cuda_lib, rows, row_len):
    import attention_dit_attn_b200 as dit
    g = torch.Generator().manual_seed(rows + row_len)
    x = torch.randn((rows, row_len), generator=g) * torch.exp2(torch.randint(-6, 6, (rows, 1), generator=g).float())
    x = x.to(torch.bfloat16)
    if rows > 2:
        x[1] = 0
    xd = x.cuda()
    amax = dit.dit_attn_absmax_rows(xd, rows)
    torch.cuda.synchronize()
    xn = x.double().numpy()
    ra = ep.absmax_rows(xn, rows)
    assert np.array_equal(amax.cpu().numpy(), ra.astype(np.float32))
    if rows > 2:
        amax[2] *= 0.5                                   # half the true max: codes saturate at 448
        ra[2] *= 0.5
    q, s = dit.dit_attn_quantize_e4m3_rows(xd, amax)
    torch.cuda.synchronize()
    rq, rs = ep.quantize_rows(xn, ra)
    assert np.array_equal(s.cpu().numpy(), rs)
    assert np.array_equal(q.cpu().view(torch.uint8).numpy(), rq)


def test_full_size_payload_matches_oracle(cuda_lib):
    import attention_dit_attn_b200 as dit
    B, H, L, D, N = 2, 24, 16896, 128, 8
    rows = B * H
    g = torch.Generator(device="cuda").manual_seed(1003)
    x = torch.randn((B, H, L, D), generator=g, device="cuda").to(torch.bfloat16)
    amax = dit.dit_attn_absmax_rows(x, rows)
    q, s = dit.dit_attn_quantize_e4m3_rows(x, amax)
    out = dit.dit_attn_block_transpose(q, B, N)
    torch.cuda.synchronize()
    xc = x.reshape(rows, -1).cpu()
    ra = np.array([ep.absmax_rows(xc[r].double().numpy(), 1)[0] for r in range(rows)])
    assert np.array_equal(amax.cpu().numpy(), ra.astype(np.float32))
    qc = q.reshape(rows, -1).cpu().view(torch.uint8).numpy()
    for r in (0, 23, rows - 1):
        rq, rs = ep.quantize_rows(xc[r:r + 1].double().numpy(), ra[r:r + 1])
        assert np.array_equal(qc[r:r + 1], rq) and s[r].item() == rs[0]
    assert np.array_equal(out.cpu().view(torch.uint8).numpy().reshape(-1), ep.block_transpose(qc, B, N))
