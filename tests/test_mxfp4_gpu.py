"""GPU parity of dit_attn_mxfp4_quantize against the fp64 MXFP4 oracle, bit for
bit (codes and E8M0 scales): random activations, constructed ties, saturation,
signed zeros, subnormal and extreme blocks, and sampled rows at full size."""
import numpy as np
import pytest
import torch

from oracle import mxfp4

pytestmark = pytest.mark.gpu


def _gpu(x_bf16):
    import attention_dit_attn_b200 as dit
    q, s = dit.dit_attn_mxfp4_quantize(x_bf16.cuda())
    torch.cuda.synchronize()
    return q.cpu().numpy(), s.cpu().numpy()


def _check(x_bf16):
    q, s = _gpu(x_bf16)
    rq, rs = mxfp4.quantize(x_bf16.double().numpy().reshape(-1, x_bf16.shape[-1]))
    np.testing.assert_array_equal(s.reshape(rs.shape), rs)
    np.testing.assert_array_equal(q.reshape(rq.shape), rq)


@pytest.mark.parametrize("rows,K", [(1, 32), (7, 96), (33, 64), (1000, 3072), (3, 32 * 37)])
def test_random_activations_bit_exact(cuda_lib, rows, K):
    g = torch.Generator().manual_seed(rows * 1000 + K)
    scale = torch.exp2(torch.randint(-6, 6, (rows, 1), generator=g).float())
    x = (torch.randn((rows, K), generator=g) * scale).to(torch.bfloat16)
    _check(x)


def test_ties_saturation_and_signs(cuda_lib):
    ties = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.2490234375, 0.751953125]
    rows = []
    for s in (-3, 0, 4):
        blk = np.zeros(32)
        blk[0] = 6.0
        blk[1:1 + len(ties)] = ties
        blk[12:12 + len(ties)] = [-t for t in ties]
        blk[25], blk[26], blk[27], blk[28] = -0.01, -0.0, 0.0, -6.0
        rows.append(blk * 2.0 ** s)
        sat = np.zeros(32)
        sat[0], sat[1], sat[2] = 7.5, -7.0, 6.5                   # amax/2^s in (6, 8): saturation
        rows.append(sat * 2.0 ** s)
    _check(torch.tensor(np.stack(rows)).to(torch.bfloat16))


def test_zero_subnormal_and_extreme_blocks(cuda_lib):
    tiny = float(torch.tensor(2.0 ** -133, dtype=torch.bfloat16))   # bf16 subnormal
    big = float(torch.finfo(torch.bfloat16).max)
    rows = [np.zeros(32), -np.zeros(32), np.full(32, tiny), np.linspace(-big, big, 32),
            np.linspace(-1e-38, 1e-38, 32), np.full(32, 2.0 ** -126)]
    _check(torch.tensor(np.stack(rows)).to(torch.bfloat16))


def test_full_size_sampled_rows(cuda_lib):
    """The bench's activation size: (2 * 16896) x 3072 bf16; 256 sampled rows compared."""
    import attention_dit_attn_b200 as dit
    rows, K = 2 * 16896, 3072
    g = torch.Generator(device="cuda").manual_seed(7)
    x = torch.randn((rows, K), generator=g, device="cuda").to(torch.bfloat16)
    q, s = dit.dit_attn_mxfp4_quantize(x)
    torch.cuda.synchronize()
    idx = np.sort(np.random.default_rng(1).choice(rows, 256, replace=False))
    idx[0], idx[-1] = 0, rows - 1
    ti = torch.from_numpy(idx).cuda()
    rq, rs = mxfp4.quantize(x[ti].double().cpu().numpy())
    np.testing.assert_array_equal(s[ti].cpu().numpy(), rs)
    np.testing.assert_array_equal(q[ti].cpu().numpy(), rq)
