"""Pins of the Ulysses FP8 payload oracle (oracle/e4m3_payload.py) to facts
outside it: values of the OCP E4M3 format fixed by its definition, the rounding
rule at every midpoint, saturation and underflow, torch's float8_e4m3fn
conversion (a library routine) and the generator's quantisation recipe as the
attention inputs use it."""
import numpy as np
import pytest
import torch

from oracle import e4m3_payload as ep
from ulysses_ref import RefOps


def test_decode_table_matches_the_format_and_torch():
    t = ep.decode_table()
    # Values fixed by the format: bias 7, 3 mantissa bits, subnormals m/8 * 2^-6.
    assert t[0x38] == 1.0 and t[0x3C] == 1.5 and t[0xB8] == -1.0
    assert t[0x7E] == 448.0 and t[0xFE] == -448.0
    assert t[0x01] == 2.0 ** -9 and t[0x07] == 7 * 2.0 ** -9 and t[0x08] == 2.0 ** -6
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF]) and np.isnan(t).sum() == 2
    lib = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    fin = ~np.isnan(t)
    assert np.array_equal(fin, ~np.isnan(lib)) and np.array_equal(t[fin], lib[fin])


def test_every_finite_code_round_trips():
    t = ep.decode_table()
    codes = np.array([c for c in range(256) if not np.isnan(t[c])])
    assert np.array_equal(ep.encode(t[codes]), codes.astype(np.uint8))


def test_midpoints_round_to_the_even_code_and_neighbours_to_the_nearest():
    t = ep.decode_table()
    for c in range(0x7E):
        a, b = t[c], t[c + 1]
        mid = (a + b) / 2
        even = c if c % 2 == 0 else c + 1
        assert ep.encode(np.array([mid]))[0] == even, c
        assert ep.encode(np.array([-mid]))[0] == even | 0x80, c
        eps = (b - a) * 1e-6
        assert ep.encode(np.array([mid - eps]))[0] == c
        assert ep.encode(np.array([mid + eps]))[0] == c + 1


def test_saturation_underflow_and_signed_zero():
    v = np.array([448.0, 463.9, 464.0, 500.0, 1e30, -1e30, 2.0 ** -10, 2.0 ** -10 * 1.001,
                  -2.0 ** -11, -0.0, 0.0])
    assert list(ep.encode(v)) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x00, 0x01, 0x80, 0x80, 0x00]


def test_encode_matches_torch_conversion_in_range():
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.standard_normal(50000) * 60, rng.standard_normal(20000) * 1e-2,
                        rng.uniform(-448, 448, 20000)])
    x32 = np.clip(x, -448, 448).astype(np.float32)
    lib = torch.from_numpy(x32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ep.encode(x32.astype(np.float64)), lib)


def test_absmax_and_scales():
    x = np.array([[0.5, -3.0, 2.0, 1.0], [0.0, 0.0, -0.0, 0.0], [448.0, 1.0, -7.0, 0.25]])
    amax = ep.absmax_rows(x, 3)
    assert list(amax) == [3.0, 0.0, 448.0]
    s = ep.row_scales(amax)
    assert s.dtype == np.float32
    assert s[0] == np.float32(3.0 / 448.0) and s[1] == 1.0 and s[2] == 1.0


def test_quantize_rows_puts_the_absmax_element_at_448_and_zero_rows_at_0():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((4, 64)) * np.array([[1.0], [1e-3], [50.0], [0.0]])
    x = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    amax = ep.absmax_rows(x, 4)
    q, s = ep.quantize_rows(x, amax)
    for r in range(3):
        i = int(np.argmax(np.abs(x[r])))
        assert q[r, i] & 0x7F == 0x7E
        assert (q[r] & 0x7F).max() == 0x7E
    assert s[3] == 1.0 and not (q[3] & 0x7F).any()          # -0.0 inputs keep their sign bit


@pytest.mark.parametrize("seed", [1, 2])
def test_quantize_rows_matches_the_generator_recipe(seed):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn((6, 4, 96), generator=g) * torch.exp2(torch.randint(-8, 8, (6, 1, 1), generator=g))).to(torch.bfloat16)
    x[2] = 0
    ref = RefOps()
    amax = ref.absmax_rows(x, 6)
    amax[4] *= 0.5                                     # half the true max: saturation at 448
    rq, rs = ref.quantize_e4m3_rows(x, amax)
    q, s = ep.quantize_rows(x.double().numpy(), amax.double().numpy())
    assert np.array_equal(s, rs.numpy())
    assert np.array_equal(q, rq.view(torch.uint8).numpy())


def test_block_transpose_by_hand():
    b = np.arange(12, dtype=np.uint8)                   # R=2 rows of C=3 blocks of 2 bytes
    out = ep.block_transpose(b, 2, 3)
    assert list(out) == [0, 1, 6, 7, 2, 3, 8, 9, 4, 5, 10, 11]
    assert np.array_equal(ep.block_transpose(out, 3, 2), b)


def test_block_transpose_and_absmax_agree_with_the_torch_reference_ops():
    g = torch.Generator().manual_seed(11)
    x = torch.randn((2, 6, 40, 16), generator=g).to(torch.bfloat16)
    ref = RefOps()
    got = ep.block_transpose(x.view(torch.int16).numpy(), 2, 3)
    want = ref.block_transpose(x, 2, 3).contiguous().view(torch.uint8).numpy().reshape(-1)
    assert np.array_equal(got, want)
    assert np.array_equal(ep.absmax_rows(x.double().numpy(), 12), ref.absmax_rows(x, 12).double().numpy())
