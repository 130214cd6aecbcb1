"""Pins of the MXFP4 quantiser oracle (CPU only): exhaustive nearest-value checks
against the E2M1 grid, ties, saturation, round trips of representable blocks,
the shared-exponent rule at powers of two, signs, packing order and the error
bound of the format."""
import numpy as np
import pytest

from oracle import mxfp4

GRID = np.array(mxfp4.E2M1_MAGNITUDES)


def test_rounding_is_a_nearest_grid_value_brute_force():
    y = np.linspace(0, 6, 24001)
    codes = mxfp4.e2m1_round(y)
    dist = np.abs(y[:, None] - GRID[None, :])
    best = dist.min(axis=1)
    assert np.all(np.abs(GRID[codes] - y) <= best + 1e-15)


@pytest.mark.parametrize("y,code", [(0.25, 0), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6), (5.0, 6),
                                    (0.2499, 0), (0.2501, 1), (4.999, 6), (5.001, 7)])
def test_ties_go_to_the_even_mantissa(y, code):
    assert int(mxfp4.e2m1_round(np.array([y]))[0]) == code


def test_saturates_at_six():
    assert list(mxfp4.e2m1_round(np.array([6.0, 6.5, 7.99, 100.0]))) == [7, 7, 7, 7]


def test_round_trip_of_representable_blocks():
    rng = np.random.default_rng(0)
    rows, K = 6, 128
    codes = rng.integers(0, 16, size=(rows, K)).astype(np.uint8)
    codes[:, ::32] = 7                                       # every block holds a +-6 (fixes the exponent)
    s = rng.integers(-20, 20, size=(rows, K // 32))
    scales = (s + 127).astype(np.uint8)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    x = mxfp4.dequantize(packed, scales)
    p2, s2 = mxfp4.quantize(x)
    np.testing.assert_array_equal(s2, scales)
    # -0 and +0 decode alike; compare values, then the non-zero codes bit for bit
    np.testing.assert_array_equal(mxfp4.dequantize(p2, s2), x)
    nz = (codes & 7) != 0
    full = np.empty_like(codes)
    full[:, 0::2], full[:, 1::2] = p2 & 0xF, p2 >> 4
    np.testing.assert_array_equal(full[nz], codes[nz])


def test_shared_exponent_at_powers_of_two():
    for k in (-10, 0, 1, 5, 30):
        assert int(mxfp4.shared_exponent(np.array([2.0 ** k]))[0]) == k - 2
        assert int(mxfp4.shared_exponent(np.array([2.0 ** k * (1 - 1e-9)]))[0]) == k - 3
    assert int(mxfp4.shared_exponent(np.array([0.0]))[0]) == -127
    assert int(mxfp4.shared_exponent(np.array([2.0 ** 200]))[0]) == 127
    assert int(mxfp4.shared_exponent(np.array([2.0 ** -200]))[0]) == -127


def test_block_max_lands_in_four_to_six():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((50, 64)) * np.exp2(rng.integers(-8, 8, size=(50, 1)))
    packed, scales = mxfp4.quantize(x)
    deq = mxfp4.dequantize(packed, scales)
    s = np.repeat(np.exp2(scales.astype(np.int64) - 127.0), 32, axis=1)
    amax = np.abs(deq / s).reshape(50, 2, 32).max(axis=2)
    assert np.all((amax == 4.0) | (amax == 6.0))


def test_error_bound_of_the_format():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((40, 256)) * 3.0
    packed, scales = mxfp4.quantize(x)
    deq = mxfp4.dequantize(packed, scales)
    unit = np.repeat(np.exp2(scales.astype(np.int64) - 127.0), 32, axis=1)
    y = np.abs(x) / unit
    half_step = np.where(y < 2, 0.25, np.where(y < 4, 0.5, 1.0))
    bound = np.where(y > 6, y - 6, half_step) * unit
    assert np.all(np.abs(deq - x) <= bound + 1e-12)


def test_signs_and_negative_zero():
    x = np.zeros((1, 32))
    x[0, 0], x[0, 1], x[0, 2] = 6.0, -6.0, -0.01           # s = 0
    packed, scales = mxfp4.quantize(x)
    assert scales[0, 0] == 127
    assert packed[0, 0] == (0x7 | (0xF << 4))               # +6 low nibble, -6 high nibble
    assert packed[0, 1] & 0xF == 0x8                         # -0.01 rounds to -0
    x[0, 1] = 0.0
    packed, _ = mxfp4.quantize(-np.zeros((1, 32)))
    assert np.all(packed == 0x88)                            # -0.0 keeps its sign
    packed, scales = mxfp4.quantize(np.zeros((1, 32)))
    assert np.all(packed == 0) and scales[0, 0] == 0


def test_packing_order_first_element_low_nibble():
    x = np.zeros((1, 32))
    x[0, 0], x[0, 1] = 1.0, 6.0                              # amax 6 -> s = 0; codes 2 and 7
    packed, _ = mxfp4.quantize(x)
    assert packed[0, 0] == 0x72


def test_rejects_ragged_rows():
    with pytest.raises(ValueError):
        mxfp4.quantize(np.zeros((2, 48)))
