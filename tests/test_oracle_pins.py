"""Pins for the fp64 oracle: facts that hold independently of its code.

Each test fixes the oracle to something other than itself: the FP8/bf16
format definitions, closed forms of softmax attention, its invariants, a
brute-force loop on tiny inputs and torch's own scaled_dot_product_attention
in fp64.  The pages print no attention values, so there is no page-printed
worked example; tests/golden holds a hand-derived one.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from attention_dit_attn_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _sdpa64(q, k, v, scale):
    """torch's SDPA in fp64 on the CPU (a library routine, independent of the oracle)."""
    qt, kt, vt = (torch.from_numpy(np.ascontiguousarray(x)) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)
    lse = torch.logsumexp(scale * (qt @ kt.transpose(-1, -2)), dim=-1)
    return o.numpy(), lse.numpy()


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ---------------------------------------------------------------- decoders

def test_e4m3_decoder_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert set(np.flatnonzero(nan)) == {0x7F, 0xFF}
    assert np.array_equal(ours[~nan], ref[~nan])


def test_e4m3_decoder_format_landmarks():
    # OCP FP8 E4M3: max normal S.1111.110 = 448, min normal 2^-6, min subnormal 2^-9.
    d = lambda c: oracle.e4m3_to_f64(np.array([c], dtype=np.uint8))[0]
    assert d(0x7E) == 448.0 and d(0xFE) == -448.0
    assert d(0x08) == 2.0 ** -6
    assert d(0x01) == 2.0 ** -9
    assert d(0x07) == 7 * 2.0 ** -9
    assert d(0x38) == 1.0 and d(0x00) == 0.0
    assert math.copysign(1.0, d(0x80)) == -1.0
    assert oracle.e4m3_to_f64(np.array([0x38], dtype=np.uint8), scale=0.375)[0] == 0.375


def test_bf16_decoder_all_patterns_match_torch():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.bf16_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


# ---------------------------------------------------------------- closed forms

def test_golden_hand_derived_example():
    with open(os.path.join(GOLDEN, "attention_ratios_123.json")) as f:
        g = json.load(f)
    L, D = g["L"], g["D"]
    q = np.array(g["q"], dtype=np.float64).reshape(1, 1, L, D)
    k = np.array([[math.log(j + 1), 0.0] for j in range(L)]).reshape(1, 1, L, D)
    v = np.array(g["v"], dtype=np.float64).reshape(1, 1, L, D)
    o, lse = oracle.attention(q, k, v, g["scale"], dtype=oracle.F64)
    assert np.allclose(o[0, 0], np.array(g["o"]), rtol=0, atol=g["tol"])
    want_lse = [math.log(6), math.log(3), math.log(14)]
    assert np.allclose(lse[0, 0], want_lse, rtol=0, atol=g["tol"])


def test_single_key_returns_its_value_and_logit():
    q, k, v = _rand((2, 3, 1, 16), 1), _rand((2, 3, 1, 16), 2), _rand((2, 3, 1, 16), 3)
    o, lse = oracle.attention(q, k, v, 0.25, dtype=oracle.F64)
    assert np.array_equal(o, v)
    s0 = 0.25 * np.einsum("bhld,bhld->bhl", q, k)
    assert np.allclose(lse, s0, rtol=0, atol=1e-14)


def test_two_keys_weight_is_sigmoid_of_logit_gap():
    q, k, v = _rand((1, 2, 2, 8), 4), _rand((1, 2, 2, 8), 5), _rand((1, 2, 2, 8), 6)
    scale = 0.7
    o, lse = oracle.attention(q, k, v, scale, dtype=oracle.F64)
    for h in range(2):
        for i in range(2):
            s0 = scale * q[0, h, i] @ k[0, h, 0]
            s1 = scale * q[0, h, i] @ k[0, h, 1]
            w = 1.0 / (1.0 + math.exp(-(s0 - s1)))
            want = w * v[0, h, 0] + (1 - w) * v[0, h, 1]
            assert np.allclose(o[0, h, i], want, rtol=0, atol=1e-14)
            assert abs(lse[0, h, i] - (max(s0, s1) + math.log1p(math.exp(-abs(s0 - s1))))) < 1e-14


def test_identical_keys_give_mean_value_and_log_count():
    L, D = 37, 16
    q = _rand((1, 1, L, D), 7)
    krow = _rand((D,), 8)
    k = np.broadcast_to(krow, (1, 1, L, D)).copy()
    v = _rand((1, 1, L, D), 9)
    o, lse = oracle.attention(q, k, v, 0.5, dtype=oracle.F64)
    assert np.allclose(o[0, 0], np.broadcast_to(v[0, 0].mean(0), (L, D)), rtol=0, atol=1e-13)
    assert np.allclose(lse[0, 0], 0.5 * q[0, 0] @ krow + math.log(L), rtol=0, atol=1e-13)


def test_zero_scale_gives_mean_value():
    q, k, v = _rand((1, 2, 19, 8), 10), _rand((1, 2, 19, 8), 11), _rand((1, 2, 19, 8), 12)
    o, lse = oracle.attention(q, k, v, 0.0, dtype=oracle.F64)
    assert np.allclose(o, np.broadcast_to(v.mean(2, keepdims=True), o.shape), rtol=0, atol=1e-14)
    assert np.allclose(lse, math.log(19), rtol=0, atol=1e-14)


def test_dominant_key_returns_its_value_row():
    L, D = 64, 32
    q = np.zeros((1, 1, L, D)); q[..., 0] = 1.0
    k = _rand((1, 1, L, D), 13) * 0.1
    k[0, 0, 17, 0] = 60.0                     # logit gap >= 50 at scale 1
    v = _rand((1, 1, L, D), 14)
    o, _ = oracle.attention(q, k, v, 1.0, dtype=oracle.F64)
    assert np.allclose(o[0, 0], np.broadcast_to(v[0, 0, 17], (L, D)), rtol=0, atol=1e-15)


# ---------------------------------------------------------------- invariants

def test_uniform_values_give_that_value_so_rows_sum_to_one():
    L, D = 50, 24
    q, k = _rand((2, 2, L, D), 15) * 3, _rand((2, 2, L, D), 16) * 3
    c = _rand((D,), 17)
    v = np.broadcast_to(c, (2, 2, L, D)).copy()
    o, _ = oracle.attention(q, k, v, 1.0 / math.sqrt(D), dtype=oracle.F64)
    # sum_j p_j c / sum_j p_j: two L-term fp64 sums, relative error <= ~2 L eps.
    tol = 4 * L * np.finfo(np.float64).eps
    assert np.allclose(o, np.broadcast_to(c, o.shape), rtol=tol, atol=tol)


def test_permuting_keys_with_values_leaves_output_unchanged():
    L, D = 41, 16
    q, k, v = _rand((1, 2, L, D), 18), _rand((1, 2, L, D), 19), _rand((1, 2, L, D), 20)
    perm = np.random.default_rng(21).permutation(L)
    o1, l1 = oracle.attention(q, k, v, 0.3, dtype=oracle.F64)
    o2, l2 = oracle.attention(q, k[:, :, perm], v[:, :, perm], 0.3, dtype=oracle.F64)
    assert np.allclose(o1, o2, rtol=0, atol=1e-13)
    assert np.allclose(l1, l2, rtol=0, atol=1e-13)
    # A transposed or mis-paired operand would break this: permute values only.
    o3, _ = oracle.attention(q, k, v[:, :, perm], 0.3, dtype=oracle.F64)
    assert not np.allclose(o1, o3, atol=1e-3)


def test_permuting_queries_permutes_output_rows():
    L, D = 33, 16
    q, k, v = _rand((1, 1, L, D), 22), _rand((1, 1, L, D), 23), _rand((1, 1, L, D), 24)
    perm = np.random.default_rng(25).permutation(L)
    o1, l1 = oracle.attention(q, k, v, 0.25, dtype=oracle.F64)
    o2, l2 = oracle.attention(q[:, :, perm], k, v, 0.25, dtype=oracle.F64)
    assert np.array_equal(o1[:, :, perm], o2)
    assert np.array_equal(l1[:, :, perm], l2)


def test_sampled_rows_equal_full_rows():
    B, H, L, D = 1, 3, 300, 32
    q, k, v = _rand((B, H, L, D), 26), _rand((B, H, L, D), 27), _rand((B, H, L, D), 28)
    rows = wl.sample_rows(B, H, L, 20, seed=99)
    o_full, l_full = oracle.attention(q, k, v, 0.2, dtype=oracle.F64)
    o_s, l_s = oracle.attention(q, k, v, 0.2, dtype=oracle.F64, rows=rows)
    for bh in range(B * H):
        b, h = divmod(bh, H)
        assert np.array_equal(o_full[b, h, rows[bh]], o_s[b, h])
        assert np.array_equal(l_full[b, h, rows[bh]], l_s[b, h])


# ---------------------------------------------------------------- brute force / library

def test_brute_force_loop_tiny():
    """Naive loops, no max subtraction (N(0,1) logits cannot overflow exp here)."""
    B, H, L, D = 1, 2, 12, 5
    q, k, v = _rand((B, H, L, D), 29), _rand((B, H, L, D), 30), _rand((B, H, L, D), 31)
    scale = 0.6
    o, lse = oracle.attention(q, k, v, scale, dtype=oracle.F64)
    for h in range(H):
        for i in range(L):
            w = [math.exp(scale * sum(q[0, h, i, d] * k[0, h, j, d] for d in range(D)))
                 for j in range(L)]
            z = sum(w)
            for d in range(D):
                want = sum(w[j] * v[0, h, j, d] for j in range(L)) / z
                assert abs(o[0, h, i, d] - want) < 1e-13
            assert abs(lse[0, h, i] - math.log(z)) < 1e-13


@pytest.mark.parametrize("B,H,L,D", [(1, 1, 64, 64), (2, 3, 200, 64), (1, 2, 512, 128)])
def test_matches_torch_sdpa_fp64(B, H, L, D):
    q, k, v = _rand((B, H, L, D), L), _rand((B, H, L, D), L + 1), _rand((B, H, L, D), L + 2)
    scale = 1.0 / math.sqrt(D)
    o, lse = oracle.attention(q, k, v, scale, dtype=oracle.F64)
    o_ref, lse_ref = _sdpa64(q, k, v, scale)
    assert np.allclose(o, o_ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(lse, lse_ref, rtol=1e-12, atol=1e-12)


def test_bf16_input_path_matches_sdpa_on_decoded_values():
    inp = wl.generate(1, 2, 160, 64, "bf16", seed=5, text_rows=16, text_scale=2.0)
    o, lse = oracle.attention(wl.as_bits(inp.q), wl.as_bits(inp.k), wl.as_bits(inp.v),
                              0.125, dtype=oracle.BF16)
    o_ref, lse_ref = _sdpa64(*(t.to(torch.float64).numpy() for t in (inp.q, inp.k, inp.v)), 0.125)
    assert np.allclose(o, o_ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(lse, lse_ref, rtol=1e-12, atol=1e-12)


def test_e4m3_input_path_applies_per_head_dequant_scales():
    inp = wl.generate(2, 3, 96, 64, "e4m3", seed=6)
    o, lse = oracle.attention(wl.as_bits(inp.q), wl.as_bits(inp.k), wl.as_bits(inp.v), 0.125,
                              dtype=oracle.E4M3, q_scale=inp.q_scale.numpy(),
                              k_scale=inp.k_scale.numpy(), v_scale=inp.v_scale.numpy())
    deq = [t.to(torch.float64) * s.to(torch.float64)[:, :, None, None]
           for t, s in ((inp.q, inp.q_scale), (inp.k, inp.k_scale), (inp.v, inp.v_scale))]
    o_ref, lse_ref = _sdpa64(*(x.numpy() for x in deq), 0.125)
    assert np.allclose(o, o_ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(lse, lse_ref, rtol=1e-12, atol=1e-12)
    # Scales are per (b, h): swapping two heads' v scales must change the output.
    vs = inp.v_scale.numpy().copy(); vs[0, 0], vs[1, 2] = vs[1, 2], vs[0, 0]
    o_bad, _ = oracle.attention(wl.as_bits(inp.q), wl.as_bits(inp.k), wl.as_bits(inp.v), 0.125,
                                dtype=oracle.E4M3, q_scale=inp.q_scale.numpy(),
                                k_scale=inp.k_scale.numpy(), v_scale=vs)
    assert not np.allclose(o_bad, o_ref, rtol=1e-6)


def test_bad_arguments_are_rejected():
    q = np.zeros((1, 1, 4, 8))
    with pytest.raises(RuntimeError):
        oracle.attention(q, q, q, 1.0, dtype=oracle.F64, rows=np.array([[0, 4]]))
    with pytest.raises(ValueError):
        oracle.attention(q, q[:, :, :3], q, 1.0, dtype=oracle.F64)
