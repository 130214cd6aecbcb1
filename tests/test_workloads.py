"""Host-side checks of the seeded input generator (no GPU)."""
import math

import numpy as np
import pytest
import torch

from attention_dit_attn_b200 import workloads as wl


def test_five_workloads_have_the_stated_shapes():
    got = {n: (w.B, w.H, w.L, w.D, w.dtype) for n, w in wl.WORKLOADS.items()}
    assert got == {
        "tiny_256": (1, 2, 256, 64, "bf16"),
        "flux_1024x768": (1, 24, 3584, 128, "bf16"),
        "flux_2048_cfg": (2, 24, 16896, 128, "bf16"),
        "sd35_1024_fp8": (2, 38, 4250, 64, "e4m3"),
        "wan_720p_81f": (1, 40, 75600, 128, "bf16"),
    }
    assert wl.ORDER == list(wl.WORKLOADS)
    assert wl.WORKLOADS["flux_2048_cfg"].flops == pytest.approx(7.016e12, rel=1e-3)
    assert wl.WORKLOADS["wan_720p_81f"].flops == pytest.approx(1.171e14, rel=1e-3)
    assert wl.WORKLOADS["tiny_256"].scale == 0.125


def test_generation_is_deterministic_per_seed():
    a = wl.generate(1, 2, 40, 64, "bf16", seed=3)
    b = wl.generate(1, 2, 40, 64, "bf16", seed=3)
    c = wl.generate(1, 2, 40, 64, "bf16", seed=4)
    assert torch.equal(a.q, b.q) and torch.equal(a.v, b.v)
    assert not torch.equal(a.q, c.q)


def test_text_rows_scale_q_and_k_only():
    base = wl.generate(1, 1, 32, 64, "bf16", seed=8)
    txt = wl.generate(1, 1, 32, 64, "bf16", seed=8, text_rows=8, text_scale=2.0)
    assert torch.equal(txt.q[:, :, :8].float(), 2 * base.q[:, :, :8].float())
    assert torch.equal(txt.k[:, :, :8].float(), 2 * base.k[:, :, :8].float())
    assert torch.equal(txt.q[:, :, 8:], base.q[:, :, 8:])
    assert torch.equal(txt.v, base.v)


def test_lowrank_component_peaks_the_logits():
    plain = wl.generate(1, 2, 512, 128, "bf16", seed=9)
    peak = wl.generate(1, 2, 512, 128, "bf16", seed=9, lowrank=8)
    def logit_std(x):
        s = (x.q.float() @ x.k.float().transpose(-1, -2)) / math.sqrt(128)
        return s.std().item()
    assert logit_std(plain) < 1.5 < 3.0 < logit_std(peak)
    assert torch.equal(plain.v, peak.v)


def test_e4m3_quantisation_is_per_head_absmax():
    x = wl.generate(2, 3, 64, 64, "e4m3", seed=10)
    assert x.q.dtype == torch.float8_e4m3fn and x.q_scale.shape == (2, 3)
    deq = x.q.to(torch.float32) * x.q_scale[:, :, None, None]
    amax = deq.abs().reshape(2, 3, -1).amax(-1)
    # The absmax element maps to +-448 exactly, so it dequantises to amax.
    codes = x.q.to(torch.float32).abs().reshape(2, 3, -1).amax(-1)
    assert torch.all(codes == 448.0)
    assert torch.allclose(amax, x.q_scale * 448.0)


def test_sample_rows_include_ends_and_are_distinct():
    r = wl.sample_rows(2, 3, 1000, 512, seed=1003)
    assert r.shape == (6, 512)
    for row in r:
        assert row[0] == 0 and row[-1] == 999
        assert len(np.unique(row)) == 512 and np.all(np.diff(row) > 0)
    assert not np.array_equal(r[0], r[1])
    full = wl.sample_rows(1, 1, 10, 512, seed=0)
    assert np.array_equal(full[0], np.arange(10))
