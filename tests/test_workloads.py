"""The seeded workloads: shapes and parameter counts the pages print."""
import numpy as np
import pytest
import torch

from golden.reader import load
from mixture_experts_layer_50_b200 import workloads as W


def _expert_params(s):
    return s.gu_rows * s.d + s.d * s.F


def test_v41flash_expert_and_layer_counts():
    g = load("param_counts.txt")
    s = W.PRESETS["v41flash-n64"]
    assert (s.d, s.F) == (int(g["v41_d"]), int(g["v41_F"]))
    assert s.G == int(g["v41_experts_per_layer"])
    per = _expert_params(s)
    assert per == 3 * 5120 * 2304 == 35389440
    total = per * s.G * int(g["v41_layers"])
    assert round(total / 1e9, 1) == float(g["v41_moe_params_G"])
    assert round(100 * total / 552e9, 1) == float(g["v41_share_of_552G_percent"])
    active = s.k + s.n_shared
    assert round(100 * active / s.G, 1) == float(g["v41_active_over_total_percent"])
    assert s.clamp == 10.0 and s.n_bias_sets == 2 and s.k == 6


def test_dsv3_expert_count():
    g = load("param_counts.txt")
    s = W.PRESETS["dsv3-n64"]
    assert _expert_params(s) == int(g["dsv3_expert_params"])
    assert round(58 * s.G * _expert_params(s) / 1e9) == int(g["dsv3_moe_layers_params_B"])


def test_toy_counts_and_draws():
    g = load("param_counts.txt")
    s = W.PRESETS["toy"]
    per = _expert_params(s)
    assert s.E * per == int(g["toy_expert_params_total"])
    assert s.k * per == int(g["toy_expert_params_used"])
    t = W.make_inputs(s)
    assert t["x"].shape == (1000, 64) and t["x"].dtype == torch.float32
    assert t["W_gu"].shape == (8, 256, 64) and t["W_down"].shape == (8, 64, 256)
    assert t["W_g"].shape == (8, 64)
    # the page's draw order: W1 first, so the first stored W1 value is the first draw
    first = np.random.default_rng(42).normal(0, 0.1, (8, 64, 256))[0, 0, 0]
    assert t["W_gu"][0, 0, 0].item() == pytest.approx(first, rel=1e-6)


def test_trace_model_ratio():
    g = load("param_counts.txt")
    total = (64 + 1) * 0.4
    active = (2 + 1) * 0.4
    assert total == pytest.approx(float(g["trace_total_Md"]))
    assert active == pytest.approx(float(g["trace_active_Md"]))
    assert int(total / active) == 21


def test_small_bf16_draws_and_distributions():
    s = W.PRESETS["v41flash-n64"].replace(d=256, F=128, E=16, k=4, N=4000)
    t = W.make_inputs(s)
    assert t["x"].dtype == torch.bfloat16 and t["W_gu"].shape == (17, 256, 256)
    assert t["W_down"].shape == (17, 256, 128)
    assert t["bias"].shape == (2, 16) and float(t["bias"].abs().max()) <= 0.1
    frac = float(t["modality"].float().mean())
    assert 0.26 < frac < 0.34
    assert abs(float(t["W_gu"].float().std()) - 0.02) < 1e-3
    # same seed, same draw
    t2 = W.make_inputs(s)
    assert torch.equal(t["x"], t2["x"]) and torch.equal(t["bias"], t2["bias"])


def test_zipf_offsets():
    off = W.zipf_logit_offsets(64)
    assert off[0] == 0.0
    np.testing.assert_allclose(off[1], -2.2 * np.log(2.0), rtol=1e-6)
    assert np.all(np.diff(off) < 0)


def test_capacity_presets():
    from fractions import Fraction
    assert W.PRESETS["capacity-cf1"].capacity_factor == 1
    assert W.PRESETS["capacity-cf1.25"].capacity_factor == Fraction(5, 4)
    assert W.PRESETS["capacity-cfinf"].capacity_factor is None
    sw = W.PRESETS["switch-cf1"]
    assert sw.k == 1 and sw.renorm == 0
