"""The seeded input generator follows its stated recipe (no step of the method is involved).

- Rounding to bf16 is torch's round-to-nearest-even, and widening back is exact.
- Activation columns have std sigma_i = exp(N(0, s)). s is 1 with round(1% of C) distinct
  outlier columns scaled by 20 (dense, activation-aware and MoE layers), and 1.5 with none
  for the WMSE layer.
- Weights are N(0, 1/C), or N(0, 0.02^2) fp32 for the tiny layer.
- MoE routing gives each token top_k distinct experts, as CSR sorted by expert with tokens
  ascending.
- Everything is a function of the seed.
"""
import numpy as np
import torch

from scale_calibration_lh_b200 import synth


def test_bf16_rounding_is_round_to_nearest_even_and_widening_is_exact():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.normal(0, 1, 100000) * np.exp(rng.normal(0, 5, 100000)),
                        [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 0.0, -0.0, 3e38, 1e-40]]).astype(np.float32)
    bits = synth.f32_to_bf16_bits(v)
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(bits, want)
    back = synth.bf16_bits_to_f32(bits)
    np.testing.assert_array_equal(back, torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy())


def test_column_stds_and_outliers_follow_the_recipe():
    # Outlier columns: round(1% of 4096) = 41, round(1% of 2560) = 26; none for WMSE.
    for name, log_std, n_out in (("dense", 1.0, 41), ("act", 1.0, 41), ("moe", 1.0, 26), ("wmse", 1.5, 0)):
        cin = 2560 if name == "moe" else 4096
        sigma = synth.make_layer(name, 0, tokens=1, cin=cin, rows=1, groups=1).meta["sigma"]
        base = np.exp(synth._rng(0, "sigma").normal(0.0, log_std, size=cin)).astype(np.float32)
        scaled = sigma == base * np.float32(20.0)  # the fp32 product the generator forms
        assert int(scaled.sum()) == n_out and np.array_equal(sigma[~scaled], base[~scaled]), name
        assert abs(np.std(np.log(base)) - log_std) < 0.05 * log_std and abs(np.mean(np.log(base))) < 0.06


def test_layers_have_the_stated_column_and_weight_scales():
    layer = synth.make_layer("dense", 0, tokens=4096, cin=64, rows=512)
    x = layer.x_f32().astype(np.float64)
    sigma = layer.meta["sigma"].astype(np.float64)
    np.testing.assert_allclose(x.std(axis=0) / sigma, 1.0, atol=0.06)
    assert abs(layer.w_f32().std() * np.sqrt(64) - 1.0) < 0.02
    assert layer.dtype == "bf16" and layer.mode == "full" and layer.group_offsets is None
    tiny = synth.make_layer("tiny", 0)
    assert tiny.dtype == "f32" and tiny.x.shape == (256, 64) and tiny.w.shape == (1, 32, 64)
    assert abs(tiny.w.std() - 0.02) < 0.002 and abs(tiny.x.std() - 1.0) < 0.02


def test_moe_routing_is_top_k_distinct_experts_in_sorted_csr():
    offsets, ids = synth.moe_routing(3000, 64, 10, 5)
    assert offsets[0] == 0 and offsets[-1] == len(ids) == 3000 * 10 and np.all(np.diff(offsets) >= 0)
    seen = np.zeros((3000, 64), np.int64)
    for e in range(64):
        rows = ids[offsets[e]:offsets[e + 1]]
        assert np.all(np.diff(rows) > 0)  # ascending, so no token twice in one expert
        seen[rows, e] += 1
    assert np.all(seen.sum(axis=1) == 10) and seen.max() == 1
    counts = np.diff(offsets)
    assert abs(counts.mean() - 3000 * 10 / 64) < 1e-9 and counts.min() > 0.5 * counts.mean()


def test_inputs_are_a_function_of_the_seed():
    a = synth.make_layer("moe", 3, tokens=64, cin=32, rows=8, groups=6, top_k=2)
    b = synth.make_layer("moe", 3, tokens=64, cin=32, rows=8, groups=6, top_k=2)
    c = synth.make_layer("moe", 4, tokens=64, cin=32, rows=8, groups=6, top_k=2)
    for f in ("x", "w", "group_offsets", "token_ids"):
        np.testing.assert_array_equal(getattr(a, f), getattr(b, f))
    assert not np.array_equal(a.x, c.x) and not np.array_equal(a.w, c.w)
