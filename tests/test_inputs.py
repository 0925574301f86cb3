"""The seeded input generators: bf16 rounding, determinism, and the workload recipe."""
import numpy as np
import torch

from hadamard_bit_quant_hbl_b200 import inputs


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(7)
    a = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        np.array([0.0, -0.0, 1.0, 65504.0, 1e-30, -3.3895314e38], np.float32)])
    want = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(inputs.f32_to_bf16_bits(a), want)
    np.testing.assert_array_equal(inputs.bf16_bits_to_f32(want),
                                  torch.from_numpy(want.view(np.int16)).view(torch.bfloat16).float().numpy())


def test_rows_do_not_depend_on_row_count_and_are_seeded():
    spec = inputs.WORKLOADS["wo_1p3b_a4"]
    a = inputs.activations(spec.with_m(5))
    b = inputs.activations(spec.with_m(9))
    np.testing.assert_array_equal(a, b[:5])
    np.testing.assert_array_equal(a, inputs.activations(spec.with_m(5)))
    w1 = inputs.weights(spec)
    assert w1.shape == (spec.K, spec.N) and w1.dtype == np.float32
    assert abs(float(w1.std()) - 0.02) < 1e-3


def test_recipe_shapes_and_statistics():
    spec = inputs.WORKLOADS["wo_1p3b_a4"].with_m(64)
    x = inputs.bf16_bits_to_f32(inputs.activations(spec))
    assert x.shape == (64, 2048)
    zero = np.mean(x == 0)
    assert 0.27 < zero < 0.33  # 30% exact zeros
    col_scale = np.abs(x).mean(axis=0)
    big = np.sort(col_scale)[-spec.n_outlier:]
    assert spec.n_outlier == 20 and big.min() > 10 * np.median(col_scale)
    single = inputs.WORKLOADS["single_a8_16x256"]
    assert single.n_outlier == 4 and single.abits == 8
    assert inputs.WORKLOADS["wdown_nonpow2_a4"].K == 43 * 256
