"""The seeded synthetic inputs have the shapes and statistics the input recipe
states: the attention weight's outlier columns (1% of the inputs, x20), the
standard deviations of W, x and the bias, bf16 rounding to nearest even, and
determinism (same key, same bytes; different keys, different streams)."""
import numpy as np
import torch

import wlq_inputs as wi


def test_attention_weight_outlier_columns():
    W = wi.weight(1, 2, 512, 4096, outlier_frac=0.01)
    col_std = W.std(axis=0)
    big = col_std > 0.2
    assert int(big.sum()) == round(0.01 * 4096) == 41
    assert abs(float(np.median(col_std[~big])) - 0.02) < 0.002
    assert abs(float(np.median(col_std[big])) - 0.4) < 0.05
    # every row's absmax sits in an outlier column with overwhelming probability
    assert np.mean(big[np.argmax(np.abs(W), axis=1)]) > 0.99


def test_standard_deviations():
    x = wi.bf16_to_f32(wi.activations(1, 1, 256, 4096))
    b = wi.bf16_to_f32(wi.bias(1, 3, 4096))
    assert abs(float(x.std()) - 1.0) < 0.01 and abs(float(x.mean())) < 0.01
    assert abs(float(b.std()) - 0.01) < 0.001


def test_bf16_bits_round_to_nearest_even_like_torch():
    g = np.random.default_rng(0)
    a = (g.standard_normal(100000) * np.exp(g.uniform(-30, 30, 100000))).astype(np.float32)
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(wi.bf16_bits(a), ref)


def test_generators_are_deterministic_and_keyed():
    a1 = wi.weight(4, 2, 64, 128)
    a2 = wi.weight(4, 2, 64, 128)
    b = wi.weight(4, 3, 64, 128)
    assert np.array_equal(a1, a2)
    assert not np.array_equal(a1, b)
    x16 = wi.activations(1, 1, 16, 256)
    x17 = wi.activations(1, 1, 17, 256)
    assert not np.array_equal(x16, x17[:16])  # the token count is part of the key


def test_workload_shapes():
    d = wi.attn_w8(16)
    assert d["W"].shape == (4096, 4096) and d["x"].shape == (16, 4096) and d["b"].shape == (4096,)
    assert (d["bits"], d["group"]) == (8, 0)
    up, down = wi.mlp_w4(16, "up"), wi.mlp_w4(16, "down")
    assert up["W"].shape == (16384, 4096) and down["W"].shape == (4096, 16384)
    assert (up["bits"], up["group"]) == (4, 64)
    lr = wi.svdq_w4_lr(8)
    assert lr["L1"].shape == (4096, 32) and lr["L2"].shape == (32, 4096)
