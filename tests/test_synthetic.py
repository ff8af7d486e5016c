"""The seeded input generator: determinism, distribution, and bf16 rounding
against torch's own float32 -> bfloat16 conversion."""

import numpy as np
import torch

from synthetic import (attention_inputs, bf16_bits_to_f32, f32_to_bf16_bits, normal,
                       sign_vector, splitmix64, uniform01, WORKLOADS)


def test_splitmix64_is_counter_based_and_deterministic():
    a = splitmix64(42, np.arange(10, dtype=np.uint64))
    b = splitmix64(42, np.arange(5, 10, dtype=np.uint64))
    np.testing.assert_array_equal(a[5:], b)
    assert len(set(a.tolist())) == 10
    assert not np.array_equal(a, splitmix64(43, np.arange(10, dtype=np.uint64)))


def test_splitmix64_known_answers():
    """Known-answer values of SplitMix64 (Steele, Lea and Flood 2014; the
    reference C implementation's next()): the first outputs with the state
    seeded to 1234567, and the first output from state 0 (0xE220A8397B1DCDAF).
    Output i of the counter form is output i of the sequential generator."""
    got = splitmix64(1234567, np.arange(5, dtype=np.uint64)).tolist()
    assert got == [6457827717110365317, 3203168211198807973, 9817491932198370423, 4593380528125082431,
                   16408922859458223821]
    assert int(splitmix64(0, np.zeros(1, dtype=np.uint64))[0]) == 0xE220A8397B1DCDAF


def test_normal_moments():
    x = normal(7, 0, 1 << 20)
    assert abs(x.mean()) < 5e-3
    assert abs(x.std() - 1) < 5e-3
    assert abs(np.mean(x ** 4) - 3) < 0.05
    u = uniform01(7, 4, 1 << 18)
    assert 0 <= u.min() and u.max() < 1 and abs(u.mean() - 0.5) < 5e-3


def test_bf16_rounding_matches_torch():
    x = np.concatenate([normal(1, 0, 100000).astype(np.float32),
                        np.array([1.00390625, 1.01171875, -3.0e-5, 65504.0], np.float32)])
    ours = f32_to_bf16_bits(x)
    theirs = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, theirs)
    np.testing.assert_array_equal(bf16_bits_to_f32(ours),
                                  torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_inputs_shapes_and_outliers():
    x = attention_inputs(2, 4, 2, 64, 16, seed=5, outlier_rate=0.05)
    assert x["q"].shape == (2, 4, 64, 16) and x["k"].shape == (2, 2, 64, 16)
    assert x["do"].shape == (2, 4, 64, 16) and x["q"].dtype == np.uint16
    big = np.abs(bf16_bits_to_f32(x["q"])) > 6
    assert 0.01 < big.mean() < 0.1
    y = attention_inputs(2, 4, 2, 64, 16, seed=5, outlier_rate=0.05)
    for n in x:
        np.testing.assert_array_equal(x[n], y[n])


def test_sign_vector():
    s = sign_vector(3, 128)
    assert set(np.unique(s)) == {-1.0, 1.0}
    np.testing.assert_array_equal(s, sign_vector(3, 128))
    assert not np.array_equal(s, sign_vector(4, 128))


def test_workloads_flop_counts():
    w = WORKLOADS["long128"]
    assert w.fwd_flops(True) == 4 * 2 * 16 * 8192 ** 2 * 128 / 2
    assert w.bwd_flops(True) == 2.5 * w.fwd_flops(True)
    assert [w.seed for w in WORKLOADS.values()] == [42, 43, 44, 45, 46, 47]
