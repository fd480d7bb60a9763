"""Pins of the oracle's expert-bias update (torchtitan MoE._update_expert_bias,
auxiliary-loss-free load balancing) from properties of the definition."""
import numpy as np

import oracle


def test_balanced_counts_leave_the_bias_alone():
    bias = np.linspace(-1, 1, 16).astype(np.float32)
    assert np.array_equal(oracle.expert_bias_update(np.full(16, 37), bias, 1e-3), bias)


def test_overloaded_experts_go_down_and_the_update_sums_to_zero():
    counts = np.array([10, 0, 5, 5, 30, 0, 5, 5], np.int32)     # mean 7.5: 2 above, 6 below
    new = oracle.expert_bias_update(counts, np.zeros(8, np.float32), 0.01).astype(np.float64)
    assert np.all(new[counts > 7.5] < 0) and np.all(new[counts < 7.5] > 0)
    assert abs(new.sum()) < 1e-7
    # closed form: delta = -0.01 above, +0.01 below; its mean is 0.01 * (6 - 2) / 8
    assert np.allclose(new, np.where(counts > 7.5, -0.01, 0.01) - 0.005, rtol=1e-6, atol=0)


def test_ties_with_the_mean_get_only_the_centring_term():
    counts = np.array([3, 3, 6, 0], np.int32)                   # mean 3: two ties
    new = oracle.expert_bias_update(counts, np.zeros(4, np.float32), 1.0).astype(np.float64)
    assert np.allclose(new, [0, 0, -1, 1], atol=1e-7)           # delta [0, 0, -1, 1], mean 0
    counts = np.array([4, 4, 4, 0], np.int32)                   # mean 3: three above, one below
    new = oracle.expert_bias_update(counts, np.zeros(4, np.float32), 1.0).astype(np.float64)
    assert np.allclose(new, np.array([-1, -1, -1, 1]) + 0.5, atol=1e-7)   # mean of delta is -0.5
    # the update adds to the bias it is given
    base = np.array([0.25, -0.5, 1.0, 2.0], np.float32)
    assert np.allclose(oracle.expert_bias_update(counts, base, 1.0), base + new, atol=1e-6)
