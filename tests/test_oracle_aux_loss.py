"""Pins of the oracle's auxiliary load-balancing loss (Transformer Engine
"Mixture of Experts", Load balancing: fused_compute_score_for_moe_aux_loss and
fused_moe_aux_loss). The page names the inputs but prints no formula; the
oracle's reading is loss = coeff * E / (k T^2) * sum_e (sum_t s[t,e]) * c_e.
These tests pin that reading by hand-worked cases and closed forms, and its
gradient by central differences."""
import numpy as np
import pytest

import oracle


def test_hand_worked_cases():
    # softmax: both rows [0, ln 3] give scores [1/4, 3/4], so sum_t s = [1/2, 3/2];
    # counts [0, 2] (k=1, T=2): loss = 0.01 * 2 / (1 * 4) * (1/2 * 0 + 3/2 * 2) = 0.015
    l = np.array([[0.0, np.log(3.0)], [0.0, np.log(3.0)]], np.float32)
    assert oracle.aux_loss(l, [0, 2], 1, 0.01) == pytest.approx(0.015, rel=1e-7)
    # the same counts on the other expert: 0.005 * (1/2 * 2) = 0.005
    assert oracle.aux_loss(l, [2, 0], 1, 0.01) == pytest.approx(0.005, rel=1e-7)
    # sigmoid, one token [0, ln 3]: scores [1/2, 3/4]; counts [1, 0] (k=1, T=1):
    # loss = 0.1 * 2 / 1 * (1/2 * 1) = 0.1
    l1 = np.array([[0.0, np.log(3.0)]], np.float32)
    assert oracle.aux_loss(l1, [1, 0], 1, 0.1, score=1) == pytest.approx(0.1, rel=1e-7)
    assert oracle.aux_loss(l1, [0, 1], 1, 0.1, score=1) == pytest.approx(0.15, rel=1e-7)


def test_uniform_scores_give_coeff_whatever_the_counts():
    # equal logits: every score is 1/E, sum_t s_e = T/E, and sum_e c_e = T k,
    # so loss = coeff * E / (k T^2) * (T / E) * T k = coeff
    rng = np.random.default_rng(1)
    T, E, k = 37, 12, 3
    l = np.zeros((T, E), np.float32)
    for _ in range(4):
        counts = np.bincount(rng.integers(0, E, T * k), minlength=E).astype(np.int32)
        assert oracle.aux_loss(l, counts, k, 0.02) == pytest.approx(0.02, rel=1e-12)


def test_concentrated_scores():
    # one expert 60 above the rest: its softmax score is 1 within 1e-25
    T, E, k = 10, 8, 2
    l = np.zeros((T, E), np.float32)
    l[:, 3] = 60.0
    on_three = np.zeros(E, np.int32)
    on_three[3] = T * k
    # all assignments on it too: coeff * E / (k T^2) * T * T k = coeff * E
    assert oracle.aux_loss(l, on_three, k, 0.5) == pytest.approx(0.5 * E, rel=1e-12)
    # balanced counts: coeff * E / (k T^2) * T * (T k / E) = coeff
    balanced = np.full(E, T * k // E, np.int32)
    balanced[: T * k - balanced.sum()] += 1
    expect = 0.5 * E / (k * T * T) * T * balanced[3]
    assert oracle.aux_loss(l, balanced, k, 0.5) == pytest.approx(expect, rel=1e-12)


def test_linear_in_coeff_and_relabelling_invariant():
    rng = np.random.default_rng(2)
    T, E, k = 19, 7, 2
    l = rng.standard_normal((T, E)).astype(np.float32)
    counts = rng.integers(0, 9, E).astype(np.int32)
    for score in (0, 1):
        a = oracle.aux_loss(l, counts, k, 0.01, score)
        assert oracle.aux_loss(l, counts, k, 0.03, score) == pytest.approx(3 * a, rel=1e-12)
        perm = rng.permutation(E)
        assert oracle.aux_loss(l[:, perm], counts[perm], k, 0.01, score) == pytest.approx(a, rel=1e-12)
        g = oracle.aux_loss_backward(l, counts, k, 0.01, score)
        gp = oracle.aux_loss_backward(l[:, perm], counts[perm], k, 0.01, score)
        assert np.allclose(gp, g[:, perm], rtol=1e-12, atol=1e-18)
        assert np.allclose(oracle.aux_loss_backward(l, counts, k, 0.01, score, grad_loss=-2.5), -2.5 * g,
                           rtol=1e-12, atol=1e-18)


@pytest.mark.parametrize("score", [0, 1])
def test_backward_matches_central_differences(score):
    rng = np.random.default_rng(3 + score)
    T, E, k = 6, 9, 3
    l = rng.uniform(-3, 3, (T, E)).astype(np.float32)
    counts = rng.integers(0, 7, E).astype(np.int32)
    coeff = 0.7
    g = oracle.aux_loss_backward(l, counts, k, coeff, score)
    h = np.float32(2.0 ** -12)   # exact in fp32 for |l| < 2^11
    scale = np.abs(g).max()
    for _ in range(20):
        t, e = int(rng.integers(T)), int(rng.integers(E))
        lp, lm = l.copy(), l.copy()
        lp[t, e] += h
        lm[t, e] -= h
        fd = (oracle.aux_loss(lp, counts, k, coeff, score) - oracle.aux_loss(lm, counts, k, coeff, score)) / (
            float(lp[t, e]) - float(lm[t, e]))
        assert abs(fd - g[t, e]) <= 1e-6 * scale, (t, e, fd, g[t, e])


def test_softmax_gradient_rows_sum_to_zero():
    # sum_i s_i (G_i - sum_e s_e G_e) = 0 for every token
    rng = np.random.default_rng(5)
    l = rng.standard_normal((13, 16)).astype(np.float32)
    counts = rng.integers(0, 20, 16).astype(np.int32)
    g = oracle.aux_loss_backward(l, counts, 4, 1.0, 0)
    assert np.abs(g.sum(axis=1)).max() <= 1e-15 * max(1.0, np.abs(g).max() * 16)
