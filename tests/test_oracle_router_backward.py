"""Pins of the oracle's router backward (dL/dlogits from dL/dtopk_prob) that
do not come from the function itself: central differences of the oracle's
forward routing weights (Transformer Engine "Mixture of Experts", Router),
the zero-sum property of softmax gradients, and the sigmoid special case."""
import numpy as np
import pytest

import oracle

MODES = [(0, True), (0, False), (1, False), (1, True)]


def _separated_logits(T, E, seed):
    # distinct logits at least 0.05 apart inside a row, so a small step never
    # changes which experts are chosen
    rng = np.random.default_rng(seed)
    rows = []
    for _ in range(T):
        v = np.arange(E, dtype=np.float64) * 0.05 + rng.uniform(0, 0.02, E)
        rows.append(rng.permutation(v) - 0.05 * E / 2)
    return np.array(rows, np.float32) * 2.0


@pytest.mark.parametrize("score,renorm", MODES)
@pytest.mark.parametrize("scaling", [1.0, 2.5])
def test_router_backward_matches_central_differences(score, renorm, scaling):
    T, E, k = 6, 12, 4
    logits = _separated_logits(T, E, seed=score * 10 + int(renorm))
    r = oracle.router_topk(logits, k, score, renorm, scaling)
    rng = np.random.default_rng(3)
    dprob = rng.standard_normal((T, k)).astype(np.float32)
    dl = oracle.router_backward(logits, r["topk_idx"], dprob, score, renorm, scaling)
    h = 1e-3
    for t in range(T):
        for e in range(E):
            lp = logits.copy(); lp[t, e] += h
            lm = logits.copy(); lm[t, e] -= h
            rp = oracle.router_topk(lp, k, score, renorm, scaling)
            rm = oracle.router_topk(lm, k, score, renorm, scaling)
            assert np.array_equal(rp["topk_idx"][t], r["topk_idx"][t])   # the step keeps the selection
            assert np.array_equal(rm["topk_idx"][t], r["topk_idx"][t])
            fd = float(np.dot(rp["topk_prob"][t].astype(np.float64) - rm["topk_prob"][t], dprob[t])) / (2 * h)
            assert abs(dl[t, e] - fd) <= 2e-3 * (1.0 + abs(fd)), (t, e, dl[t, e], fd)


def test_router_backward_softmax_gradients_sum_to_zero():
    rng = np.random.default_rng(5)
    logits = rng.standard_normal((50, 64)).astype(np.float32) * 2
    dprob = rng.standard_normal((50, 8)).astype(np.float32)
    for renorm in (True, False):
        r = oracle.router_topk(logits, 8, 0, renorm)
        dl = oracle.router_backward(logits, r["topk_idx"], dprob, 0, renorm).astype(np.float64)
        assert np.all(np.abs(dl.sum(axis=1)) <= 1e-6 * (1 + np.abs(dl).sum(axis=1)))
        if renorm:   # only the chosen experts get a gradient
            mask = np.zeros_like(dl, bool)
            np.put_along_axis(mask, r["topk_idx"].astype(np.int64), True, axis=1)
            assert np.all(dl[~mask] == 0)


def test_router_backward_sigmoid_is_the_logistic_derivative():
    # one expert chosen, no renormalisation: dl = g s (1 - s) at the chosen expert
    logits = np.array([[0.3, -1.2, 2.0, 0.0]], np.float32)
    r = oracle.router_topk(logits, 1, 1, False)
    assert r["topk_idx"][0, 0] == 2
    dl = oracle.router_backward(logits, r["topk_idx"], np.array([[1.5]], np.float32), 1, False, 2.0)
    s = 1 / (1 + np.exp(-2.0))
    assert dl[0, 2] == pytest.approx(2.0 * 1.5 * s * (1 - s), rel=1e-6)
    assert np.count_nonzero(dl) == 1
