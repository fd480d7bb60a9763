"""Pins of the oracle's router (score function, top-k, routing weights,
counts and offsets) against brute force, closed forms and invariants.

Transformer Engine "Mixture of Experts", section Router; te_mixtral.py,
TEMixtralSparseMoeBlock.forward.
"""
import math

import numpy as np
import pytest

import workloads as wl


def brute_topk(keys, k):
    """Full sort of the experts by (key descending, index ascending)."""
    E = len(keys)
    def rank_key(e):
        v = float(keys[e])
        return (1 if math.isnan(v) else 0, -v if not math.isnan(v) else 0.0, e)
    return sorted(range(E), key=rank_key)[:k]


@pytest.mark.parametrize("E,k,quant", [(8, 2, 0.0), (16, 1, 0.0), (128, 8, 0.0), (130, 8, 0.0),
                                       (256, 16, 0.0), (128, 8, 0.5), (8, 2, 1.0), (33, 5, 0.25)])
def test_topk_matches_full_sort(oracle_lib, E, k, quant):
    rng = np.random.default_rng(E * 100 + k)
    logits = rng.standard_normal((300, E)).astype(np.float32)
    if quant:
        logits = (np.round(logits / quant) * quant).astype(np.float32)
    r = oracle_lib.router_topk(logits, k)
    for t in range(logits.shape[0]):
        assert list(r["topk_idx"][t]) == brute_topk(logits[t], k)


def test_tie_workload_exercises_lower_index_rule(oracle_lib):
    w = wl.WORKLOADS["tie_t64"]
    logits = wl.make_logits(w).numpy()
    r = oracle_lib.router_topk(logits, w.k)
    ties_at_boundary = 0
    for t in range(w.T):
        sel = list(r["topk_idx"][t])
        assert sel == brute_topk(logits[t], w.k)
        kth = logits[t, sel[-1]]
        unselected_equal = [e for e in range(w.E) if e not in sel and logits[t, e] == kth]
        # every unselected expert with the k-th score has a larger index
        assert all(e > sel[-1] for e in unselected_equal)
        ties_at_boundary += bool(unselected_equal)
    assert ties_at_boundary > w.T // 2     # the workload really has boundary ties


def test_softmax_renormalised_weights_closed_form(oracle_lib):
    rng = np.random.default_rng(7)
    logits = (rng.standard_normal((500, 64)) * 3).astype(np.float32)
    k = 6
    r = oracle_lib.router_topk(logits, k)
    l64 = logits.astype(np.float64)
    # softmax over all experts, then keep the chosen and renormalise (te_mixtral)
    full = np.exp(l64 - l64.max(1, keepdims=True))
    full /= full.sum(1, keepdims=True)
    sel = np.take_along_axis(full, r["topk_idx"].astype(np.int64), 1)
    expect = sel / sel.sum(1, keepdims=True)
    np.testing.assert_allclose(r["topk_prob"], expect, rtol=2e-6, atol=0)
    np.testing.assert_allclose(r["topk_prob"].astype(np.float64).sum(1), 1.0, rtol=0, atol=1e-6)
    # weights come out in selection order, so they never increase along a row
    assert np.all(np.diff(r["topk_prob"], axis=1) <= 0)


def test_equal_logits_get_identical_weights(oracle_lib):
    logits = np.zeros((4, 16), np.float32)
    logits[1, :] = 2.5
    logits[2, ::2] = 1.0
    logits[3] = np.arange(16, dtype=np.float32) // 4
    r = oracle_lib.router_topk(logits, 4)
    assert np.all(r["topk_prob"][0] == np.float32(0.25))
    assert list(r["topk_idx"][0]) == [0, 1, 2, 3]
    assert list(r["topk_idx"][2]) == [0, 2, 4, 6]
    assert len(set(r["topk_prob"][2].tolist())) == 1
    assert list(r["topk_idx"][3]) == [12, 13, 14, 15]


def test_pre_softmax_weights(oracle_lib):
    rng = np.random.default_rng(3)
    logits = rng.standard_normal((200, 32)).astype(np.float32)
    r = oracle_lib.router_topk(logits, 4, renormalize=False)
    l64 = logits.astype(np.float64)
    full = np.exp(l64 - l64.max(1, keepdims=True))
    full /= full.sum(1, keepdims=True)
    expect = np.take_along_axis(full, r["topk_idx"].astype(np.int64), 1)
    np.testing.assert_allclose(r["topk_prob"], expect, rtol=2e-6)
    assert np.all(r["topk_prob"].sum(1) < 1.0)


def test_sigmoid_top1_is_not_renormalised(oracle_lib):
    w = wl.WORKLOADS["llama4_17bx16e"].scaled(T=300)
    logits = wl.make_logits(w).numpy()
    r = oracle_lib.router_topk(logits, 1, score=wl.SCORE_SIGMOID, renormalize=False)
    l = logits[np.arange(300), r["topk_idx"][:, 0]].astype(np.float64)
    expect = 1.0 / (1.0 + np.exp(-l))
    np.testing.assert_allclose(r["topk_prob"][:, 0], expect, rtol=1e-6)
    assert np.all(r["topk_prob"] < 1.0)        # top-1 weight is not one: must be applied
    for t in range(300):
        assert r["topk_idx"][t, 0] == brute_topk(logits[t], 1)[0]


def test_scaling_factor_and_bias(oracle_lib):
    rng = np.random.default_rng(11)
    logits = rng.standard_normal((200, 16)).astype(np.float32)
    a = oracle_lib.router_topk(logits, 3, score=1, renormalize=True)
    b = oracle_lib.router_topk(logits, 3, score=1, renormalize=True, scaling=2.5)
    assert np.array_equal(a["topk_idx"], b["topk_idx"])
    np.testing.assert_allclose(b["topk_prob"], 2.5 * a["topk_prob"], rtol=1e-6)
    bias = (rng.standard_normal(16) * 0.5).astype(np.float32)
    c = oracle_lib.router_topk(logits, 3, score=1, renormalize=False, expert_bias=bias)
    sig = (1.0 / (1.0 + np.exp(-logits.astype(np.float64))))
    for t in range(200):
        assert list(c["topk_idx"][t]) == brute_topk(sig[t] + bias, 3)
    # the bias picks the experts but does not enter the weights
    l = np.take_along_axis(logits.astype(np.float64), c["topk_idx"].astype(np.int64), 1)
    np.testing.assert_allclose(c["topk_prob"], 1.0 / (1.0 + np.exp(-l)), rtol=1e-6)
    with pytest.raises(ValueError):
        oracle_lib.router_topk(logits, 3, score=0, expert_bias=bias)


@pytest.mark.parametrize("name", ["tiny", "qwen3_30b_a3b", "skew_t16384", "tie_t64"])
def test_counts_offsets_invariants(oracle_lib, name):
    w = wl.WORKLOADS[name]
    logits = wl.make_logits(w).numpy()
    r = oracle_lib.router_topk(logits, w.k)
    rmap = r["routing_map"]
    assert np.all(rmap.sum(1) == w.k)
    assert np.array_equal(r["counts"], rmap.sum(0).astype(np.int32))
    assert r["counts"].sum() == w.T * w.k
    assert r["offsets"][0] == 0 and r["offsets"][-1] == w.T * w.k
    assert np.array_equal(np.diff(r["offsets"]), r["counts"])
    for t in range(min(w.T, 512)):
        assert len(set(r["topk_idx"][t].tolist())) == w.k
    if w.dead_experts:
        dead = wl.skew_bias(w).numpy() < -1e3
        assert dead.sum() == w.dead_experts
        assert np.all(r["counts"][dead] == 0)
        # the 3 ln(1/rank) bias concentrates the load on the best-ranked experts
        assert r["counts"].max() > 4 * w.T * w.k / w.E


def test_degenerate_logits(oracle_lib):
    logits = np.array([[0.0, -np.inf, 1.0, np.nan, -np.inf, 1.0]], np.float32)
    r = oracle_lib.router_topk(logits, 6)
    assert list(r["topk_idx"][0]) == [2, 5, 0, 1, 4, 3]     # NaN last, -inf before it
    r = oracle_lib.router_topk(logits, 3)
    assert list(r["topk_idx"][0]) == [2, 5, 0]
    e = np.exp(np.float64(-1.0))
    np.testing.assert_allclose(r["topk_prob"][0], [1 / (2 + e), 1 / (2 + e), e / (2 + e)], rtol=1e-6)
    with pytest.raises(ValueError):
        oracle_lib.router_topk(logits, 7)
