"""Pins of the oracle's dispatch (permutation) and combine bookkeeping.

Transformer Engine "Mixture of Experts", sections Token dispatch, Token
combine and Token probabilities.
"""
import numpy as np
import pytest
import torch

import workloads as wl


def routed(oracle_lib, name, T=None):
    w = wl.WORKLOADS[name]
    if T is not None:
        w = w.scaled(T=T)
    logits = wl.make_logits(w).numpy()
    r = oracle_lib.router_topk(logits, w.k, score=w.score, renormalize=w.renormalize)
    return w, r


@pytest.mark.parametrize("name,T", [("tiny", None), ("qwen3_30b_a3b", 1000), ("skew_t64", None),
                                    ("skew_t1", None), ("llama4_17bx16e", 300)])
def test_dispatch_is_stable_sort_by_expert(oracle_lib, name, T):
    w, r = routed(oracle_lib, name, T)
    st, row_of = oracle_lib.dispatch(r["topk_idx"], r["offsets"], w.E)
    # brute force: sort all assignments by (expert, token); Python's sort is stable
    pairs = sorted(((int(e), t) for t in range(w.T) for e in r["topk_idx"][t]), key=lambda p: p)
    assert st.tolist() == [t for _, t in pairs]
    # row_of is a bijection onto [0, A) and the inverse of sorted_token
    A = w.T * w.k
    assert sorted(row_of.ravel().tolist()) == list(range(A))
    for t in range(w.T):
        for j in range(w.k):
            row = row_of[t, j]
            assert st[row] == t
            e = r["topk_idx"][t, j]
            assert r["offsets"][e] <= row < r["offsets"][e + 1]


def test_dispatch_rejects_bad_indices(oracle_lib):
    idx = np.array([[0, 1], [1, 5]], np.int32)
    offs = np.array([0, 1, 3, 4], np.int32)
    with pytest.raises(ValueError):
        oracle_lib.dispatch(idx, offs, 3)
    idx = np.array([[0, 1], [1, 1]], np.int32)          # counts disagree with offsets
    with pytest.raises(ValueError):
        oracle_lib.dispatch(idx, np.array([0, 2, 3, 4], np.int32), 3)


def test_gather_and_unpermute_roundtrip(oracle_lib):
    w, r = routed(oracle_lib, "tiny")
    x = oracle_lib.bf16_bits(wl.make_x(w))
    st, row_of = oracle_lib.dispatch(r["topk_idx"], r["offsets"], w.E)
    xp = oracle_lib.gather_rows(x, st)
    assert np.array_equal(xp, x[st])
    xf = oracle_lib.bits_to_float(x)
    xpf = oracle_lib.bits_to_float(xp)
    # unweighted combine of an identity expert: k copies of each token
    np.testing.assert_array_equal(oracle_lib.combine(xpf, row_of), w.k * xf)
    # k = 1: exactly the input back
    w1, r1 = routed(oracle_lib, "llama4_17bx16e", 64)
    x1 = oracle_lib.bf16_bits(wl.make_x(w1.scaled(H=128)))
    st1, ro1 = oracle_lib.dispatch(r1["topk_idx"], r1["offsets"], w1.E)
    back = oracle_lib.combine(oracle_lib.bits_to_float(oracle_lib.gather_rows(x1, st1)), ro1)
    np.testing.assert_array_equal(back, oracle_lib.bits_to_float(x1))


def test_identity_experts_with_renormalised_weights_return_x(oracle_lib):
    w, r = routed(oracle_lib, "qwen3_30b_a3b", 257)
    x = oracle_lib.bf16_bits(wl.make_x(w.scaled(H=64)))
    st, row_of = oracle_lib.dispatch(r["topk_idx"], r["offsets"], w.E)
    y = oracle_lib.bits_to_float(oracle_lib.gather_rows(x, st))
    out = oracle_lib.combine(y, row_of, r["topk_prob"])
    np.testing.assert_allclose(out, oracle_lib.bits_to_float(x), rtol=1e-6, atol=1e-7)


def test_combine_weights_follow_their_rows(oracle_lib):
    """Expert e multiplies by (e + 1): each output row must be
    sum_j p_j (e_j + 1) x, so a weight paired with the wrong row fails."""
    w, r = routed(oracle_lib, "tiny")
    x = oracle_lib.bf16_bits(wl.make_x(w))
    st, row_of = oracle_lib.dispatch(r["topk_idx"], r["offsets"], w.E)
    xpf = oracle_lib.bits_to_float(oracle_lib.gather_rows(x, st))
    scale = np.zeros(len(st))
    for e in range(w.E):
        scale[r["offsets"][e]:r["offsets"][e + 1]] = e + 1
    out = oracle_lib.combine(xpf * scale[:, None], row_of, r["topk_prob"])
    coef = (r["topk_prob"].astype(np.float64) * (r["topk_idx"] + 1)).sum(1)
    np.testing.assert_allclose(out, coef[:, None] * oracle_lib.bits_to_float(x), rtol=1e-12)


def test_shared_expert_output_is_the_base(oracle_lib):
    rng = np.random.default_rng(0)
    y = rng.standard_normal((6, 8))
    row_of = np.array([[0], [1], [2], [3], [4], [5]], np.int32)
    shared = rng.standard_normal((6, 8))
    p = rng.random((6, 1)).astype(np.float32)
    out = oracle_lib.combine(y, row_of, p, shared=shared)
    np.testing.assert_allclose(out, shared + p.astype(np.float64) * y, rtol=1e-15)


def test_bf16_rounding(oracle_lib):
    rng = np.random.default_rng(5)
    vals = np.concatenate([rng.standard_normal(2000) * 10.0 ** rng.integers(-30, 30, 2000),
                           [0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.0e38, 1e-40, -2.5]])
    for v in vals:
        b = oracle_lib.round_bf16(v)
        # brute force: the nearest of the bf16 neighbours, ties to the even pattern
        f = np.float32(v)
        base = int(np.array([f], np.float32).view(np.uint32)[0] >> 16)
        cands = [c & 0xFFFF for c in (base - 1, base, base + 1, base + 2)]
        cv = oracle_lib.bits_to_float(np.array(cands, np.uint16))
        d = np.abs(cv - v)
        d[np.isnan(d)] = np.inf
        best = [c for c, dd in zip(cands, d) if dd == d.min()]
        if len(best) > 1:
            best = [c for c in best if c % 2 == 0]
        assert b == best[0], (v, hex(b), [hex(c) for c in best])
    # agrees with torch's fp32 -> bf16 conversion on fp32 inputs
    f32 = (rng.standard_normal(5000) * 3).astype(np.float32)
    tb = torch.from_numpy(f32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert all(oracle_lib.round_bf16(float(a)) == int(b) for a, b in zip(f32, tb))


# ------------------------------------------------------------ padded dispatch
# Transformer Engine "Mixture of Experts", Token permutation, Padding and alignment.

def test_padded_dispatch_pages_example(oracle_lib):
    """The page's example: counts of 129 and 127 take 384 rows at an
    alignment of 128, although only 256 tokens arrive."""
    topk = np.array([[0]] * 129 + [[1]] * 127, np.int32)
    offsets = np.array([0, 129, 256], np.int32)
    padded, st, row_of = oracle_lib.dispatch_padded(topk, offsets, 2, 128)
    assert padded.tolist() == [0, 256, 384]
    assert len(st) == 384
    assert np.all(st[129:256] == -1) and np.all(st[256 + 127:] == -1)
    assert st[:129].tolist() == list(range(129)) and st[256:383].tolist() == list(range(129, 256))


def test_padded_dispatch_with_align_one_is_the_dispatch(oracle_lib):
    w, r = routed(oracle_lib, "qwen3_30b_a3b", 300)
    st, row_of = oracle_lib.dispatch(r["topk_idx"], r["offsets"], w.E)
    padded, st1, row_of1 = oracle_lib.dispatch_padded(r["topk_idx"], r["offsets"], w.E, 1)
    assert np.array_equal(padded, r["offsets"]) and np.array_equal(st1, st) and np.array_equal(row_of1, row_of)


@pytest.mark.parametrize("name,T,align", [("qwen3_30b_a3b", 500, 16), ("skew_t64", None, 128),
                                          ("mixtral_8x7b", 700, 256), ("tiny", None, 3)])
def test_padded_dispatch_invariants(oracle_lib, name, T, align):
    w, r = routed(oracle_lib, name, T)
    offsets = r["offsets"].astype(np.int64)
    padded, st, row_of = oracle_lib.dispatch_padded(r["topk_idx"], r["offsets"], w.E, align)
    padded = padded.astype(np.int64)
    counts, pcounts = np.diff(offsets), np.diff(padded)
    assert np.all(padded % align == 0)                       # every block starts aligned
    assert np.all((pcounts - counts >= 0) & (pcounts - counts < align))
    assert np.all((pcounts == 0) == (counts == 0))           # an empty block stays empty
    # the pad rows are exactly the tail of each block
    pad = np.zeros(len(st), bool)
    for e in range(w.E):
        pad[padded[e] + counts[e]:padded[e + 1]] = True
    assert np.all((st < 0) == pad)
    # row_of is a bijection onto the real rows, inverse to sorted_token, and keeps
    # the unpadded order inside each block
    rows = row_of.ravel()
    assert len(np.unique(rows)) == rows.size and not np.any(pad[rows])
    t_of = np.repeat(np.arange(w.T), w.k)
    assert np.array_equal(st[rows], t_of)
    _, row_plain = oracle_lib.dispatch(r["topk_idx"], r["offsets"], w.E)
    e_of = r["topk_idx"].ravel()
    assert np.array_equal(rows - padded[e_of], row_plain.ravel() - offsets[e_of])


def test_gather_rows_zero_fills_pad_rows(oracle_lib):
    x = np.arange(12, dtype=np.uint16).reshape(3, 4) + 1
    out = oracle_lib.gather_rows(x, np.array([2, -1, 0, -1], np.int32))
    assert out.tolist() == [[9, 10, 11, 12], [0, 0, 0, 0], [1, 2, 3, 4], [0, 0, 0, 0]]
