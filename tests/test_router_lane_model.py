"""The argument behind the large-T router's 32-bit selection, checked on the
host against the oracle's exact picks (Transformer Engine "Mixture of
Experts", Router: top-k with ties to the lower expert index).

The kernel sorts 32-bit entries: the top 32 - ib bits of the score's signed
order key, with 2^ib - 1 - e in the low ib bits. Its claim is that this order
differs from the exact one (larger score, then the lower index) only between
entries that share a prefix (+0 and -0 counted as one), so that:
  - when no two neighbours among the picks and the entry after them share a
    prefix, and no infinity or NaN sits at either end, the 32-bit picks are
    the exact picks, in order;
  - when only picks share prefixes, the set is exact and only the order may
    differ;
  - when the last pick and the entry after it share a prefix pb, the exact
    set is the picks with larger prefixes plus the best experts of prefix pb.
This model applies those rules with numpy sorts on thousands of adversarial
rows and compares each case with the oracle; the GPU tests compare the kernel
itself with the warp kernel and the oracle."""
import numpy as np
import pytest

import oracle


def entries(scores, ib):
    b = scores.astype(np.float32).view(np.int32).astype(np.int64)
    ks = b ^ ((b >> 31) & 0x7FFFFFFF)
    E = scores.shape[1]
    cmax = (1 << ib) - 1
    return (ks & ~cmax) | (cmax - np.arange(E)), cmax


def adversarial_rows(rng, T, E):
    l = rng.standard_normal((T, E)).astype(np.float32)
    bits = l.view(np.uint32)
    for t in range(T):
        kind = t % 6
        cols = rng.choice(E, int(rng.integers(2, 14)), replace=False)
        if kind == 0:     # a run of values inside one prefix, above the rest
            base = np.float32(rng.uniform(1.5, 4.0)).view(np.uint32) & np.uint32(0xFFFFFF00)
            bits[t, cols] = base | rng.integers(0, 256, len(cols)).astype(np.uint32)
        elif kind == 1:   # the same around the 8th largest
            base = np.sort(l[t])[-8].view(np.uint32) & np.uint32(0xFFFFFF00)
            bits[t, cols] = base | rng.integers(0, 256, len(cols)).astype(np.uint32)
        elif kind == 2:   # exact ties (quantised values)
            l[t] = np.round(l[t] * 2) / 2
        elif kind == 3:   # zeros of both signs and denormals on top
            l[t] -= 10
            l[t, cols] = rng.choice(np.array([0.0, -0.0, 1e-45, -1e-45, 3e-45], np.float32), len(cols))
        elif kind == 4:   # negative values in one prefix
            l[t] -= 20
            base = np.float32(-3.0).view(np.uint32) & np.uint32(0xFFFFFF00)
            bits[t, cols] = base | rng.integers(0, 256, len(cols)).astype(np.uint32)
        elif kind == 5 and t % 12 == 5:   # infinities and NaNs of both signs
            l[t, cols[:2]] = np.array([np.inf, -np.inf], np.float32)[: len(cols[:2])]
            bits[t, cols[2:4]] = np.array([0x7FC00001, 0xFFC00002], np.uint32)[: len(cols[2:4])]
        # otherwise kind 5: plain N(0,1)
    return l


@pytest.mark.parametrize("E,ib", [(128, 7), (64, 7), (256, 8), (160, 8)])
@pytest.mark.parametrize("k", [1, 3, 8])
def test_the_32bit_order_and_its_checks_give_the_exact_picks(E, ib, k):
    rng = np.random.default_rng(E * 10 + k)
    T = 3000
    l = adversarial_rows(rng, T, E)
    exact = oracle.router_topk(l, k, 0, True, with_map=False)["topk_idx"]
    ent, cmax = entries(l, ib)
    order = np.argsort(-ent, axis=1, kind="stable")[:, : k + 1]
    top = np.take_along_axis(ent, order, axis=1)
    pfx = top >> ib
    def close(a, b):
        return (a == b) | ((a == 0) & (b == -1))
    nxt = top[:, k]
    posinf = 0x7F800000
    neginf = np.int64(np.int32(np.uint32(0x807FFFFF)))
    edge = (top[:, 0] >= (posinf & ~cmax)) | (nxt <= (neginf | cmax)) | close(pfx[:, k - 1], pfx[:, k])
    inner = np.zeros(T, bool)
    for j in range(k - 1):
        inner |= close(pfx[:, j], pfx[:, j + 1])
    picks = order[:, :k]
    clean = ~edge & ~inner
    # no flag: the 32-bit picks are the exact picks, in order
    assert np.array_equal(picks[clean], exact[clean])
    # only picks share prefixes: the set is exact
    only_inner = ~edge & inner
    assert np.array_equal(np.sort(picks[only_inner], axis=1), np.sort(exact[only_inner], axis=1))
    # an edge tie inside one finite, non-zero prefix: the picks with larger
    # prefixes stay; the rest come from the experts of that prefix, exactly ranked
    fin = edge & ~((top[:, 0] >= (posinf & ~cmax)) | (nxt <= (neginf | cmax)))
    fin &= ~np.isin(pfx[:, k - 1], [0, -1])
    for t in np.nonzero(fin)[0]:
        pb = pfx[t, k - 1]
        sure = [int(e) for e, p in zip(picks[t], pfx[t, :k]) if p != pb]
        cands = [e for e in range(E) if (ent[t, e] >> ib) == pb]
        ranked = sorted(cands, key=lambda e: (-float(l[t, e]), e))[: k - len(sure)]
        assert sorted(sure + ranked) == sorted(exact[t].tolist()), t
    # the checks fire rarely on plain rows and always somewhere in this set
    assert clean.sum() > 0 and (edge | inner).sum() > 0
