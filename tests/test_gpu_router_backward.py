"""Router backward on the GPU (moe_router_backward: dL/dlogits from
dL/dtopk_prob) against the oracle, every score/weight mode and every
experts-per-lane count, plus the Qwen3-30B-A3B shape on all tokens.

Tolerance, from the fp32 arithmetic: each output is q * (g - c) (or the
sigmoid analogue), where q comes from exp and a sum of n terms (n = E for a
softmax over all experts, else k) and c from a sum of k products. The GPU's
fp32 result is then within about (n + 8) units of 2^-24 of the magnitude of
the terms involved; the test allows 1e-5 (1 + n/16) times that magnitude,
computed per element in fp64."""
import numpy as np
import pytest
import torch

import oracle
from helpers import require_gpu

pytestmark = pytest.mark.gpu

MODES = {"softmax_renorm": (0, True), "softmax_all": (0, False), "sigmoid": (1, False),
         "sigmoid_renorm": (1, True)}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _scale(logits, idx, dprob, score, renorm, scaling):
    """Per element: the magnitude of the terms its value is made of."""
    l = logits.astype(np.float64)
    g = np.abs(scaling * dprob.astype(np.float64))
    T, E = l.shape
    out = np.zeros((T, E))
    rows = np.arange(T)[:, None]
    if score == 0:
        src = l[rows, idx] if renorm else l
        q = np.exp(src - src.max(axis=1, keepdims=True))
        q /= q.sum(axis=1, keepdims=True)
        qsel = q if renorm else q[rows, idx]
        c = (qsel * g).sum(axis=1, keepdims=True)
        if renorm:
            out[rows, idx] = qsel * (g + c)
        else:
            out = q * c
            out[rows, idx] = qsel * (g + c)
    else:
        s = 1 / (1 + np.exp(-l[rows, idx]))
        S = s.sum(axis=1, keepdims=True) if renorm else 1.0
        c = ((s / S) * g).sum(axis=1, keepdims=True) if renorm else 0.0
        out[rows, idx] = (g + c) / S * s * (1 - s)
    return out


def _check(logits, k, score, renorm, scaling=1.0, seed=0):
    import routing_grouped_gemm_score_b200 as m
    opts = m.RouterOpts(score, renorm, scaling)
    lg = torch.from_numpy(logits).cuda()
    fwd = m.moe_router_topk(lg, k, opts)
    rng = np.random.default_rng(seed)
    dprob = rng.standard_normal((logits.shape[0], k)).astype(np.float32)
    dl = m.moe_router_backward(lg, fwd["topk_idx"], torch.from_numpy(dprob).cuda(), opts)
    torch.cuda.synchronize()
    assert m.moe_get_device_status() == 0
    idx = fwd["topk_idx"].cpu().numpy()
    ref = oracle.router_backward(logits, idx, dprob, score, renorm, scaling).astype(np.float64)
    got = dl.cpu().numpy().astype(np.float64)
    n = logits.shape[1] if (score == 0 and not renorm) else k
    tol = 1e-5 * (1 + n / 16) * _scale(logits, idx, dprob, score, renorm, scaling) + 1e-12
    bad = np.abs(got - ref) > tol
    assert not bad.any(), (f"{int(bad.sum())} of {bad.size} off; first {tuple(np.argwhere(bad)[0])}: "
                           f"gpu {got[bad][0]!r} ref {ref[bad][0]!r} tol {tol[bad][0]!r}")
    if score == 0 and renorm or score == 1:    # only the chosen experts carry a gradient
        mask = np.zeros_like(got, bool)
        np.put_along_axis(mask, idx.astype(np.int64), True, axis=1)
        assert np.all(got[~mask] == 0)


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("E,k", [(20, 3), (64, 8), (128, 8), (256, 16), (48, 1)])
def test_router_backward_matches_oracle(E, k, mode):
    score, renorm = MODES[mode]
    rng = np.random.default_rng(E * 7 + k)
    logits = (rng.standard_normal((97, E)) * 3).astype(np.float32)
    _check(logits, k, score, renorm, scaling=1.5, seed=E)


def test_router_backward_qwen3_shape_all_tokens():
    import workloads as wl
    w = wl.WORKLOADS["qwen3_30b_a3b"]
    logits = wl.make_logits(w, "cpu").numpy()
    _check(logits, w.k, w.score, w.renormalize, seed=11)


def test_router_backward_empty_batch():
    import routing_grouped_gemm_score_b200 as m
    lg = torch.empty((0, 16), device="cuda")
    out = m.moe_router_backward(lg, torch.empty((0, 2), dtype=torch.int32, device="cuda"),
                                torch.empty((0, 2), device="cuda"))
    assert out.shape == (0, 16)
