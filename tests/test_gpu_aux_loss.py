"""Auxiliary load-balancing loss on the GPU (Transformer Engine "Mixture of
Experts", Load balancing), through the C ABI, against the oracle's fp64
reading of it: the loss, the dense scores and the gradient to the logits.

Tolerances come from the fp32 arithmetic. A score has a few ulp of error
(expf, one division). The loss sums at most T/(warps of the grid) + 8 scores
per expert in fp32 before the fp64 sum over blocks, hence 1e-5 relative. A
gradient element s_i (G_i - sum_e s_e G_e) carries the rounding of an E-term
dot product of terms up to max|G|, hence 2e-6 * max|G| + 1e-5 |ref|."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from helpers import require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def case(T, E, k, score, seed, counts_from_router=True):
    import routing_grouped_gemm_score_b200 as m
    g = torch.Generator().manual_seed(seed)
    logits = (torch.randn((T, E), generator=g) * 2.0).float()
    if counts_from_router:
        r = m.moe_router_topk(logits.cuda(), k, m.RouterOpts(score, score == 0))
        counts = r["counts"]
    else:
        counts = torch.randint(0, 3 * T * k // E + 2, (E,), generator=g, dtype=torch.int32).cuda()
    return m, logits, counts


SHAPES = [(64, 8, 2, 0), (4096, 128, 8, 0), (1000, 16, 1, 1), (1, 256, 16, 0), (3000, 40, 4, 1),
          (70000, 128, 8, 0), (257, 64, 6, 1)]


@pytest.mark.parametrize("T,E,k,score", SHAPES)
def test_loss_and_scores_match_the_oracle(T, E, k, score):
    m, logits, counts = case(T, E, k, score, seed=T + E)
    coeff = 0.01
    loss, scores = m.moe_aux_loss(logits.cuda(), counts, k, coeff, score, want_scores=True)
    torch.cuda.synchronize()
    ref = oracle.aux_loss(logits.numpy(), counts.cpu().numpy(), k, coeff, score)
    assert abs(float(loss) - ref) <= 1e-5 * abs(ref), (float(loss), ref)
    sref = oracle.aux_scores(logits.numpy(), score)
    np.testing.assert_allclose(scores.cpu().numpy(), sref, rtol=2e-6, atol=1e-12)
    # the same bits on a second call
    loss2, _ = m.moe_aux_loss(logits.cuda(), counts, k, coeff, score)
    assert torch.equal(loss.view(torch.int32), loss2.view(torch.int32))


def test_workload_logits_and_random_counts():
    """The Qwen3 workload's own logits, counts from the router and counts
    unrelated to the scores."""
    import routing_grouped_gemm_score_b200 as m
    w = wl.WORKLOADS["qwen3_30b_a3b"]
    logits = wl.make_logits(w, "cuda")
    r = m.moe_router_topk(logits, w.k)
    for counts in (r["counts"], torch.arange(w.E, dtype=torch.int32, device="cuda") * 3):
        loss, _ = m.moe_aux_loss(logits, counts, w.k, 1e-3)
        ref = oracle.aux_loss(logits.cpu().numpy(), counts.cpu().numpy(), w.k, 1e-3)
        assert abs(float(loss) - ref) <= 1e-5 * abs(ref)


@pytest.mark.parametrize("T,E,k,score", SHAPES[:5])
@pytest.mark.parametrize("accumulate", [False, True])
def test_gradient_matches_the_oracle(T, E, k, score, accumulate):
    m, logits, counts = case(T, E, k, score, seed=3 * T + E, counts_from_router=False)
    coeff = 0.05
    gl = torch.tensor(2.5, device="cuda")
    base = torch.randn((T, E), generator=torch.Generator().manual_seed(7)).float().cuda()
    d = base.clone() if accumulate else None
    out = m.moe_aux_loss_backward(logits.cuda(), counts, k, coeff, score, grad_loss=gl, dlogits=d,
                                  accumulate=accumulate)
    torch.cuda.synchronize()
    assert m.moe_get_device_status() == 0
    ref = oracle.aux_loss_backward(logits.numpy(), counts.cpu().numpy(), k, coeff, score, grad_loss=2.5)
    got = out.cpu().numpy().astype(np.float64)
    if accumulate:
        got = got - base.cpu().numpy().astype(np.float64)
        slack = 1e-6 * np.abs(base.cpu().numpy()).max()     # one fp32 rounding of the sum
    else:
        slack = 0.0
    G = 2.5 * coeff * E * counts.cpu().numpy().astype(np.float64) / (k * T * T)
    tol = 2e-6 * np.abs(G).max() + 1e-5 * np.abs(ref) + slack
    assert np.all(np.abs(got - ref) <= tol), np.abs(got - ref).max()


def test_gradient_without_a_grad_tensor_is_the_unit_gradient():
    m, logits, counts = case(128, 32, 4, 0, seed=11)
    a = m.moe_aux_loss_backward(logits.cuda(), counts, 4, 0.3, 0)
    b = m.moe_aux_loss_backward(logits.cuda(), counts, 4, 0.3, 0, grad_loss=torch.tensor(1.0, device="cuda"))
    assert torch.equal(a, b)
