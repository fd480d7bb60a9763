"""Router parity on the GPU: topk_idx, routing_map, counts and offsets
bit-exact, routing weights within 1e-6 relative, against the oracle on the
same seeded logits (Transformer Engine "Mixture of Experts", Router)."""
import numpy as np
import pytest
import torch

import helpers
import workloads as wl
from helpers import assert_equal, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def run_both(logits, k, score=0, renormalize=True, scaling=1.0, bias=None):
    import oracle
    import routing_grouped_gemm_score_b200 as m
    opts = m.RouterOpts(score, renormalize, scaling, None if bias is None else bias.cuda())
    g = m.moe_router_topk(logits.cuda(), k, opts, routing_map=True)
    torch.cuda.synchronize()
    assert m.moe_get_device_status() == 0
    r = oracle.router_topk(logits.cpu().numpy(), k, score, renormalize, scaling,
                           None if bias is None else bias.cpu().numpy())
    return g, r


def check(g, r):
    assert_equal(g["topk_idx"], r["topk_idx"], "topk_idx")
    assert_equal(g["routing_map"], r["routing_map"], "routing_map")
    assert_equal(g["counts"], r["counts"], "counts")
    assert_equal(g["offsets"], r["offsets"], "offsets")
    np.testing.assert_allclose(g["topk_prob"].cpu().numpy(), r["topk_prob"], rtol=1e-6, atol=0)


@pytest.mark.parametrize("name", ["tiny", "mixtral_8x7b", "qwen3_30b_a3b", "llama4_17bx16e",
                                  "skew_t1", "skew_t8", "skew_t64", "skew_t16384", "tie_t64"])
def test_router_workloads(name):
    w = wl.WORKLOADS[name]
    logits = wl.make_logits(w, "cuda")
    g, r = run_both(logits, w.k, w.score, w.renormalize)
    check(g, r)


@pytest.mark.parametrize("E,k", [(1, 1), (7, 3), (31, 4), (32, 8), (33, 1), (64, 16), (100, 6),
                                 (129, 8), (256, 16), (256, 1)])
def test_router_shapes_ragged_token_blocks(E, k):
    g_ = torch.Generator().manual_seed(E * 17 + k)
    logits = torch.randn((193, E), generator=g_)      # 193 = three token blocks + a tail
    g, r = run_both(logits, k)
    check(g, r)


def test_router_ties_and_degenerate_values():
    g_ = torch.Generator().manual_seed(5)
    logits = torch.round(torch.randn((300, 64), generator=g_) * 2) / 2
    logits[0] = 0.0
    logits[1, ::3] = float("-inf")
    logits[2, 5] = float("nan")
    logits[3] = -0.0
    logits[3, 10] = 0.0
    logits[4, :] = float("-inf")
    logits[4, 7] = 1.0
    g, r = run_both(logits, 8)
    assert_equal(g["topk_idx"], r["topk_idx"], "topk_idx")
    assert_equal(g["counts"], r["counts"], "counts")
    gp, rp = g["topk_prob"].cpu().numpy(), r["topk_prob"]
    finite = np.isfinite(rp)
    np.testing.assert_allclose(gp[finite], rp[finite], rtol=1e-6, atol=0)
    assert np.array_equal(np.isnan(gp), np.isnan(rp))


MODES = {"softmax_renorm": (0, True), "softmax_all": (0, False), "sigmoid": (1, False),
         "sigmoid_renorm": (1, True)}


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("k", [1, 2, 3, 4, 6, 8, 16])
@pytest.mark.parametrize("E", [20, 64, 128, 256])
def test_router_every_slot_count_and_k(E, k, mode):
    """Each lane holds E/32 experts (1, 2, 4 or 8 slots) and k = 1, 2, 4, 6, 8
    have kernels of their own, other k a generic one: every pairing, every
    score function and weight mode."""
    score, renorm = MODES[mode]
    g_ = torch.Generator().manual_seed(E * 131 + k * 7 + score * 3 + renorm)
    logits = torch.randn((97, E), generator=g_) * 3
    check(*run_both(logits, k, score, renorm))


@pytest.mark.parametrize("mode", list(MODES))
def test_router_degenerate_values_every_mode(mode):
    """NaN at expert 0 (the row maximum scan then yields NaN), a NaN elsewhere,
    rows of -inf, signed zeros: indices exact, NaN where the oracle has NaN."""
    score, renorm = MODES[mode]
    g_ = torch.Generator().manual_seed(17)
    logits = torch.randn((64, 128), generator=g_)
    logits[0, 0] = float("nan")
    logits[1, 77] = float("nan")
    logits[2] = float("-inf")
    logits[3] = -0.0
    logits[3, 100] = 0.0
    logits[4, :120] = float("nan")
    g, r = run_both(logits, 8, score, renorm)
    assert_equal(g["topk_idx"], r["topk_idx"], "topk_idx")
    assert_equal(g["routing_map"], r["routing_map"], "routing_map")
    assert_equal(g["counts"], r["counts"], "counts")
    gp, rp = g["topk_prob"].cpu().numpy(), r["topk_prob"]
    assert np.array_equal(np.isnan(gp), np.isnan(rp)), "NaN positions"
    finite = np.isfinite(rp)
    np.testing.assert_allclose(gp[finite], rp[finite], rtol=1e-6, atol=0)


def test_router_options():
    g_ = torch.Generator().manual_seed(9)
    logits = torch.randn((500, 48), generator=g_) * 2
    check(*run_both(logits, 6, renormalize=False))                  # softmax before top-k
    check(*run_both(logits, 6, score=1, renormalize=False))         # sigmoid
    check(*run_both(logits, 6, score=1, renormalize=True))          # sigmoid, renormalised
    check(*run_both(logits, 6, scaling=2.5))                        # scaling factor
    bias = torch.randn(48, generator=g_) * 0.3
    check(*run_both(logits, 6, score=1, renormalize=False, bias=bias))


def test_router_empty_batch():
    import routing_grouped_gemm_score_b200 as m
    g = m.moe_router_topk(torch.empty((0, 16), device="cuda"), 2)
    assert g["counts"].sum().item() == 0 and g["offsets"].abs().sum().item() == 0


def test_router_large_sweep_invariants():
    """T = 2^18 tokens at E=128, k=8: checked against the oracle on every row."""
    g_ = torch.Generator().manual_seed(21)
    logits = torch.randn((1 << 18, 128), generator=g_)
    g, r = run_both(logits, 8)
    check(g, r)


@pytest.mark.parametrize("E", [1, 8, 100, 128, 256])
def test_expert_bias_update_matches_oracle(E):
    """Aux-loss-free load balancing: the bias update from the router's own
    counts, on the device, against the oracle; then the next routing with the
    new bias (sigmoid score)."""
    import oracle
    import routing_grouped_gemm_score_b200 as m
    g_ = torch.Generator().manual_seed(E)
    logits = torch.randn((777, E), generator=g_) * 2
    k = min(E, 4)
    bias = (torch.randn(E, generator=g_) * 0.1).cuda()
    opts = m.RouterOpts(m.SCORE_SIGMOID, False, 1.0, bias)
    r = m.moe_router_topk(logits.cuda(), k, opts)
    before = bias.cpu().numpy().copy()
    m.moe_expert_bias_update(r["counts"], bias, 1e-3)
    torch.cuda.synchronize()
    ref = oracle.expert_bias_update(r["counts"].cpu().numpy(), before, 1e-3)
    np.testing.assert_allclose(bias.cpu().numpy(), ref, rtol=0, atol=1e-6 * 1e-3 + 1e-7 * np.abs(ref).max())
    g, o = run_both(logits, k, 1, False, 1.0, bias.cpu())
    check(g, o)


LANE_CASES = [(1, 32, 1, "softmax_renorm"), (255, 64, 2, "softmax_renorm"), (256, 128, 8, "softmax_renorm"),
              (1000, 128, 8, "sigmoid"), (777, 256, 3, "sigmoid_renorm"), (513, 96, 6, "softmax_renorm"),
              (40001, 128, 8, "softmax_renorm"), (9000, 160, 7, "sigmoid")]


def _router_outputs(logits, k, score, renorm, kernel, monkeypatch, bias=None, scaling=1.0):
    import routing_grouped_gemm_score_b200 as m
    helpers.force_kernels(router=kernel)
    opts = m.RouterOpts(score, renorm, scaling, bias)
    g = m.moe_router_topk(logits, k, opts, routing_map=True)
    torch.cuda.synchronize()
    assert m.moe_get_device_status() == 0
    return {n: v.clone() for n, v in g.items() if v is not None}


@pytest.mark.parametrize("T,E,k,mode", LANE_CASES)
def test_lane_router_matches_warp_router_bit_for_bit(T, E, k, mode, monkeypatch):
    """The lane-per-token kernel (large T) and the warp-per-token kernel give
    the same bits in every output, on ragged T (not a multiple of the
    256-token lane block), E = 32 .. 256 and k = 1 .. 8."""
    score, renorm = MODES[mode]
    g_ = torch.Generator().manual_seed(T * 3 + E + k)
    logits = (torch.randn((T, E), generator=g_) * 2).cuda()
    a = _router_outputs(logits, k, score, renorm, "lane", monkeypatch)
    b = _router_outputs(logits, k, score, renorm, "warp", monkeypatch)
    for n in b:
        assert torch.equal(a[n].view(torch.uint8), b[n].view(torch.uint8)), n


def _near_tie_logits(T, E, seed):
    """Rows where a dozen experts hold floats that differ only in the low 8
    bits of their order key (one 24-bit prefix, different values), on both
    signs and around the 8th largest, so that the picks and the first entry
    after them fall inside one prefix; rows of +0, -0 and denormals on top;
    rows with +inf on top of near-equal values; rows where only the first
    three picks share a prefix (their order, not the set, is in question)."""
    rng = np.random.default_rng(seed)
    base = rng.standard_normal((T, E)).astype(np.float32)
    bits = base.view(np.uint32)
    for t in range(T):
        cols = rng.choice(E, 12, replace=False)
        kind = t % 6
        if kind == 3:      # zeros of both signs and tiny denormals above the rest
            base[t] -= 10.0
            base[t, cols] = np.array([0.0, -0.0, 1e-45, -1e-45, 2e-45, -3e-45] * 2, np.float32)
            continue
        if kind == 1:      # negative, with the rest pushed below
            base[t] -= 10.0
        if kind == 5:      # three picks far above the rest, inside one prefix
            cols = cols[:3]
        b0 = {0: np.float32(3.0), 1: np.float32(-2.5), 2: np.sort(base[t])[-8], 4: np.float32(1.75),
              5: np.float32(6.0)}[kind]
        low = rng.integers(0, 256, len(cols)).astype(np.uint32)
        bits[t, cols] = (np.float32(b0).view(np.uint32) & np.uint32(0xFFFFFF00)) | low
        if kind == 4:      # +inf above them
            base[t, cols[0]] = np.inf
    return torch.from_numpy(base)


@pytest.mark.parametrize("k,E", [(8, 128), (3, 128), (7, 128), (8, 256), (5, 160)])
@pytest.mark.parametrize("mode", ["softmax_renorm", "sigmoid"])
def test_lane_router_near_ties_take_the_exact_pass(k, E, mode, monkeypatch):
    """Values that the lane kernel's 32-bit entries cannot tell apart (the same
    top 24 bits of the order key) must still be picked in the exact order:
    the kernel detects them and selects those tokens again on full keys."""
    score, renorm = MODES[mode]
    logits = _near_tie_logits(1500, E, seed=5 + k + E).cuda()
    a = _router_outputs(logits, k, score, renorm, "lane", monkeypatch)
    b = _router_outputs(logits, k, score, renorm, "warp", monkeypatch)
    for n in b:
        assert torch.equal(a[n].view(torch.uint8), b[n].view(torch.uint8)), n
    # and against the oracle's picks
    import oracle
    r = oracle.router_topk(logits.cpu().numpy(), k, score, renorm)
    assert np.array_equal(a["topk_idx"].cpu().numpy(), r["topk_idx"])


@pytest.mark.parametrize("mode", ["softmax_renorm", "sigmoid", "sigmoid_renorm"])
def test_lane_router_degenerate_values_bias_and_scaling(mode, monkeypatch):
    score, renorm = MODES[mode]
    g_ = torch.Generator().manual_seed(41)
    logits = torch.round(torch.randn((700, 128), generator=g_) * 2) / 2      # many exact ties
    logits[0, 0] = float("nan")
    logits[1, 77] = float("nan")
    logits[2] = float("-inf")
    logits[3] = -0.0
    logits[3, 100] = 0.0
    logits[4, :120] = float("nan")
    logits = logits.cuda()
    bias = (torch.randn(128, generator=g_) * 0.3).cuda() if score == 1 else None
    a = _router_outputs(logits, 8, score, renorm, "lane", monkeypatch, bias=bias, scaling=1.5)
    b = _router_outputs(logits, 8, score, renorm, "warp", monkeypatch, bias=bias, scaling=1.5)
    for n in b:
        assert torch.equal(a[n].view(torch.uint8), b[n].view(torch.uint8)), n


def test_lane_router_ranks_drive_the_same_dispatch(monkeypatch):
    """The fused layer permutes with the router's per-block ranks: the lane
    kernel's ranks give the same permutation and output bits."""
    import routing_grouped_gemm_score_b200 as m
    w = wl.WORKLOADS["qwen3_30b_a3b"].scaled(T=1500, H=256, I=128, E=64)
    d = wl.make_inputs(w, "cuda")
    res = {}
    for kernel in ("lane", "warp"):
        helpers.force_kernels(router=kernel)
        out, st = m.moe_layer_forward(d["logits"], d["x"], d["w_gate_up"], d["w_down"], w.k,
                                      save_for_backward=True)
        torch.cuda.synchronize()
        assert m.moe_get_device_status() == 0
        res[kernel] = (out.clone(), st["row_of"].clone(), st["x_perm"].clone(), st["offsets"].clone())
    for a, b in zip(res["lane"], res["warp"]):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
