"""Full-size parity: every workload at its full shape, through the call the
benchmark times (moe_layer_forward, and moe_grouped_mlp_backward for the
training workload). Routing is compared on every token. Layer outputs and
gradients are compared on sampled tokens and experts, which the oracle
computes one by one.

Shapes: Mixtral-8x7B (T=4096, H=4096, I=14336, E=8, k=2), Qwen3-30B-A3B
(T=4096, H=2048, I=768, E=128, k=8, forward and backward), Llama-4-17Bx16E
(T=8192, H=5120, I=8192, E=16, k=1, sigmoid, shared expert), and the skewed
sweep at the Qwen3 shape (T = 1, 8, 64, 16384; 16 dead experts), with the
tie case (T=64, logits in multiples of 0.5).
"""
import numpy as np
import pytest
import torch

import helpers
import oracle
import workloads as wl
from helpers import assert_close, assert_close_flips, assert_equal, bf16_round_np, bits, require_gpu

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def sample_tokens(T, n=16, seed=0):
    rng = np.random.default_rng(seed)
    picks = {0, T - 1} | set(rng.integers(0, T, size=n).tolist())
    return np.array(sorted(picks), np.int64)


def run_forward(w, d, save=False):
    import routing_grouped_gemm_score_b200 as m
    opts = m.RouterOpts(w.score, w.renormalize)
    ws = m.LayerWorkspace(w.T, w.H, w.I, w.E, w.k, w.shared_expert)
    res = m.moe_layer_forward(d["logits"], d["x"], d["w_gate_up"], d["w_down"], w.k, opts,
                              d["shared_gate_up"], d["shared_down"], save_for_backward=save,
                              workspace=ws)
    torch.cuda.synchronize()
    assert m.moe_get_device_status() == 0
    return res


@pytest.mark.parametrize("name", ["mixtral_8x7b", "qwen3_30b_a3b", "llama4_17bx16e", "skew_t1",
                                  "skew_t8", "skew_t64", "skew_t16384", "tie_t64"])
def test_full_size_forward(name):
    w = wl.WORKLOADS[name]
    d = wl.make_inputs(w, "cuda")
    out, st = run_forward(w, d, save=True)
    logits = d["logits"].cpu().numpy()
    r = oracle.router_topk(logits, w.k, w.score, w.renormalize, with_map=False)
    assert_equal(st["topk_idx"], r["topk_idx"], f"{name}: topk_idx")
    assert_equal(st["counts"], r["counts"], f"{name}: counts")
    assert_equal(st["offsets"], r["offsets"], f"{name}: offsets")
    np.testing.assert_allclose(st["topk_prob"].cpu().numpy(), r["topk_prob"], rtol=1e-6, atol=0)
    sorted_token, row_of = oracle.dispatch(r["topk_idx"], r["offsets"], w.E)
    assert_equal(st["row_of"], row_of, f"{name}: row_of")
    tokens = sample_tokens(w.T)
    ref = oracle.moe_forward_tokens(
        bits(d["x"]), logits, bits(d["w_gate_up"]), bits(d["w_down"]), w.k, tokens=tokens,
        score=w.score, renormalize=w.renormalize,
        shared_gu_bits=None if d["shared_gate_up"] is None else bits(d["shared_gate_up"][0]),
        shared_d_bits=None if d["shared_down"] is None else bits(d["shared_down"][0]))
    assert_close_flips(out[torch.from_numpy(tokens).cuda()], ref,
                       helpers.forward_terms(w, d, tokens, logits), f"{name}: out rows {tokens.tolist()}")


def _assignment_terms(x_row, e, p, dout_row, wgu, wd, wgu_f, wd_f):
    """One assignment's stored bf16 values (oracle) and its gradient pieces,
    for the one-flip allowance of the backward comparison."""
    y, g, u, h = oracle.expert_mlp(x_row[None], wgu[e], wd[e], True, True)
    dy = bf16_round_np((np.float32(p) * oracle.bits_to_float(dout_row).astype(np.float32)).astype(np.float64))
    gb, ub = bf16_round_np(g[0]), bf16_round_np(u[0])
    dh = dy @ wd_f[e].T
    sg = 1.0 / (1.0 + np.exp(-gb))
    dgu = np.concatenate([dh * ub * (sg + gb * sg * (1 - sg)), dh * gb * sg])
    dxp = dgu @ wgu_f[e].T
    return y[0], h[0], dy, dgu, dxp


def test_full_size_backward_sampled():
    """Qwen3-30B-A3B fwd+bwd at full size: dx and dprob on sampled tokens,
    dW_down and dW_gate_up of the busiest expert and of one more."""
    import routing_grouped_gemm_score_b200 as m
    w = wl.WORKLOADS["qwen3_30b_a3b"]
    d = wl.make_inputs(w, "cuda", with_dout=True)
    out, st = run_forward(w, d, save=True)
    gr = m.moe_grouped_mlp_backward(d["dout"], st, d["w_gate_up"], d["w_down"])
    torch.cuda.synchronize()
    assert m.moe_get_device_status() == 0
    logits = d["logits"].cpu().numpy()
    r = oracle.router_topk(logits, w.k, with_map=False)
    assert_equal(st["topk_idx"], r["topk_idx"], "topk_idx")
    x, wgu, wd, dout = bits(d["x"]), bits(d["w_gate_up"]), bits(d["w_down"]), bits(d["dout"])

    class _F(dict):        # float64 copies of the expert weights, made on first use
        def __init__(self, src):
            super().__init__()
            self.src = src

        def __missing__(self, e):
            self[e] = oracle.bits_to_float(self.src[e])
            return self[e]
    wgu_f, wd_f = _F(wgu), _F(wd)

    # tokens: dx and dprob
    tokens = sample_tokens(w.T, n=12, seed=1)
    ref = oracle.moe_backward(x, r["topk_idx"], r["topk_prob"], wgu, wd, dout, tokens=tokens,
                              want=("dx", "dprob"))
    t_dx = np.zeros((len(tokens), w.H))
    t_dp = np.zeros((len(tokens), w.k))
    for n, t in enumerate(tokens):
        for j in range(w.k):
            e, p = int(r["topk_idx"][t, j]), r["topk_prob"][t, j]
            y, h, dy, dgu, dxp = _assignment_terms(x[t], e, p, dout[t], wgu, wd, wgu_f, wd_f)
            t_dx[n] += np.abs(dxp)
            t_dp[n, j] = np.abs(oracle.bits_to_float(dout[t]) * y).max()
    tk = torch.from_numpy(tokens).cuda()
    assert_close_flips(gr["dx"][tk], ref["dx"], t_dx, "dx (sampled tokens)")
    assert_close_flips(gr["dprob"][tk], ref["dprob"], t_dp, "dprob (sampled tokens)")

    # experts: dW of the busiest one and of one picked at random
    counts = r["counts"]
    experts = [int(np.argmax(counts)), int(np.random.default_rng(2).integers(0, w.E))]
    for e in experts:
        ge = oracle.moe_backward(x, r["topk_idx"], r["topk_prob"], wgu, wd, dout, only_expert=e,
                                 want=("dw_gate_up", "dw_down"))
        t_wd = np.zeros((w.I, w.H))
        t_wgu = np.zeros((w.H, 2 * w.I))
        for t, j in zip(*np.nonzero(r["topk_idx"] == e)):
            y, h, dy, dgu, dxp = _assignment_terms(x[t], e, r["topk_prob"][t, j], dout[t], wgu, wd,
                                                   wgu_f, wd_f)
            np.maximum(t_wd, np.outer(np.abs(h), np.abs(dy)), out=t_wd)
            np.maximum(t_wgu, np.outer(np.abs(oracle.bits_to_float(x[t])), np.abs(dgu)), out=t_wgu)
        assert_close_flips(gr["dw_down"][e], ge["dw_down"][0], t_wd, f"dw_down[{e}]")
        assert_close_flips(gr["dw_gate_up"][e], ge["dw_gate_up"][0], t_wgu, f"dw_gate_up[{e}]")
