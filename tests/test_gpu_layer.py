"""The fused layer (moe_layer_forward) and the grouped-MLP backward on the
GPU, through the C ABI, against the oracle's per-token definition of the
layer and its chain-rule gradients (Transformer Engine "Mixture of Experts",
Example: MoE layer on a single device)."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from helpers import assert_close, assert_equal, bits, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def layer(w, d, save=False):
    import routing_grouped_gemm_score_b200 as m
    opts = m.RouterOpts(w.score, w.renormalize)
    res = m.moe_layer_forward(d["logits"], d["x"], d["w_gate_up"], d["w_down"], w.k, opts,
                              d["shared_gate_up"], d["shared_down"], save_for_backward=save)
    torch.cuda.synchronize()
    assert m.moe_get_device_status() == 0
    return res


def oracle_out(w, d, tokens=None):
    return oracle.moe_forward_tokens(
        bits(d["x"]), d["logits"].cpu().numpy(), bits(d["w_gate_up"]), bits(d["w_down"]), w.k,
        tokens=tokens, score=w.score, renormalize=w.renormalize,
        shared_gu_bits=None if d["shared_gate_up"] is None else bits(d["shared_gate_up"][0]),
        shared_d_bits=None if d["shared_down"] is None else bits(d["shared_down"][0]))


SMALL = {
    "tiny": wl.WORKLOADS["tiny"],
    "qwen3_small": wl.WORKLOADS["qwen3_30b_a3b"].scaled(T=256, H=256, I=128, E=32),
    "llama4_small": wl.WORKLOADS["llama4_17bx16e"].scaled(T=300, H=256, I=256, E=16),
    "skew_small": wl.WORKLOADS["skew_t64"].scaled(H=256, I=192),
    "tie_small": wl.WORKLOADS["tie_t64"].scaled(H=128, I=128),
    "mixtral_small": wl.WORKLOADS["mixtral_8x7b"].scaled(T=512, H=512, I=512),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_layer_forward_matches_per_token_definition(name):
    w = SMALL[name]
    d = wl.make_inputs(w, "cuda")
    out = layer(w, d)
    assert_close(out, oracle_out(w, d), f"{name}: out")


def test_layer_forward_saved_state_and_empty_batch():
    import routing_grouped_gemm_score_b200 as m
    w = SMALL["qwen3_small"]
    d = wl.make_inputs(w, "cuda")
    out, st = layer(w, d, save=True)
    r = oracle.router_topk(d["logits"].cpu().numpy(), w.k)
    assert_equal(st["topk_idx"], r["topk_idx"], "topk_idx")
    assert_equal(st["offsets"], r["offsets"], "offsets")
    sorted_token, row_of = oracle.dispatch(r["topk_idx"], r["offsets"], w.E)
    assert_equal(st["row_of"], row_of, "row_of")
    assert_equal(st["x_perm"].view(torch.int16).cpu().numpy().view(np.uint16),
                 oracle.gather_rows(bits(d["x"]), sorted_token), "x_perm")
    empty = m.moe_layer_forward(d["logits"][:0], d["x"][:0], d["w_gate_up"], d["w_down"], w.k)
    assert empty.shape == (0, w.H)


@pytest.mark.parametrize("name", ["tiny", "qwen3_small", "skew_small", "mixtral_small"])
def test_backward_matches_oracle(name):
    import routing_grouped_gemm_score_b200 as m
    w = SMALL[name]
    d = wl.make_inputs(w, "cuda", with_dout=True)
    out, st = layer(w, d, save=True)
    gr = m.moe_grouped_mlp_backward(d["dout"], st, d["w_gate_up"], d["w_down"])
    torch.cuda.synchronize()
    assert m.moe_get_device_status() == 0
    ref = oracle.moe_backward(bits(d["x"]), st["topk_idx"].cpu().numpy(), st["topk_prob"].cpu().numpy(),
                              bits(d["w_gate_up"]), bits(d["w_down"]), bits(d["dout"]))
    assert_close(gr["dprob"], ref["dprob"], f"{name}: dprob")
    assert_close(gr["dx"], ref["dx"], f"{name}: dx")
    assert_close(gr["dw_down"], ref["dw_down"], f"{name}: dw_down")
    assert_close(gr["dw_gate_up"], ref["dw_gate_up"], f"{name}: dw_gate_up")
    counts = st["counts"].cpu().numpy()
    for e in np.nonzero(counts == 0)[0]:
        assert torch.all(gr["dw_down"][e] == 0) and torch.all(gr["dw_gate_up"][e] == 0)
