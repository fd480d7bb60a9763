"""Permute folded into the gate_up GEMM (Transformer Engine "Mixture of
Experts", Token permutation: the permutation can be folded into the copy that
feeds the expert computation). Without a requested x_perm, on single-CTA tiles,
the layer forward gathers the GEMM's A rows from x by token id instead of
writing and re-reading a permuted copy. The tile contents are the same bf16
values either way and the MMA order is unchanged, so the output must be
bit-identical to the path through x_perm, and match the oracle's per-token
layer like it."""
import numpy as np
import pytest
import torch

import helpers
import oracle
import workloads as wl
from helpers import bits, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


CASES = {
    "qwen3_small": wl.WORKLOADS["qwen3_30b_a3b"].scaled(T=1000, H=256, I=128, E=32),
    # three K slices, 64-wide h, ragged expert blocks
    "small_k": wl.WORKLOADS["qwen3_30b_a3b"].scaled(T=333, H=192, I=64, E=16),
    "skew": wl.WORKLOADS["skew_t64"].scaled(H=256, I=192),
    "tiny": wl.WORKLOADS["tiny"],
    "tie": wl.WORKLOADS["tie_t64"].scaled(H=128, I=128),
    "wide_h": wl.WORKLOADS["qwen3_30b_a3b"].scaled(T=300, H=2112, I=256, E=8),
    "qwen3_full": wl.WORKLOADS["qwen3_30b_a3b"],
}


def forward(w, d, gather, monkeypatch):
    import routing_grouped_gemm_score_b200 as m
    helpers.force_kernels(gemm_tiles="single")
    helpers.force_kernels(fold_permute=gather)
    out = m.moe_layer_forward(d["logits"], d["x"], d["w_gate_up"], d["w_down"], w.k,
                              m.RouterOpts(w.score, w.renormalize), d["shared_gate_up"], d["shared_down"])
    torch.cuda.synchronize()
    assert m.moe_get_device_status() == 0
    return out


@pytest.mark.parametrize("name", list(CASES))
def test_gathered_rows_give_the_same_bits_as_x_perm(name, monkeypatch):
    w = CASES[name]
    d = wl.make_inputs(w, "cuda")
    a = forward(w, d, True, monkeypatch)
    b = forward(w, d, False, monkeypatch)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("name", ["qwen3_small", "small_k", "skew"])
def test_gathered_layer_matches_the_oracle(name, monkeypatch):
    w = CASES[name]
    d = wl.make_inputs(w, "cuda")
    out = forward(w, d, True, monkeypatch)
    ref = oracle.moe_forward_tokens(bits(d["x"]), d["logits"].cpu().numpy(), bits(d["w_gate_up"]),
                                    bits(d["w_down"]), w.k, score=w.score, renormalize=w.renormalize)
    helpers.assert_close_flips(out, ref, helpers.lazy_forward_terms(w, d, np.arange(w.T)), name)
