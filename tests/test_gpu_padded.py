"""Padded dispatch and ScaledSwiGLU on the GPU (Transformer Engine "Mixture of
Experts": Token permutation, Padding and alignment; Grouped MLP, ScaledSwiGLU),
through the C ABI, against the oracle: the padded permutation bit-exact, and
the layer computed through padded blocks, with the weights applied either in
combine or before FC2, within the layer's bf16 bound."""
import numpy as np
import pytest
import torch

import helpers
import oracle
import workloads as wl
from helpers import assert_equal, bits, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


CASES = {
    "qwen3_a16": (wl.WORKLOADS["qwen3_30b_a3b"].scaled(T=1000, H=256, I=128, E=32), 16),
    "mixtral_a256": (wl.WORKLOADS["mixtral_8x7b"].scaled(T=700, H=512, I=256), 256),
    "skew_a128": (wl.WORKLOADS["skew_t64"].scaled(H=256, I=192), 128),
    "tiny_a3": (wl.WORKLOADS["tiny"], 3),
    "tiny_a1": (wl.WORKLOADS["tiny"], 1),
}


def routed(w):
    import routing_grouped_gemm_score_b200 as m
    d = wl.make_inputs(w, "cuda")
    r = m.moe_router_topk(d["logits"], w.k, m.RouterOpts(w.score, w.renormalize))
    return m, d, r


@pytest.mark.parametrize("name", list(CASES))
def test_padded_dispatch_matches_the_oracle(name):
    w, align = CASES[name]
    m, d, r = routed(w)
    p = m.moe_permute_padded(d["x"], r["topk_idx"], r["offsets"], align, r["topk_prob"])
    torch.cuda.synchronize()
    assert m.moe_get_device_status() == 0
    padded, st, row_of = oracle.dispatch_padded(r["topk_idx"].cpu().numpy(), r["offsets"].cpu().numpy(), w.E,
                                                align)
    n = int(padded[-1])
    assert_equal(p["padded_offsets"], padded, "padded_offsets")
    assert_equal(p["sorted_token"][:n], st, "sorted_token")
    assert_equal(p["row_of"], row_of, "row_of")
    assert_equal(p["x_perm"][:n].view(torch.int16).cpu().numpy().view(np.uint16),
                 oracle.gather_rows(bits(d["x"]), st), "x_perm (pad rows zero)")
    prob = p["prob_perm"][:n].cpu().numpy()
    expect = np.zeros(n, np.float32)
    expect[row_of.ravel()] = r["topk_prob"].cpu().numpy().ravel()
    assert np.array_equal(prob.view(np.uint32), expect.view(np.uint32)), "prob_perm"
    # the bound on rows holds
    assert n <= m.moe_permute_padded_max_rows(w.T, w.E, w.k, align)


@pytest.mark.parametrize("tiles", ["auto", "pair", "swap"])
@pytest.mark.parametrize("scaled", [False, True])
@pytest.mark.parametrize("name", ["qwen3_a16", "mixtral_a256", "tiny_a3"])
def test_layer_through_padded_blocks(name, scaled, tiles):
    """permute_padded -> grouped MLP on the padded blocks -> combine, with the
    weights in combine, or (ScaledSwiGLU) applied to h before FC2 with an
    unweighted combine; both against the oracle's per-token layer."""
    helpers.force_kernels(gemm_tiles=tiles)
    w, align = CASES[name]
    m, d, r = routed(w)
    p = m.moe_permute_padded(d["x"], r["topk_idx"], r["offsets"], align, r["topk_prob"])
    n = int(p["padded_offsets"][-1])
    mlp = m.moe_grouped_mlp(p["x_perm"][:n], p["padded_offsets"], d["w_gate_up"], d["w_down"],
                            row_scale=p["prob_perm"][:n] if scaled else None)
    out = m.moe_unpermute_combine(mlp["y_perm"], p["row_of"], None if scaled else r["topk_prob"])
    torch.cuda.synchronize()
    assert m.moe_get_device_status() == 0
    ref = oracle.moe_forward_tokens(bits(d["x"]), d["logits"].cpu().numpy(), bits(d["w_gate_up"]),
                                    bits(d["w_down"]), w.k, score=w.score, renormalize=w.renormalize)
    terms = helpers.lazy_forward_terms(w, d, np.arange(w.T))
    helpers.assert_close_flips(out, ref, terms, f"{name} scaled={scaled}")
    # the pad rows' outputs are zero rows (zero inputs, no bias)
    y = mlp["y_perm"].float().cpu().numpy()
    pad = p["sorted_token"][:n].cpu().numpy() < 0
    assert np.all(y[pad] == 0)
