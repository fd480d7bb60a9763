"""Pins of the oracle's expert MLP, grouped loop and layer forward.

Transformer Engine "Mixture of Experts": sections Grouped GEMM (the per-expert
loop and the grouped call give the same outputs), Grouped MLP (FC1, SwiGLU,
FC2; weights folded before FC2), Token probabilities (weights applied exactly
once; scaling the input of a nonlinear expert differs). te_mixtral.py
_expert_ffn: gate and up are the two halves of FC1's output.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import workloads as wl


def small(name="tiny", **kw):
    w = wl.WORKLOADS[name].scaled(**kw)
    d = wl.make_inputs(w)
    return w, d


def dense_swiglu_torch(x, wgu, wd, round_bf16):
    """A dense SwiGLU MLP from torch primitives, in fp64: the special case
    the layer reduces to with one expert."""
    x64, wgu64, wd64 = x.double(), wgu.double(), wd.double()
    I = wd.shape[0]
    h = F.silu(x64 @ wgu64[:, :I]) * (x64 @ wgu64[:, I:])
    if round_bf16:
        h = h.float().to(torch.bfloat16).double()
    y = h @ wd64
    if round_bf16:
        y = y.float().to(torch.bfloat16).double()
    return y.numpy()


@pytest.mark.parametrize("round_bf16", [False, True])
def test_single_expert_is_a_dense_swiglu_mlp(oracle_lib, round_bf16):
    # H != I != 2I, so a transposed operand or a swapped gate/up fails
    w, d = small(T=40, H=48, I=40, E=1, k=1)
    bits = oracle_lib.bf16_bits
    out = oracle_lib.moe_forward_tokens(bits(d["x"]), d["logits"].numpy(), bits(d["w_gate_up"]),
                                        bits(d["w_down"]), 1, round_bf16=round_bf16)
    ref = dense_swiglu_torch(d["x"], d["w_gate_up"][0], d["w_down"][0], round_bf16)
    if round_bf16:
        # torch rounds through fp32, so a rare double-rounding tie can move h or
        # y by one bf16 ulp: almost every element is equal, and none is further
        # than one ulp away
        assert np.mean(out == ref) > 0.99
        np.testing.assert_allclose(out, ref, rtol=2.0 ** -7, atol=1e-6)
    else:
        np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_identical_experts_reduce_to_dense_mlp(oracle_lib):
    """All experts equal and renormalised weights: sum_j p_j MLP(x) = MLP(x)."""
    w, d = small(T=30, H=32, I=24, E=6, k=3)
    wgu = d["w_gate_up"][:1].expand(6, -1, -1).contiguous()
    wd = d["w_down"][:1].expand(6, -1, -1).contiguous()
    bits = oracle_lib.bf16_bits
    out = oracle_lib.moe_forward_tokens(bits(d["x"]), d["logits"].numpy(), bits(wgu), bits(wd), 3,
                                        round_bf16=False)
    ref = dense_swiglu_torch(d["x"], wgu[0], wd[0], False)
    np.testing.assert_allclose(out, ref, rtol=1e-6, atol=1e-7)


def test_shared_expert_adds_a_dense_mlp(oracle_lib):
    w, d = small("llama4_17bx16e", T=20, H=32, I=16, E=4)
    bits = oracle_lib.bf16_bits
    kw = dict(score=w.score, renormalize=w.renormalize, round_bf16=False)
    routed = oracle_lib.moe_forward_tokens(bits(d["x"]), d["logits"].numpy(), bits(d["w_gate_up"]),
                                           bits(d["w_down"]), 1, **kw)
    both = oracle_lib.moe_forward_tokens(bits(d["x"]), d["logits"].numpy(), bits(d["w_gate_up"]),
                                         bits(d["w_down"]), 1, shared_gu_bits=bits(d["shared_gate_up"]),
                                         shared_d_bits=bits(d["shared_down"]), **kw)
    shared = dense_swiglu_torch(d["x"], d["shared_gate_up"][0], d["shared_down"][0], False)
    np.testing.assert_allclose(both - routed, shared, rtol=1e-9, atol=1e-12)


@pytest.mark.parametrize("name,T", [("tiny", None), ("skew_t64", None), ("qwen3_30b_a3b", 100)])
def test_per_token_definition_equals_grouped_path(oracle_lib, name, T):
    """Loop over tokens (no permutation) == permute -> per-expert loop -> combine."""
    kw = {} if T is None else {"T": T}
    w, d = small(name, **kw)
    if w.H > 256:
        w, d = small(name, H=128, I=64, **kw)
    bits = oracle_lib.bf16_bits
    x, wgu, wd = bits(d["x"]), bits(d["w_gate_up"]), bits(d["w_down"])
    logits = d["logits"].numpy()
    r = oracle_lib.router_topk(logits, w.k, score=w.score, renormalize=w.renormalize)
    st, row_of = oracle_lib.dispatch(r["topk_idx"], r["offsets"], w.E)
    y = oracle_lib.grouped_mlp(oracle_lib.gather_rows(x, st), r["offsets"], wgu, wd)
    out_grouped = oracle_lib.combine(y, row_of, r["topk_prob"])
    out_tokens = oracle_lib.moe_forward_tokens(x, logits, wgu, wd, w.k, score=w.score,
                                               renormalize=w.renormalize)
    np.testing.assert_allclose(out_grouped, out_tokens, rtol=1e-12, atol=1e-13)


def test_empty_expert_contributes_nothing(oracle_lib):
    w, d = small(T=16, H=32, I=16, E=4, k=1)
    logits = d["logits"].numpy().copy()
    logits[:, 2] = -1e4                               # expert 2 gets no token
    bits = oracle_lib.bf16_bits
    r = oracle_lib.router_topk(logits, 1)
    assert r["counts"][2] == 0
    x, wgu, wd = bits(d["x"]), bits(d["w_gate_up"]), bits(d["w_down"])
    st, _ = oracle_lib.dispatch(r["topk_idx"], r["offsets"], 4)
    y1 = oracle_lib.grouped_mlp(oracle_lib.gather_rows(x, st), r["offsets"], wgu, wd)
    wgu2 = wgu.copy()
    wgu2[2] = 0x7FC0                                  # NaN weights of the empty expert
    y2 = oracle_lib.grouped_mlp(oracle_lib.gather_rows(x, st), r["offsets"], wgu2, wd)
    np.testing.assert_array_equal(y1, y2)


def test_input_scaling_is_not_output_weighting(oracle_lib):
    """Scaling the input of a nonlinear expert by p is not p times its output."""
    w, d = small(T=8, H=32, I=16, E=1, k=1)
    bits = oracle_lib.bf16_bits
    x = d["x"]
    p = 0.3
    xs = (x.float() * p).to(torch.bfloat16)
    y_in = oracle_lib.expert_mlp(bits(xs), bits(d["w_gate_up"][0]), bits(d["w_down"][0]), False)
    y_out = p * oracle_lib.expert_mlp(bits(x), bits(d["w_gate_up"][0]), bits(d["w_down"][0]), False)
    assert np.abs(y_in - y_out).max() > 1e-2 * np.abs(y_out).max()


def test_weight_folds_before_fc2(oracle_lib):
    """p (h W2) = (p h) W2: the weight may be applied before the bias-free FC2."""
    w, d = small(T=12, H=32, I=16, E=1, k=1)
    bits = oracle_lib.bf16_bits
    y, g, u, h = oracle_lib.expert_mlp(bits(d["x"]), bits(d["w_gate_up"][0]), bits(d["w_down"][0]),
                                       False, want_intermediates=True)
    wd = oracle_lib.bits_to_float(bits(d["w_down"][0]))
    p = np.linspace(0.1, 0.9, 12)[:, None]
    np.testing.assert_allclose(p * y, (p * h) @ wd, rtol=1e-12, atol=1e-14)
    # and h itself is silu(gate) * up of the two halves of FC1
    x = oracle_lib.bits_to_float(bits(d["x"]))
    wgu = oracle_lib.bits_to_float(bits(d["w_gate_up"][0]))
    np.testing.assert_allclose(g, x @ wgu[:, :16], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(u, x @ wgu[:, 16:], rtol=1e-12, atol=1e-13)
