"""The fused layer (moe_layer_forward) and the grouped-MLP backward on the
GPU, through the C ABI, against the oracle's per-token definition of the
layer and its chain-rule gradients (Transformer Engine "Mixture of Experts",
Example: MoE layer on a single device)."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
import helpers
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
    # about 1000 rows per expert: the weight gradient streams B instead of
    # keeping each expert's rows in shared memory (more than 320 rows)
    "long_k": wl.WORKLOADS["mixtral_8x7b"].scaled(T=2048, H=256, I=192, E=4),
    # H and I multiples of 8 only (not of 32 or 64): partial column chunks everywhere
    "odd_dims": wl.WORKLOADS["qwen3_30b_a3b"].scaled(T=300, H=200, I=136, E=16),
    # at most 16 rows per expert: the swap-AB tiles of 16 token rows
    "t12": wl.WORKLOADS["tiny"].scaled(T=12),
    "odd_t12": wl.WORKLOADS["qwen3_30b_a3b"].scaled(T=12, H=200, I=136, E=16),
}


@pytest.mark.parametrize("tiles", ["auto", "single", "pair", "swap", "swap_unfused"])
@pytest.mark.parametrize("name", list(SMALL))
def test_layer_forward_matches_per_token_definition(name, tiles, monkeypatch):
    helpers.force_kernels(gemm_tiles=tiles)
    w = SMALL[name]
    d = wl.make_inputs(w, "cuda")
    out = layer(w, d)
    tokens = np.arange(w.T)
    helpers.assert_close_flips(out, oracle_out(w, d), helpers.lazy_forward_terms(w, d, tokens), f"{name}: out")


# every expert at most 64 rows (T <= 64): gate_up and down in one launch
FUSED_MLP = {
    "tiny": SMALL["tiny"],                       # 64-row token tiles, E = 8
    "skew_small": SMALL["skew_small"],           # T = 64 over 128 experts, 16 dead
    "t12": SMALL["t12"],                         # 16-row token tiles
    "odd_t12": SMALL["odd_t12"],                 # H = 200, I = 136: partial tiles
    "t1": wl.WORKLOADS["skew_t1"].scaled(H=256, I=192),
    "t8_shared": wl.WORKLOADS["skew_t8"].scaled(H=256, I=320, shared_expert=True),
}


@pytest.mark.parametrize("name", list(FUSED_MLP))
def test_fused_small_batch_mlp_is_bit_identical_to_two_launches(name):
    """For a small batch the layer can compute gate_up + SwiGLU and down in
    one launch (the down tiles wait for their expert's h through a device
    counter; forced here with "swap", which the library otherwise takes only
    when the gate_up tiles can fill the SMs). Each output element comes from
    the same tile arithmetic as on the two-launch path, so the output and the
    saved state agree bit for bit; the result is then also checked against
    the oracle."""
    w = FUSED_MLP[name]
    d = wl.make_inputs(w, "cuda")
    runs = []
    for tiles in ("swap", "swap_unfused", "swap", "auto"):
        helpers.force_kernels(gemm_tiles=tiles)
        out, st = layer(w, d, save=True)
        runs.append((out.clone(), {key: v.clone() for key, v in st.items()}))
    for out, st in runs[1:]:
        assert torch.equal(out.view(torch.int16), runs[0][0].view(torch.int16)), f"{name}: out"
        for key, v in st.items():
            a = runs[0][1][key]
            as_int = a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32)
            other = v.view(torch.int16) if v.dtype == torch.bfloat16 else v.view(torch.int32)
            assert torch.equal(as_int, other), f"{name}: {key}"
    tokens = np.arange(w.T)
    helpers.assert_close_flips(runs[0][0], oracle_out(w, d), helpers.lazy_forward_terms(w, d, tokens),
                               f"{name}: out (one launch)")


SHARED = {
    "llama4_small": SMALL["llama4_small"],
    "k4_shared": SMALL["qwen3_small"].scaled(k=4, shared_expert=True),
    "odd_dims_shared": SMALL["odd_dims"].scaled(shared_expert=True),
    # 12 tokens: the shared expert on swap-AB tiles, so the combine kernel runs
    "t12_shared": SMALL["odd_t12"].scaled(shared_expert=True),
}


@pytest.mark.parametrize("name", list(SHARED))
def test_combine_in_the_shared_expert_gemm(name):
    """With a shared expert on CTA-pair tiles the combine runs in that
    GEMM's epilogue: out[t] = bf16(s[t] + sum_j p[t,j] y[row_of[t,j]]), the
    shared output s in fp32. Checked against the oracle's shared expert (h
    rounded to bf16 as stored, its product unrounded) plus the GPU's stored
    routed rows, strictly; and the combine kernel's path (single tiles, s
    stored in bf16 first) against the same reference."""
    w = SHARED[name]
    helpers.force_kernels(gemm_tiles="auto")
    d = wl.make_inputs(w, "cuda")
    out, st = layer(w, d, save=True)
    f = oracle.bits_to_float
    sgu, sd = bits(d["shared_gate_up"][0]), bits(d["shared_down"][0])
    _, _, _, hs = oracle.expert_mlp(bits(d["x"]), sgu, sd, round_bf16=True, want_intermediates=True)
    shared = hs @ f(sd)
    y = f(bits(st["y_perm"]))
    row_of = st["row_of"].cpu().numpy()
    p = st["topk_prob"].cpu().numpy().astype(np.float64)
    ref = shared + sum(p[:, j:j + 1] * y[row_of[:, j]] for j in range(w.k))
    assert_close(out, ref, f"{name}: out, combine in the shared expert's GEMM")
    helpers.force_kernels(gemm_tiles="single")
    out2 = layer(w, d)
    assert_close(out2, ref, f"{name}: out, combine kernel after the stored shared output")


# T <= 8 is one token block: the router kernel also writes the offsets (no
# scan launch), and up to 64 KB of permuted rows (no permute launch; t8 has
# 8 x 8 rows of 512 B, t1_odd 8 rows of 400 B)
STATE = {"qwen3_small": SMALL["qwen3_small"],
         "t8": SMALL["qwen3_small"].scaled(T=8),
         "t1_odd": SMALL["odd_dims"].scaled(T=1)}


@pytest.mark.parametrize("name", list(STATE))
def test_layer_forward_saved_state_and_empty_batch(name):
    import routing_grouped_gemm_score_b200 as m
    w = STATE[name]
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


BWD = ["tiny", "qwen3_small", "skew_small", "mixtral_small", "long_k", "odd_dims", "odd_t12"]


def _oracle_backward(w, d, r):
    return oracle.moe_backward(bits(d["x"]), r["topk_idx"], r["topk_prob"], bits(d["w_gate_up"]),
                               bits(d["w_down"]), bits(d["dout"]))


@pytest.mark.parametrize("tiles", ["single", "pair"])
@pytest.mark.parametrize("name", BWD)
def test_backward_on_oracle_state(name, tiles):
    """The backward kernels fed with the oracle's own saved forward state, so
    both sides read identical bf16 inputs. dW_down and dprob then differ only
    in accumulation order; dW_gate_up and dx also carry the bf16 rounding of
    dg, du and each token row's dx, whose fp32 and fp64 pre-images can round
    apart (assert_close_flips)."""
    helpers.force_kernels(gemm_tiles=tiles)
    _check_backward_on_oracle_state(name, SMALL[name])


COMBINE_BWD = {
    "k1": wl.WORKLOADS["qwen3_30b_a3b"].scaled(T=160, H=192, I=128, E=16, k=1),
    "k3": wl.WORKLOADS["qwen3_30b_a3b"].scaled(T=150, H=192, I=128, E=8, k=3),
    "k8": wl.WORKLOADS["qwen3_30b_a3b"].scaled(T=256, H=2112, I=128, E=32),
    "k16": wl.WORKLOADS["qwen3_30b_a3b"].scaled(T=200, H=256, I=128, E=32, k=16),
}


@pytest.mark.parametrize("name", list(COMBINE_BWD))
def test_backward_combine_kernels(name):
    """The warp-per-token combine backward at k = 1, 3, 8 and 16; H = 2112 is
    not a multiple of the 64 chunks a warp covers per step."""
    _check_backward_on_oracle_state(name, COMBINE_BWD[name])


def _check_backward_on_oracle_state(name, w):
    import routing_grouped_gemm_score_b200 as m
    d = wl.make_inputs(w, "cuda", with_dout=True)
    r = oracle.router_topk(d["logits"].cpu().numpy(), w.k)
    s = helpers.oracle_saved_state(w, d, r)
    cu = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to(dt).cuda()
    state = {"topk_idx": cu(r["topk_idx"], torch.int32), "topk_prob": cu(r["topk_prob"], torch.float32),
             "offsets": cu(r["offsets"], torch.int32), "row_of": cu(s["row_of"], torch.int32),
             "x_perm": cu(s["x_perm"], torch.bfloat16),
             "gu": cu(np.concatenate([s["g"], s["u"]], axis=1), torch.bfloat16),
             "h": cu(s["h"], torch.bfloat16), "y_perm": cu(s["y"], torch.bfloat16)}
    gr = m.moe_grouped_mlp_backward(d["dout"], state, d["w_gate_up"], d["w_down"])
    torch.cuda.synchronize()
    assert m.moe_get_device_status() == 0
    ref = _oracle_backward(w, d, r)
    terms = helpers.flip_terms(w, d, r, s)
    assert_close(gr["dprob"], ref["dprob"], f"{name}: dprob")
    assert_close(gr["dw_down"], ref["dw_down"], f"{name}: dw_down")
    helpers.assert_close_flips(gr["dw_gate_up"], ref["dw_gate_up"], terms["dw_gate_up"],
                               f"{name}: dw_gate_up")
    helpers.assert_close_flips(gr["dx"], ref["dx"], terms["dx"], f"{name}: dx")


@pytest.mark.parametrize("name", BWD)
def test_backward_end_to_end(name):
    """The GPU forward, then the GPU backward on the state it saved. The saved
    state ([g | u], h, y) is checked against the oracle's forward, strictly
    within the bound; the gradients against the oracle's chain rule on that
    same state (the inputs the backward call was given). dprob and dW_down
    read only that state: strict. dx and dW_gate_up also carry the backward's
    own bf16 roundings of [dg | du] and of each permuted row's dx, whose fp32
    and fp64 pre-images can round apart (one-flip allowance, counted)."""
    import routing_grouped_gemm_score_b200 as m
    w = SMALL[name]
    d = wl.make_inputs(w, "cuda", with_dout=True)
    out, st = layer(w, d, save=True)
    gr = m.moe_grouped_mlp_backward(d["dout"], st, d["w_gate_up"], d["w_down"])
    torch.cuda.synchronize()
    assert m.moe_get_device_status() == 0
    r = oracle.router_topk(d["logits"].cpu().numpy(), w.k)
    assert_equal(st["topk_idx"], r["topk_idx"], "topk_idx")
    s = helpers.oracle_saved_state(w, d, r)
    assert_equal(st["row_of"], s["row_of"], f"{name}: row_of")
    assert_close(st["gu"][:, :w.I], s["g"], f"{name}: saved g")
    assert_close(st["gu"][:, w.I:], s["u"], f"{name}: saved u")
    assert_close(st["h"], s["h"], f"{name}: saved h")
    assert_close(st["y_perm"], s["y"], f"{name}: saved y")
    gpu_state = {"row_of": st["row_of"].cpu().numpy(), "gu": bits(st["gu"]), "h": bits(st["h"]),
                 "y": bits(st["y_perm"])}
    ref = oracle.moe_backward(bits(d["x"]), r["topk_idx"], r["topk_prob"], bits(d["w_gate_up"]),
                              bits(d["w_down"]), bits(d["dout"]), state=gpu_state)
    assert_close(gr["dprob"], ref["dprob"], f"{name}: dprob")
    assert_close(gr["dw_down"], ref["dw_down"], f"{name}: dw_down")
    terms = helpers.flip_terms(w, d, r, s)
    helpers.assert_close_flips(gr["dw_gate_up"], ref["dw_gate_up"], terms["dw_gate_up"], f"{name}: dw_gate_up")
    helpers.assert_close_flips(gr["dx"], ref["dx"], terms["dx"], f"{name}: dx")
    counts = st["counts"].cpu().numpy()
    for e in np.nonzero(counts == 0)[0]:
        assert torch.all(gr["dw_down"][e] == 0) and torch.all(gr["dw_gate_up"][e] == 0)


@pytest.mark.parametrize("name", ["qwen3_small", "llama4_small"])
def test_layer_in_cuda_graph(name):
    """A whole step captured once in a CUDA graph and replayed on new inputs
    gives bit-identical results to the same calls run eagerly: the calls
    allocate nothing, never sync, and take every buffer from the caller."""
    import routing_grouped_gemm_score_b200 as m
    w = SMALL[name]
    train = name == "qwen3_small"
    d = wl.make_inputs(w, "cuda", with_dout=True)
    opts = m.RouterOpts(w.score, w.renormalize)
    ws = m.LayerWorkspace(w.T, w.H, w.I, w.E, w.k, w.shared_expert, backward=train)
    logits, x, dout = d["logits"].clone(), d["x"].clone(), d["dout"].clone()
    out = torch.empty((w.T, w.H), dtype=torch.bfloat16, device="cuda")
    if train:
        _, state = m.moe_layer_forward(logits, x, d["w_gate_up"], d["w_down"], w.k, opts,
                                       save_for_backward=True, workspace=ws, out=out)
        grads = m.moe_grouped_mlp_backward(dout, state, d["w_gate_up"], d["w_down"], ws)
    else:   # forward only: keep just the routing outputs
        state = {"topk_idx": torch.empty((w.T, w.k), dtype=torch.int32, device="cuda"),
                 "topk_prob": torch.empty((w.T, w.k), dtype=torch.float32, device="cuda"),
                 "counts": torch.empty(w.E, dtype=torch.int32, device="cuda"),
                 "offsets": torch.empty(w.E + 1, dtype=torch.int32, device="cuda")}
        grads = None

    def step():
        m.moe_layer_forward(logits, x, d["w_gate_up"], d["w_down"], w.k, opts, d["shared_gate_up"],
                            d["shared_down"], save_for_backward=train, workspace=ws, out=out, state=state)
        if train:
            m.moe_grouped_mlp_backward(dout, state, d["w_gate_up"], d["w_down"], ws, grads)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()                       # warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    # new inputs in the captured buffers, replay, then the eager reference
    g2 = torch.Generator(device="cuda").manual_seed(99)
    logits.copy_(torch.randn(logits.shape, generator=g2, device="cuda"))
    x.copy_(torch.randn(x.shape, generator=g2, device="cuda").to(torch.bfloat16))
    dout.copy_(torch.randn(dout.shape, generator=g2, device="cuda").to(torch.bfloat16))
    g.replay()
    torch.cuda.synchronize()
    assert m.moe_get_device_status() == 0
    got = {"out": out.clone(), "topk_idx": state["topk_idx"].clone()}
    if train:
        got.update({k: v.clone() for k, v in grads.items()})
    step()
    torch.cuda.synchronize()
    assert torch.equal(got["out"], out)
    assert torch.equal(got["topk_idx"], state["topk_idx"])
    if train:
        for k, v in grads.items():
            assert torch.equal(got[k], v), k
    del g
