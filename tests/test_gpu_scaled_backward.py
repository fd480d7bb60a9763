"""The ScaledSwiGLU backward on the GPU (Transformer Engine "Mixture of
Experts": Grouped MLP with the routing weight applied to the activation before
FC2, and an unweighted Token combine), through the C ABI, against the oracle's
chain rule on the state the GPU forward saved.

The forward runs permute_padded -> moe_grouped_mlp_scaled (saving [g | u] and
the scaled h); the backward call gets that state. dprob and dW_down read only
the state and dout: strict. dx and dW_gate_up also carry the backward's own bf16
roundings of [dg | du] and of each permuted row's dx, whose fp32 and fp64
pre-images can round apart (one-flip allowance, counted)."""
import numpy as np
import pytest
import torch

import helpers
import oracle
import workloads as wl
from helpers import assert_close, bits, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


CASES = {
    "qwen3_a16": (wl.WORKLOADS["qwen3_30b_a3b"].scaled(T=1000, H=256, I=128, E=32), 16),
    "mixtral_a256": (wl.WORKLOADS["mixtral_8x7b"].scaled(T=700, H=512, I=256), 256),
    "mixtral_unpadded": (wl.WORKLOADS["mixtral_8x7b"].scaled(T=700, H=512, I=256), 1),
    # I = 136: the last 64-column group of dprob's partial sums holds 8 columns
    "odd_dims_a8": (wl.WORKLOADS["qwen3_30b_a3b"].scaled(T=300, H=200, I=136, E=16), 8),
    "skew_a128": (wl.WORKLOADS["skew_t64"].scaled(H=256, I=192), 128),
    "tiny_a3": (wl.WORKLOADS["tiny"], 3),
}


def scaled_forward(w, align):
    import routing_grouped_gemm_score_b200 as m
    d = wl.make_inputs(w, "cuda", with_dout=True)
    r = m.moe_router_topk(d["logits"], w.k, m.RouterOpts(w.score, w.renormalize))
    p = m.moe_permute_padded(d["x"], r["topk_idx"], r["offsets"], align, r["topk_prob"])
    n = int(p["padded_offsets"][-1])
    rows = {"x_perm": p["x_perm"][:n], "sorted_token": p["sorted_token"][:n], "prob_perm": p["prob_perm"][:n],
            "offsets": p["padded_offsets"], "row_of": p["row_of"]}
    mlp = m.moe_grouped_mlp_scaled(rows["x_perm"], rows["offsets"], d["w_gate_up"], d["w_down"],
                                   rows["prob_perm"], save=True)
    rows["gu"], rows["h"] = mlp["gu"], mlp["h"]
    return m, d, r, rows


def scaled_backward(m, d, rows):
    return m.moe_grouped_mlp_scaled_backward(d["dout"], rows["row_of"], rows["sorted_token"], rows["prob_perm"],
                                             rows["offsets"], rows["x_perm"], rows["gu"], rows["h"],
                                             d["w_gate_up"], d["w_down"])


def scaled_flip_terms(w, d, topk_prob, rows):
    """Largest single product per dx and dW_gate_up element (see
    assert_close_flips), from the GPU's saved rows: dy = dout of the row's
    token, ds = p * dh, [dg | du] from ds and the saved g, u."""
    f = oracle.bits_to_float
    wgu, wd, dout = f(bits(d["w_gate_up"])), f(bits(d["w_down"])), f(bits(d["dout"]))
    st = rows["sorted_token"].cpu().numpy()
    row_of = rows["row_of"].cpu().numpy()
    offs = rows["offsets"].cpu().numpy()
    xp = f(bits(rows["x_perm"]))
    gu = f(bits(rows["gu"]))
    A, I = len(st), w.I
    p_row = np.zeros(A)
    p_row[row_of.ravel()] = topk_prob.ravel()
    dy = np.zeros((A, w.H))
    dy[st >= 0] = dout[st[st >= 0]]
    t_dwgu = np.zeros((w.E, w.H, 2 * I))
    dxp = np.zeros((A, w.H))
    for e in range(w.E):
        a, b = offs[e], offs[e + 1]
        if b == a:
            continue
        g, u = gu[a:b, :I], gu[a:b, I:]
        sg = 1.0 / (1.0 + np.exp(-g))
        ds = p_row[a:b, None] * (dy[a:b] @ wd[e].T)
        dgu = np.concatenate([ds * u * (sg + g * sg * (1 - sg)), ds * g * sg], axis=1)
        dxp[a:b] = np.abs(dgu @ wgu[e].T)
        xe, dgu = np.abs(xp[a:b]), np.abs(dgu)
        for rr in range(b - a):
            np.maximum(t_dwgu[e], np.outer(xe[rr], dgu[rr]), out=t_dwgu[e])
    return dict(dw_gate_up=t_dwgu, dx=dxp[row_of].sum(axis=1))


@pytest.mark.parametrize("tiles", ["single", "pair"])
@pytest.mark.parametrize("name", list(CASES))
def test_scaled_backward_on_saved_state(name, tiles):
    w, align = CASES[name]
    m, d, r, rows = scaled_forward(w, align)
    helpers.force_kernels(gemm_tiles=tiles)
    gr = scaled_backward(m, d, rows)
    torch.cuda.synchronize()
    assert m.moe_get_device_status() == 0
    topk_idx, topk_prob = r["topk_idx"].cpu().numpy(), r["topk_prob"].cpu().numpy()
    state = {"row_of": rows["row_of"].cpu().numpy(), "gu": bits(rows["gu"]), "h": bits(rows["h"])}
    ref = oracle.moe_backward(bits(d["x"]), topk_idx, topk_prob, bits(d["w_gate_up"]), bits(d["w_down"]),
                              bits(d["dout"]), state=state, scaled=True)
    assert_close(gr["dprob"], ref["dprob"], f"{name}: scaled dprob")
    assert_close(gr["dw_down"], ref["dw_down"], f"{name}: scaled dw_down")
    lazy = {}

    def term(key):
        def get(idx):
            if not lazy:
                lazy.update(scaled_flip_terms(w, d, topk_prob, rows))
            return lazy[key][idx]
        return get
    helpers.assert_close_flips(gr["dw_gate_up"], ref["dw_gate_up"], term("dw_gate_up"), f"{name}: scaled dw_gate_up")
    helpers.assert_close_flips(gr["dx"], ref["dx"], term("dx"), f"{name}: scaled dx")
    counts = np.diff(r["offsets"].cpu().numpy())
    for e in np.nonzero(counts == 0)[0]:
        assert torch.all(gr["dw_down"][e] == 0) and torch.all(gr["dw_gate_up"][e] == 0)


@pytest.mark.parametrize("name", ["qwen3_a16", "odd_dims_a8"])
def test_scaled_backward_is_deterministic_and_tile_independent(name):
    """Each output has one writer and a fixed order of operations, and dprob's
    partial sums cover the same 64-column groups on either tile shape: the
    results are bit-identical across runs and across single and pair tiles."""
    w, align = CASES[name]
    m, d, r, rows = scaled_forward(w, align)
    outs = []
    for tiles in ("single", "single", "pair"):
        helpers.force_kernels(gemm_tiles=tiles)
        gr = scaled_backward(m, d, rows)
        torch.cuda.synchronize()
        outs.append({k: v.clone() for k, v in gr.items()})
    assert m.moe_get_device_status() == 0
    as_int = {torch.bfloat16: torch.int16, torch.float32: torch.int32}
    for o in outs[1:]:
        for key in ("dx", "dw_gate_up", "dw_down", "dprob"):
            a, b = outs[0][key], o[key]
            assert torch.equal(a.view(as_int[a.dtype]), b.view(as_int[b.dtype])), key

