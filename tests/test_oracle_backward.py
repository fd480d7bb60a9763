"""Pins of the oracle's backward: fp64 finite differences of the oracle's own
forward, and torch autograd of the layer restated with torch primitives.

Transformer Engine "Mixture of Experts", Example (every stage is
differentiable). The routing weights are inputs, so their gradient is
<dout, expert output>.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import workloads as wl


def setup(T=5, H=16, I=8, E=3, k=2, seed=0):
    w = wl.WORKLOADS["tiny"].scaled(T=T, H=H, I=I, E=E, k=k, seed=seed)
    d = wl.make_inputs(w, with_dout=True)
    return w, d


def loss(oracle_lib, w, x, logits_unused, wgu, wd, idx, prob, dout):
    """L = <dout, out> with out = sum_j p_j MLP_{e_j}(x_t), via the oracle's
    forward pieces (round_bf16 off, so L is smooth)."""
    out = np.zeros((w.T, w.H))
    for t in range(w.T):
        for j in range(w.k):
            e = idx[t, j]
            y = oracle_lib.expert_mlp(x[t:t + 1], wgu[e], wd[e], round_bf16=False)
            out[t] += float(prob[t, j]) * y[0]
    return float((oracle_lib.bits_to_float(dout) * out).sum())


def richardson(f, delta):
    """Central difference with one Richardson step: error O(delta^4)."""
    d1 = (f(delta) - f(-delta)) / (2 * delta)
    d2 = (f(2 * delta) - f(-2 * delta)) / (4 * delta)
    return (4 * d1 - d2) / 3


def test_backward_matches_finite_differences(oracle_lib):
    w, d = setup()
    bits = oracle_lib.bf16_bits
    x, wgu, wd, dout = bits(d["x"]), bits(d["w_gate_up"]), bits(d["w_down"]), bits(d["dout"])
    r = oracle_lib.router_topk(d["logits"].numpy(), w.k)
    idx, prob = r["topk_idx"], r["topk_prob"]
    rng = np.random.default_rng(1)
    c = 0.5          # a perturbed bf16 coordinate is set to c; c +- delta, c +- 2 delta are exact
    delta = 2.0 ** -6

    def with_value(arr, pos, v):
        a = arr.copy()
        a[pos] = oracle_lib.round_bf16(v)
        assert oracle_lib.bits_to_float(a[pos]) == v
        return a

    checked = 0
    for name in ("x", "w_gate_up", "w_down"):
        base = {"x": x, "w_gate_up": wgu, "w_down": wd}[name]
        for _ in range(12):
            pos = tuple(int(rng.integers(0, s)) for s in base.shape)
            arrs = {"x": x, "w_gate_up": wgu, "w_down": wd}
            arrs[name] = with_value(base, pos, c)
            g = oracle_lib.moe_backward(arrs["x"], idx, prob, arrs["w_gate_up"], arrs["w_down"],
                                        dout, round_bf16=False)
            analytic = {"x": g["dx"], "w_gate_up": g["dw_gate_up"], "w_down": g["dw_down"]}[name][pos]

            def f(dl):
                a2 = dict(arrs)
                a2[name] = with_value(base, pos, c + dl)
                return loss(oracle_lib, w, a2["x"], None, a2["w_gate_up"], a2["w_down"], idx, prob, dout)
            numeric = richardson(f, delta)
            assert abs(numeric - analytic) <= 1e-6 + 1e-5 * abs(analytic), (name, pos, numeric, analytic)
            checked += 1
    # routing weights: fp32 inputs
    g = oracle_lib.moe_backward(x, idx, prob, wgu, wd, dout, round_bf16=False)
    for t in range(w.T):
        for j in range(w.k):
            def f(dl):
                p2 = prob.astype(np.float64).copy()
                p2[t, j] += dl
                out = 0.0
                y = oracle_lib.expert_mlp(x[t:t + 1], wgu[idx[t, j]], wd[idx[t, j]], round_bf16=False)
                return float((oracle_lib.bits_to_float(dout[t]) * y[0]).sum() * p2[t, j])
            numeric = richardson(f, 1e-3)
            assert abs(numeric - g["dprob"][t, j]) <= 1e-9 + 1e-9 * abs(numeric)
            checked += 1
    assert checked == 36 + w.T * w.k


class _RoundValue(torch.autograd.Function):
    """Forward: round to bf16. Backward: gradient passed through unchanged."""
    @staticmethod
    def forward(ctx, v):
        return v.float().to(torch.bfloat16).double()

    @staticmethod
    def backward(ctx, g):
        return g


class _RoundGrad(torch.autograd.Function):
    """Forward: identity. Backward: the gradient is rounded to bf16 (a stored
    gradient tensor of a bf16 pipeline)."""
    @staticmethod
    def forward(ctx, v):
        return v.clone()

    @staticmethod
    def backward(ctx, g):
        return g.float().to(torch.bfloat16).double()


class _WeightedGrad(torch.autograd.Function):
    """Forward: p * y. Backward: dy = bf16(fp32(p) * fp32(dout)) and
    dp = <dout, y>, as a bf16 pipeline stores the expert-output gradient."""
    @staticmethod
    def forward(ctx, y, p):
        ctx.save_for_backward(y, p)
        return p * y

    @staticmethod
    def backward(ctx, g):
        y, p = ctx.saved_tensors
        dy = (p.float() * g.float()).to(torch.bfloat16).double()
        return dy, (g * y).sum()


def _round_both(v):
    return _RoundGrad.apply(_RoundValue.apply(v))


@pytest.mark.parametrize("round_bf16", [False, True])
def test_backward_matches_torch_autograd(oracle_lib, round_bf16):
    """torch autograd of the layer written with torch primitives. With
    rounding: the stored tensors (g, u, h, y) round their values, and the
    stored gradients (dy, dg, du, dx_perm) round theirs."""
    w, d = setup(T=24, H=32, I=24, E=5, k=2, seed=3)
    bits = oracle_lib.bf16_bits
    r = oracle_lib.router_topk(d["logits"].numpy(), w.k)
    idx = torch.from_numpy(r["topk_idx"].astype(np.int64))
    prob = torch.from_numpy(r["topk_prob"]).double().requires_grad_(True)
    x = d["x"].double().requires_grad_(True)
    wgu = d["w_gate_up"].double().requires_grad_(True)
    wd = d["w_down"].double().requires_grad_(True)
    I = w.I
    out = torch.zeros(w.T, w.H, dtype=torch.float64)
    for t in range(w.T):
        for j in range(w.k):
            e = int(idx[t, j])
            xr = _RoundGrad.apply(x[t]) if round_bf16 else x[t]
            g = xr @ wgu[e][:, :I]
            u = xr @ wgu[e][:, I:]
            if round_bf16:
                gb, ub = _round_both(g), _round_both(u)
                # value from the unrounded g, u; gradient through the stored g, u
                h = F.silu(gb) * ub + (F.silu(g) * u - F.silu(gb) * ub).detach()
                h = _RoundValue.apply(h)
                y = _RoundValue.apply(h @ wd[e])
                # the stored gradient of y is bf16(p * dout) with the product in fp32
                y = _WeightedGrad.apply(y, prob[t, j])
                out[t] = out[t] + y
            else:
                y = (F.silu(g) * u) @ wd[e]
                out[t] = out[t] + prob[t, j] * y
    (out * d["dout"].double()).sum().backward()
    g = oracle_lib.moe_backward(bits(d["x"]), r["topk_idx"], r["topk_prob"], bits(d["w_gate_up"]),
                                bits(d["w_down"]), bits(d["dout"]), round_bf16=round_bf16)
    np.testing.assert_allclose(g["dx"], x.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(g["dw_gate_up"], wgu.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(g["dw_down"], wd.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(g["dprob"], prob.grad.numpy(), rtol=1e-9, atol=1e-11)


def test_backward_empty_expert_and_expert_filter(oracle_lib):
    w, d = setup(T=10, H=16, I=8, E=4, k=1, seed=4)
    logits = d["logits"].numpy().copy()
    logits[:, 1] = -1e4
    r = oracle_lib.router_topk(logits, 1)
    assert r["counts"][1] == 0
    bits = oracle_lib.bf16_bits
    args = (bits(d["x"]), r["topk_idx"], r["topk_prob"], bits(d["w_gate_up"]), bits(d["w_down"]),
            bits(d["dout"]))
    g = oracle_lib.moe_backward(*args)
    assert np.all(g["dw_gate_up"][1] == 0) and np.all(g["dw_down"][1] == 0)
    for e in range(4):
        ge = oracle_lib.moe_backward(*args, only_expert=e, want=("dw_gate_up", "dw_down"))
        np.testing.assert_array_equal(ge["dw_gate_up"][0], g["dw_gate_up"][e])
        np.testing.assert_array_equal(ge["dw_down"][0], g["dw_down"][e])
    toks = [7, 2, 9]
    gt = oracle_lib.moe_backward(*args, tokens=toks, want=("dx", "dprob"))
    np.testing.assert_array_equal(gt["dx"], g["dx"][toks])
    np.testing.assert_array_equal(gt["dprob"], g["dprob"][toks])


def _own_state(oracle_lib, w, d, r):
    """The oracle's own forward state in the layout a saved state has: one
    row per permuted assignment, [g | u], h and y as bf16 bit patterns."""
    bits = oracle_lib.bf16_bits
    x, wgu, wd = bits(d["x"]), bits(d["w_gate_up"]), bits(d["w_down"])
    st, row_of = oracle_lib.dispatch(r["topk_idx"], r["offsets"], w.E)
    xp = oracle_lib.gather_rows(x, st)
    A = len(st)
    gu = np.zeros((A, 2 * w.I), np.uint16)
    h = np.zeros((A, w.I), np.uint16)
    y = np.zeros((A, w.H), np.uint16)
    offs = r["offsets"]
    for e in range(w.E):
        a, b = offs[e], offs[e + 1]
        if b > a:
            ye, ge, ue, he = oracle_lib.expert_mlp(xp[a:b], wgu[e], wd[e], True, True)
            gu[a:b, :w.I] = oracle_lib.round_bf16_array(ge)
            gu[a:b, w.I:] = oracle_lib.round_bf16_array(ue)
            h[a:b] = oracle_lib.round_bf16_array(he)
            y[a:b] = oracle_lib.round_bf16_array(ye)
    return {"row_of": row_of, "gu": gu, "h": h, "y": y}


def test_backward_from_saved_state_equals_recomputed_forward(oracle_lib):
    """Given the oracle's own rounded forward state, the saved-state mode
    returns exactly what the mode that recomputes the forward returns."""
    w, d = setup(T=12, H=24, I=16, E=4, k=2, seed=7)
    r = oracle_lib.router_topk(d["logits"].numpy(), w.k)
    bits = oracle_lib.bf16_bits
    args = (bits(d["x"]), r["topk_idx"], r["topk_prob"], bits(d["w_gate_up"]), bits(d["w_down"]),
            bits(d["dout"]))
    a = oracle_lib.moe_backward(*args)
    b = oracle_lib.moe_backward(*args, state=_own_state(oracle_lib, w, d, r))
    for key in ("dx", "dw_gate_up", "dw_down", "dprob"):
        np.testing.assert_array_equal(a[key], b[key], err_msg=key)


def test_backward_reads_the_given_state(oracle_lib):
    """The saved state is what the chain rule reads: a change of one stored
    row moves exactly the gradients that row feeds. dprob of the assignment
    stored in row r is <dout_t, y_r>, so changing y_r by delta moves it by
    <dout_t, delta> and moves nothing else; changing h_r moves only
    dW_down of its expert, by the outer product of the change with that
    assignment's bf16(p * dout)."""
    w, d = setup(T=10, H=16, I=8, E=3, k=2, seed=8)
    r = oracle_lib.router_topk(d["logits"].numpy(), w.k)
    bits = oracle_lib.bf16_bits
    args = (bits(d["x"]), r["topk_idx"], r["topk_prob"], bits(d["w_gate_up"]), bits(d["w_down"]),
            bits(d["dout"]))
    s0 = _own_state(oracle_lib, w, d, r)
    g0 = oracle_lib.moe_backward(*args, state=s0)
    t, j = 3, 1
    row = s0["row_of"][t, j]
    e = r["topk_idx"][t, j]
    dout = oracle_lib.bits_to_float(bits(d["dout"]))
    # y: a new stored row
    s1 = {k_: v.copy() for k_, v in s0.items()}
    y_new = oracle_lib.round_bf16_array(np.linspace(-2.0, 2.0, w.H))
    s1["y"][row] = y_new
    g1 = oracle_lib.moe_backward(*args, state=s1)
    delta = oracle_lib.bits_to_float(y_new) - oracle_lib.bits_to_float(s0["y"][row])
    want = g0["dprob"].copy()
    want[t, j] += float(dout[t] @ delta)
    np.testing.assert_allclose(g1["dprob"], want, rtol=1e-12, atol=1e-12)
    for key in ("dx", "dw_gate_up", "dw_down"):
        np.testing.assert_array_equal(g1[key], g0[key], err_msg=key)
    # h: a new stored row
    s2 = {k_: v.copy() for k_, v in s0.items()}
    h_new = oracle_lib.round_bf16_array(np.linspace(0.5, -0.5, w.I))
    s2["h"][row] = h_new
    g2 = oracle_lib.moe_backward(*args, state=s2)
    dh = oracle_lib.bits_to_float(h_new) - oracle_lib.bits_to_float(s0["h"][row])
    dy = oracle_lib.bits_to_float(oracle_lib.round_bf16_array(
        (np.float32(r["topk_prob"][t, j]) * dout[t].astype(np.float32)).astype(np.float64)))
    want = g0["dw_down"].copy()
    want[e] += np.outer(dh, dy)
    np.testing.assert_allclose(g2["dw_down"], want, rtol=1e-12, atol=1e-12)
    for key in ("dx", "dw_gate_up", "dprob"):
        np.testing.assert_array_equal(g2[key], g0[key], err_msg=key)


def test_backward_state_shapes_are_checked(oracle_lib):
    w, d = setup(T=6, H=16, I=8, E=3, k=2, seed=9)
    r = oracle_lib.router_topk(d["logits"].numpy(), w.k)
    bits = oracle_lib.bf16_bits
    s = _own_state(oracle_lib, w, d, r)
    s["h"] = s["h"][:, :4]
    with pytest.raises(ValueError):
        oracle_lib.moe_backward(bits(d["x"]), r["topk_idx"], r["topk_prob"], bits(d["w_gate_up"]),
                                bits(d["w_down"]), bits(d["dout"]), state=s)


def test_scaled_backward_equals_weighting_in_the_combine_when_exact(oracle_lib):
    """ScaledSwiGLU (Transformer Engine Grouped MLP: the weight multiplies the
    SwiGLU output before FC2, the combine is unweighted) is the same layer
    as the weight applied in the combine, since FC2 is linear: p (s Wd) =
    (p s) Wd. Without the bf16 roundings, its four gradients therefore equal
    those of the weights-in-combine backward (itself pinned by finite
    differences above)."""
    w, d = setup(T=9, H=24, I=16, E=4, k=2, seed=11)
    r = oracle_lib.router_topk(d["logits"].numpy(), w.k)
    bits = oracle_lib.bf16_bits
    args = (bits(d["x"]), r["topk_idx"], r["topk_prob"], bits(d["w_gate_up"]), bits(d["w_down"]),
            bits(d["dout"]))
    a = oracle_lib.moe_backward(*args, round_bf16=False)
    b = oracle_lib.moe_backward(*args, round_bf16=False, scaled=True)
    for key in ("dx", "dw_gate_up", "dw_down", "dprob"):
        np.testing.assert_allclose(b[key], a[key], rtol=1e-10, atol=1e-12, err_msg=key)


def test_scaled_backward_weight_gradient_by_finite_differences(oracle_lib):
    """d out / d p of the ScaledSwiGLU layer: central differences in fp64 of
    the layer restated with the weight on the SwiGLU output (torch
    primitives on the exact bf16 inputs) against the oracle's dprob."""
    w, d = setup(T=5, H=16, I=8, E=3, k=2, seed=12)
    r = oracle_lib.router_topk(d["logits"].numpy(), w.k)
    bits = oracle_lib.bf16_bits
    x = d["x"].double()
    wgu, wd, dout = d["w_gate_up"].double(), d["w_down"].double(), d["dout"].double()
    idx = torch.from_numpy(r["topk_idx"]).long()

    def loss(prob):
        out = torch.zeros((w.T, w.H), dtype=torch.float64)
        for t in range(w.T):
            for j in range(w.k):
                e = idx[t, j]
                g = x[t] @ wgu[e][:, :w.I]
                u = x[t] @ wgu[e][:, w.I:]
                out[t] += (prob[t, j] * F.silu(g) * u) @ wd[e]
        return float((dout * out).sum())

    g = oracle_lib.moe_backward(bits(d["x"]), r["topk_idx"], r["topk_prob"], bits(d["w_gate_up"]),
                                bits(d["w_down"]), bits(d["dout"]), round_bf16=False, scaled=True)
    prob = torch.from_numpy(r["topk_prob"].astype(np.float64))
    for t in range(w.T):
        for j in range(w.k):
            def f(delta):
                q = prob.clone()
                q[t, j] += delta
                return loss(q)
            fd = richardson(f, 1e-3)
            assert abs(fd - g["dprob"][t, j]) <= 1e-8 * (1 + abs(fd)), (t, j, fd, g["dprob"][t, j])


def test_scaled_backward_from_saved_state(oracle_lib):
    """Given its own rounded scaled state (h = bf16(p silu(g) u) per row),
    the saved-state mode of the scaled backward returns what the recomputing
    mode returns."""
    w, d = setup(T=12, H=24, I=16, E=4, k=2, seed=13)
    r = oracle_lib.router_topk(d["logits"].numpy(), w.k)
    bits = oracle_lib.bf16_bits
    args = (bits(d["x"]), r["topk_idx"], r["topk_prob"], bits(d["w_gate_up"]), bits(d["w_down"]),
            bits(d["dout"]))
    s0 = _own_state(oracle_lib, w, d, r)
    x, wgu = bits(d["x"]), bits(d["w_gate_up"])
    st, row_of = oracle_lib.dispatch(r["topk_idx"], r["offsets"], w.E)
    p_row = np.zeros(len(st))
    p_row[row_of.ravel()] = r["topk_prob"].ravel()
    offs = r["offsets"]
    xp = oracle_lib.gather_rows(x, st)
    for e in range(w.E):
        a_, b_ = offs[e], offs[e + 1]
        if b_ > a_:
            _, ge, ue, _ = oracle_lib.expert_mlp(xp[a_:b_], wgu[e], bits(d["w_down"])[e], True, True)
            sv = ge / (1 + np.exp(-ge)) * ue
            s0["h"][a_:b_] = oracle_lib.round_bf16_array(p_row[a_:b_, None] * sv)
    a = oracle_lib.moe_backward(*args, scaled=True)
    b = oracle_lib.moe_backward(*args, scaled=True, state={"row_of": s0["row_of"], "gu": s0["gu"], "h": s0["h"]})
    for key in ("dx", "dw_gate_up", "dw_down", "dprob"):
        np.testing.assert_array_equal(a[key], b[key], err_msg=key)
