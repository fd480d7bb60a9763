"""Full-size parity: every workload at its full shape, through the call the
benchmark times (moe_layer_forward, and moe_grouped_mlp_backward for the
training workloads). Routing is compared on every token. The rest is compared
on samples, which the oracle computes one by one:
  - the saved forward state ([g | u], h, y and the permuted x rows) of 64
    sampled assignments, each stage strictly within the bound;
  - the combine on the GPU's own stored y rows, strictly;
  - the layer output of 512 sampled tokens against the oracle's independent
    per-token definition (a counted allowance of one bf16 flip: the GPU's fp32
    and the oracle's fp64 values of a stored intermediate can round apart);
  - the backward on 512 sampled tokens (dx, dprob) and on the whole weight
    gradients of 8 experts, against the oracle's chain rule on the saved
    state the backward call was given.

Shapes: Mixtral-8x7B (T=4096, H=4096, I=14336, E=8, k=2), Qwen3-30B-A3B
(T=4096, H=2048, I=768, E=128, k=8, forward and backward), Llama-4-17Bx16E
(T=8192, H=5120, I=8192, E=16, k=1, sigmoid, shared expert), and the skewed
sweep at the Qwen3 shape (T = 1, 8, 64, 16384; 16 dead experts), with the
tie case (T=64, logits in multiples of 0.5).
"""
import os
from concurrent.futures import ThreadPoolExecutor

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


def sample_tokens(T, n=512, seed=0):
    """n distinct tokens spread over the batch (all of them when T <= n),
    always with the first and the last."""
    if T <= n:
        return np.arange(T, dtype=np.int64)
    rng = np.random.default_rng(seed)
    picks = {0, T - 1} | set(rng.choice(np.arange(1, T - 1), size=n - 2, replace=False).tolist())
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
                       helpers.lazy_forward_terms(w, d, tokens, logits), f"{name}: out ({len(tokens)} tokens)")
    check_forward_state(w, d, st, tokens)
    if not w.shared_expert:
        check_combine_on_stored_rows(w, st, out, tokens)


def check_forward_state(w, d, st, tokens, n=64, seed=5):
    """The stored forward state of n sampled assignments, stage by stage,
    against the oracle's expert on the same token: the permuted row (bit for
    bit), g and u (the gate_up GEMM), h (its SwiGLU epilogue) and y (the down
    GEMM), each strictly within the bound."""
    rng = np.random.default_rng(seed)
    ts = rng.choice(tokens, size=min(n, len(tokens)), replace=False)
    js = rng.integers(0, w.k, size=len(ts))
    rows = st["row_of"].cpu().numpy()[ts, js]
    es = st["topk_idx"].cpu().numpy()[ts, js]
    x, wgu, wd = bits(d["x"]), bits(d["w_gate_up"]), bits(d["w_down"])

    def one(i):
        return oracle.expert_mlp(x[ts[i]:ts[i] + 1], wgu[es[i]], wd[es[i]], True, True)
    with ThreadPoolExecutor(max_workers=os.cpu_count() or 1) as ex:
        res = list(ex.map(one, range(len(ts))))
    y, g, u, h = (np.concatenate([r_[q] for r_ in res]) for q in range(4))
    rt = torch.from_numpy(rows).cuda()
    assert_equal(st["x_perm"][rt].view(torch.int16).cpu().numpy().view(np.uint16), x[ts],
                 f"{w.name}: x_perm rows")
    gu = st["gu"][rt]
    assert_close(gu[:, :w.I], g, f"{w.name}: g ({len(ts)} rows)")
    assert_close(gu[:, w.I:], u, f"{w.name}: u ({len(ts)} rows)")
    assert_close(st["h"][rt], h, f"{w.name}: h ({len(ts)} rows)")
    assert_close(st["y_perm"][rt], y, f"{w.name}: y ({len(ts)} rows)")


def check_combine_on_stored_rows(w, st, out, tokens):
    """out of the sampled tokens against the oracle's combine of the GPU's
    own stored y rows and routing weights, strictly within the bound."""
    row_of = st["row_of"].cpu().numpy()[tokens]
    y = st["y_perm"][torch.from_numpy(row_of.ravel()).cuda()].double().cpu().numpy()
    sub = np.arange(len(tokens) * w.k, dtype=np.int32).reshape(len(tokens), w.k)
    ref = oracle.combine(y, sub, st["topk_prob"].cpu().numpy()[tokens])
    assert_close(out[torch.from_numpy(tokens).cuda()], ref, f"{w.name}: out on stored y ({len(tokens)} tokens)")


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


class _F(dict):
    """float64 copies of the expert weights, made on first use."""

    def __init__(self, src):
        super().__init__()
        self.src = src

    def __missing__(self, e):
        self[e] = oracle.bits_to_float(self.src[e])
        return self[e]


def pick_experts(counts, n=8, seed=2):
    """The experts whose full weight gradients are compared: the busiest, the
    smallest non-empty one, the one whose last 64-row K slice is most ragged
    (fewest rows in it), an empty one if any, then seeded random ones."""
    counts = np.asarray(counts)
    nz = np.nonzero(counts > 0)[0]
    chosen = [int(np.argmax(counts)), int(nz[np.argmin(counts[nz])])]
    tail = counts[nz] % 64
    tail = np.where(tail == 0, 64, tail)
    chosen.append(int(nz[np.argmin(tail)]))
    empty = np.nonzero(counts == 0)[0]
    if len(empty):
        chosen.append(int(empty[0]))
    rng = np.random.default_rng(seed)
    for e in rng.permutation(len(counts)):
        if len(set(chosen)) >= n:
            break
        chosen.append(int(e))
    return list(dict.fromkeys(chosen))[:n]


class _Ctx:
    """Host copies of one workload's inputs and the oracle's routing, for the
    backward comparisons."""

    def __init__(self, w, d, st):
        self.w = w
        logits = d["logits"].cpu().numpy()
        self.r = oracle.router_topk(logits, w.k, w.score, w.renormalize, with_map=False)
        assert_equal(st["topk_idx"], self.r["topk_idx"], f"{w.name}: topk_idx")
        self.x, self.wgu, self.wd = bits(d["x"]), bits(d["w_gate_up"]), bits(d["w_down"])
        self.dout = bits(d["dout"])
        self.wgu_f, self.wd_f = _F(self.wgu), _F(self.wd)
        # the saved forward state the backward call was given (bf16 bit patterns)
        self.state = {"row_of": st["row_of"].cpu().numpy(), "gu": bits(st["gu"]), "h": bits(st["h"]),
                      "y": bits(st["y_perm"])}

    def terms(self, t, j):
        e, p = int(self.r["topk_idx"][t, j]), self.r["topk_prob"][t, j]
        return _assignment_terms(self.x[t], e, p, self.dout[t], self.wgu, self.wd, self.wgu_f, self.wd_f)


def check_tokens(c, gr, tokens):
    """dx and dprob of the listed tokens against the oracle's chain rule on
    the saved state the backward was given. dprob = <dout, y> reads only that
    state: strictly within the bound. dx also carries the backward's own bf16
    roundings of [dg | du] and of each permuted row's dx (one-flip allowance,
    counted)."""
    w, r = c.w, c.r
    ref = oracle.moe_backward(c.x, r["topk_idx"], r["topk_prob"], c.wgu, c.wd, c.dout, tokens=tokens,
                              want=("dx", "dprob"), state=c.state)

    def token_terms():
        def fn(idx):
            rows = np.unique(idx[0])
            out = np.zeros((len(rows), w.H))
            for n, rr in enumerate(rows):
                t = tokens[rr]
                for j in range(w.k):
                    y, h, dy, dgu, dxp = c.terms(t, j)
                    out[n] += np.abs(dxp)
            return out[np.searchsorted(rows, idx[0]), idx[1]]
        return fn

    tk = torch.from_numpy(tokens).cuda()
    assert_close_flips(gr["dx"][tk], ref["dx"], token_terms(), f"{w.name}: dx ({len(tokens)} tokens)")
    assert_close(gr["dprob"][tk], ref["dprob"], f"{w.name}: dprob ({len(tokens)} tokens)")


def check_experts(c, gr, experts):
    """The whole dW_down and dW_gate_up of the listed experts against the
    oracle's chain rule on the saved state the backward was given (one host
    thread per expert). dW_down reads only that state and bf16(p * dout):
    strictly within the bound. dW_gate_up also carries the backward's own bf16
    rounding of [dg | du] (one-flip allowance, counted)."""
    w, r = c.w, c.r
    counts = r["counts"]

    def one(e):
        return oracle.moe_backward(c.x, r["topk_idx"], r["topk_prob"], c.wgu, c.wd, c.dout, only_expert=e,
                                   want=("dw_gate_up", "dw_down"), state=c.state)
    with ThreadPoolExecutor(max_workers=len(experts)) as ex:
        refs = dict(zip(experts, ex.map(one, experts)))

    def expert_terms(e):
        def fn(idx):
            t_w = np.zeros((w.H, 2 * w.I))
            for t, j in zip(*np.nonzero(r["topk_idx"] == e)):
                y, h, dy, dgu, dxp = c.terms(t, j)
                np.maximum(t_w, np.outer(np.abs(oracle.bits_to_float(c.x[t])), np.abs(dgu)), out=t_w)
            return t_w[idx]
        return fn

    for e in experts:
        tag = f"{w.name}: expert {e} ({int(counts[e])} rows)"
        if counts[e] == 0:
            assert torch.all(gr["dw_down"][e] == 0) and torch.all(gr["dw_gate_up"][e] == 0), tag
        assert_close(gr["dw_down"][e], refs[e]["dw_down"][0], f"{tag}: dw_down")
        assert_close_flips(gr["dw_gate_up"][e], refs[e]["dw_gate_up"][0], expert_terms(e),
                           f"{tag}: dw_gate_up")


def run_backward(name):
    import routing_grouped_gemm_score_b200 as m
    w = wl.WORKLOADS[name]
    d = wl.make_inputs(w, "cuda", with_dout=True)
    out, st = run_forward(w, d, save=True)
    gr = m.moe_grouped_mlp_backward(d["dout"], st, d["w_gate_up"], d["w_down"])
    torch.cuda.synchronize()
    assert m.moe_get_device_status() == 0
    return w, d, st, gr


def test_full_size_backward_sampled():
    """Qwen3-30B-A3B fwd+bwd at full size: dx and dprob on 512 sampled tokens,
    the whole dW_down and dW_gate_up of 8 experts (the busiest, the smallest,
    the most ragged last K slice, seeded random others)."""
    w, d, st, gr = run_backward("qwen3_30b_a3b")
    c = _Ctx(w, d, st)
    check_tokens(c, gr, sample_tokens(w.T, n=512, seed=1))
    check_experts(c, gr, pick_experts(c.r["counts"], 8))


def test_full_size_backward_with_empty_experts():
    """The grouped-MLP backward on the skewed 16384-token workload (Qwen3
    shape, 16 dead experts and more that get no token): every empty expert's
    weight gradients are exactly zero, and dx, dprob of 512 tokens and the
    whole dW of 8 experts (one empty, the smallest non-empty ones) match the
    oracle. The oracle's dW of one expert costs time in proportion to its
    rows, and the busiest experts here hold thousands, so the non-empty ones
    compared are the smallest."""
    w, d, st, gr = run_backward("skew_t16384")
    counts = st["counts"].cpu().numpy()
    empty = np.nonzero(counts == 0)[0]
    assert len(empty) >= 16
    for e in empty:
        assert torch.all(gr["dw_down"][e] == 0) and torch.all(gr["dw_gate_up"][e] == 0), e
    c = _Ctx(w, d, st)
    small = [int(e) for e in np.argsort(counts, kind="stable") if counts[e] > 0][:7]
    check_experts(c, gr, [int(empty[0])] + small)
    check_tokens(c, gr, sample_tokens(w.T, n=512, seed=3))
