"""Shared helpers of the GPU parity tests."""
import sys

import numpy as np
import pytest
import torch

# Elementwise bound for bf16 outputs and gradients: |gpu - ref| <= ATOL + RTOL * |ref|
ATOL = 1e-2
RTOL = 1e-2


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from routing_grouped_gemm_score_b200 import build
    build.build()


def to_f64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu").double().numpy()
    return np.asarray(t, np.float64)


# One record per elementwise comparison of a float result with the oracle:
# how many elements lie beyond the strict bound ATOL + RTOL |ref|. The
# terminal summary of the test run (conftest.py) prints these counts, and
# MOE_PARITY_LOG=<path> also writes them as JSON.
PARITY = []


def _record(what, g, r, err, tol, beyond_strict, allowance=None):
    ratio = np.where(tol > 0, err / tol, 0.0) if err.size else np.zeros(1)
    PARITY.append({"what": what, "elements": int(g.size), "beyond_strict": int(beyond_strict),
                   "worst_err_over_tol": float(np.nanmax(ratio)) if ratio.size else 0.0,
                   "allowance": allowance})


def assert_close(gpu, ref, what: str, atol: float = ATOL, rtol: float = RTOL) -> None:
    """Elementwise |gpu - ref| <= atol + rtol |ref|; reports the worst element,
    NaN/Inf counts and the first failing index."""
    g = to_f64(gpu)
    r = to_f64(ref)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    bad_nan = np.isnan(g) != np.isnan(r)
    err = np.abs(g - r)
    tol = atol + rtol * np.abs(r)
    viol = (err > tol) & ~(np.isnan(g) & np.isnan(r))
    viol |= bad_nan
    if atol == ATOL and rtol == RTOL:
        _record(what, g, r, np.where(np.isnan(err), 0.0, err), tol, viol.sum())
    if viol.any():
        idx = np.argwhere(viol)
        first = tuple(idx[0])
        worst = np.unravel_index(np.nanargmax(np.where(viol, err / tol, 0)), g.shape)
        raise AssertionError(
            f"{what}: {viol.sum()} of {g.size} elements out of tolerance; first at {first} "
            f"(gpu {g[first]!r}, ref {r[first]!r}); worst at {tuple(worst)} "
            f"(gpu {g[worst]!r}, ref {r[worst]!r}); gpu NaN/Inf {int((~np.isfinite(g)).sum())}")


def assert_equal(gpu, ref, what: str) -> None:
    g = gpu.detach().cpu().numpy() if isinstance(gpu, torch.Tensor) else np.asarray(gpu)
    r = np.asarray(ref)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    if not np.array_equal(g, r):
        idx = np.argwhere(g != r)
        first = tuple(idx[0])
        raise AssertionError(f"{what}: {len(idx)} mismatches; first at {first}: "
                             f"gpu {g[first]} ref {r[first]}")


def device_inputs(w, device="cuda", with_dout=None):
    import workloads as wl
    return wl.make_inputs(w, device=device, with_dout=with_dout)


def bits(t):
    import oracle
    return oracle.bf16_bits(t)


FLIP = 2.0 ** -7     # one bf16 ulp, relative, at most


def assert_close_flips(gpu, ref, term, what: str, max_frac: float = 1e-4) -> None:
    """The stated bound, |gpu - ref| <= ATOL + RTOL |ref|, on every element,
    with one counted allowance. A stored bf16 intermediate is the rounding of
    an fp32 value on the GPU and of an fp64 value in the oracle; where the two
    fall on the two sides of a rounding boundary, the stored values differ by
    one ulp (at most 2^-7 of the value). An output element that sums products
    with that term then moves by at most 2^-7 x |term|. Elements beyond the
    strict bound must lie within that one flip of their largest stored
    summand, and there may be at most `max_frac` of them. Every call records
    how many elements needed the allowance.

    `term` holds the largest such summand per element, or is a function that
    returns it for the elements given by an index tuple (computed only when
    some element lies beyond the strict bound)."""
    g, r = to_f64(gpu), to_f64(ref)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    err = np.abs(g - r)
    tol = ATOL + RTOL * np.abs(r)
    nan_bad = np.isnan(g) | np.isnan(r)
    strict = (err > tol) | nan_bad
    n_strict = int(strict.sum())
    _record(what, g, r, np.where(np.isnan(err), np.inf, err), tol, n_strict, allowance="one bf16 flip")
    if n_strict == 0:
        return
    idx = np.nonzero(strict)
    tm = term(idx) if callable(term) else to_f64(term)[idx]
    flip = (err[idx] > tol[idx] + FLIP * np.abs(tm)) | nan_bad[idx]
    if flip.any():
        n = int(np.argmax(flip))
        first = tuple(int(a[n]) for a in idx)
        raise AssertionError(f"{what}: {int(flip.sum())} elements beyond one bf16 flip; first at {first} "
                             f"(gpu {g[first]}, ref {r[first]}, term {tm[n]}); NaN {int(nan_bad.sum())}")
    assert n_strict <= max_frac * g.size, f"{what}: {n_strict} of {g.size} need the flip allowance"


def bf16_round_np(v) -> np.ndarray:
    """Round float64 values to bf16 and return them as float64."""
    import oracle
    return oracle.bits_to_float(oracle.round_bf16_array(v))


def oracle_saved_state(w, d, r):
    """The forward state a bf16 pipeline saves, computed by the oracle:
    permuted rows, [g | u], h, y (all bf16 values, as float64 arrays), plus
    the routing bookkeeping."""
    import oracle
    bits = oracle.bf16_bits
    x, wgu, wd = bits(d["x"]), bits(d["w_gate_up"]), bits(d["w_down"])
    st, row_of = oracle.dispatch(r["topk_idx"], r["offsets"], w.E)
    xp = oracle.gather_rows(x, st)
    A = len(st)
    g = np.zeros((A, w.I)); u = np.zeros((A, w.I)); h = np.zeros((A, w.I)); y = np.zeros((A, w.H))
    offs = r["offsets"]
    for e in range(w.E):
        a, b = offs[e], offs[e + 1]
        if b > a:
            y[a:b], g[a:b], u[a:b], h[a:b] = oracle.expert_mlp(xp[a:b], wgu[e], wd[e], True, True)
    return dict(sorted_token=st, row_of=row_of, x_perm=oracle.bits_to_float(xp),
                g=bf16_round_np(g), u=bf16_round_np(u), h=h, y=y)


def flip_terms(w, d, r, s):
    """Largest single product per gradient element (see assert_close_flips),
    from the oracle's stored values `s` (oracle_saved_state)."""
    import oracle
    bits = oracle.bf16_bits
    wgu = oracle.bits_to_float(bits(d["w_gate_up"]))
    wd = oracle.bits_to_float(bits(d["w_down"]))
    dout = oracle.bits_to_float(bits(d["dout"]))
    st, row_of, offs = s["sorted_token"], s["row_of"], r["offsets"]
    A = len(st)
    p_row = np.zeros(A, np.float32)
    p_row[row_of.ravel()] = r["topk_prob"].ravel()
    dy = (p_row[:, None] * dout[st].astype(np.float32)).astype(np.float64)
    dy = bf16_round_np(dy)
    I = w.I
    t_dwd = np.zeros((w.E, w.I, w.H)); t_dwgu = np.zeros((w.E, w.H, 2 * I))
    dxp = np.zeros((A, w.H))
    for e in range(w.E):
        a, b = offs[e], offs[e + 1]
        if b == a:
            continue
        he, dye, xe = np.abs(s["h"][a:b]), np.abs(dy[a:b]), np.abs(s["x_perm"][a:b])
        dh = dy[a:b] @ wd[e].T
        gb, ub = s["g"][a:b], s["u"][a:b]
        sg = 1.0 / (1.0 + np.exp(-gb))
        dgu = np.concatenate([dh * ub * (sg + gb * sg * (1 - sg)), dh * gb * sg], axis=1)
        dxp[a:b] = np.abs(dgu @ wgu[e].T)
        dgu = np.abs(dgu)
        for rr in range(b - a):
            np.maximum(t_dwd[e], np.outer(he[rr], dye[rr]), out=t_dwd[e])
            np.maximum(t_dwgu[e], np.outer(xe[rr], dgu[rr]), out=t_dwgu[e])
    t_dx = dxp[row_of].sum(axis=1)
    t_dprob = np.abs(dout[:, None, :] * s["y"][row_of]).max(axis=2)
    return dict(dw_down=t_dwd, dw_gate_up=t_dwgu, dx=t_dx, dprob=t_dprob)


def forward_terms(w, d, tokens, logits=None):
    """Largest stored bf16 summand of each output element: out[t] is
    shared[t] + sum_j p_j y_j with shared and y stored in bf16, so a flip of
    one stored summand moves the element by at most 2^-7 of it."""
    import oracle
    bits_ = oracle.bf16_bits
    x, wgu, wd = bits_(d["x"]), bits_(d["w_gate_up"]), bits_(d["w_down"])
    logits = d["logits"].cpu().numpy() if logits is None else logits
    r = oracle.router_topk(logits[tokens], w.k, w.score, w.renormalize, with_map=False)
    term = np.zeros((len(tokens), w.H))
    for n, t in enumerate(tokens):
        if d.get("shared_gate_up") is not None:
            s = oracle.expert_mlp(x[t:t + 1], bits_(d["shared_gate_up"][0]), bits_(d["shared_down"][0]))
            term[n] = np.abs(s[0])
        for j in range(w.k):
            e = int(r["topk_idx"][n, j])
            y = oracle.expert_mlp(x[t:t + 1], wgu[e], wd[e])
            np.maximum(term[n], abs(float(r["topk_prob"][n, j])) * np.abs(y[0]), out=term[n])
    return term


def lazy_forward_terms(w, d, tokens, logits=None):
    """forward_terms of the rows `tokens` (row n of the compared output is
    token tokens[n]), computed only for the rows that assert_close_flips asks
    for."""
    tokens = np.asarray(tokens)

    def fn(idx):
        rows = np.unique(idx[0])
        t = forward_terms(w, d, tokens[rows], logits)
        return t[np.searchsorted(rows, idx[0]), idx[1]]
    return fn


_FORCED = {}


def force_kernels(gemm_tiles=None, router=None, permute=None, fold_permute=None) -> None:
    """Force kernel variants through the library's testing hook
    (moe_testing_set_kernels) for the rest of the current test; conftest.py
    restores the library's own choice after each test. Values: gemm_tiles
    "single" | "pair", router "warp" | "lane", permute "tokens" | "warp",
    fold_permute True | False ("swap": the forward GEMMs on swap-AB tiles,
    "swap_unfused": the same with a layer's gate_up and down as two launches);
    "auto" or None leaves a setting as it is."""
    import routing_grouped_gemm_score_b200 as m
    names = {"gemm_tiles": {"auto": 0, "single": m.GEMM_SINGLE, "pair": m.GEMM_PAIR, "swap": m.GEMM_SWAP,
                            "swap_unfused": m.GEMM_SWAP_UNFUSED},
             "router": {"auto": 0, "warp": m.ROUTER_WARP, "lane": m.ROUTER_LANE},
             "permute": {"auto": 0, "tokens": m.PERMUTE_TOKENS, "warp": m.PERMUTE_WARP}}
    for key, val in (("gemm_tiles", gemm_tiles), ("router", router), ("permute", permute)):
        if val is not None:
            _FORCED[key] = names[key][val]
    if fold_permute is not None:
        _FORCED["fold_permute"] = int(bool(fold_permute))
    m.moe_testing_set_kernels(**_FORCED)


def reset_kernels() -> None:
    _FORCED.clear()
    m = sys.modules.get("routing_grouped_gemm_score_b200")
    if m is not None and getattr(m, "_lib", None) is not None:
        m.moe_testing_set_kernels()
