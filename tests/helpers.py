"""Shared helpers of the GPU parity tests."""
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
