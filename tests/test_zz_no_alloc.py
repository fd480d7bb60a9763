"""moe_router_topk_noalloc, the routing entry point that takes no workspace.

It exists for callers that cannot allocate device memory while they route,
such as a serving runtime that hands out all device memory from its own pool
at start-up. It must give the same routing as moe_router_topk. Both are
called through the C ABI on caller-owned buffers, twice in a row: the second
call reuses the library's fixed scratch array, which still holds the first
call's contents.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as wl
from helpers import assert_equal, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _buffers(T, E, k):
    dev = "cuda"
    return {"topk_idx": torch.full((T, k), -7, dtype=torch.int32, device=dev),
            "topk_prob": torch.full((T, k), -1.0, dtype=torch.float32, device=dev),
            "routing_map": torch.full((T, E), 9, dtype=torch.uint8, device=dev),
            "counts": torch.full((E,), -7, dtype=torch.int32, device=dev),
            "offsets": torch.full((E + 1,), -7, dtype=torch.int32, device=dev)}


def _route(fn_name, logits, k, opts, with_workspace):
    import routing_grouped_gemm_score_b200 as m
    l = m.lib()
    T, E = logits.shape
    b = _buffers(T, E, k)
    args = [logits.data_ptr(), T, E, k, ctypes.byref(opts), b["topk_idx"].data_ptr(),
            b["topk_prob"].data_ptr(), b["routing_map"].data_ptr(), b["counts"].data_ptr(),
            b["offsets"].data_ptr()]
    stream = torch.cuda.current_stream().cuda_stream
    if with_workspace:
        ws = torch.empty(l.moe_router_workspace_size(T, E, k), dtype=torch.uint8, device="cuda")
        rc = getattr(l, fn_name)(*args, ws.data_ptr(), ws.numel(), stream)
    else:
        rc = getattr(l, fn_name)(*args, stream)
    assert rc == 0, m.moe_status_string(rc)
    torch.cuda.synchronize()
    assert m.moe_get_device_status() == 0
    return b


def test_noalloc_router_matches_workspace_router_twice():
    import routing_grouped_gemm_score_b200 as m
    cases = [  # two calls in a row, with different shapes, scores and options
        (wl.make_logits(wl.WORKLOADS["qwen3_30b_a3b"], "cuda"), 8, m.RouterOpts()),
        (wl.make_logits(wl.WORKLOADS["llama4_17bx16e"].scaled(T=3000), "cuda"), 1,
         m.RouterOpts(m.SCORE_SIGMOID, False)),
        (wl.make_logits(wl.WORKLOADS["skew_t16384"], "cuda"), 8, m.RouterOpts(scaling=1.5)),
    ]
    for logits, k, opts in cases:
        oc = opts.c()
        ref = _route("moe_router_topk", logits, k, oc, True)
        got = _route("moe_router_topk_noalloc", logits, k, oc, False)
        for key in ("topk_idx", "routing_map", "counts", "offsets"):
            assert_equal(got[key], ref[key].cpu().numpy(), key)
        np.testing.assert_allclose(got["topk_prob"].cpu().numpy(), ref["topk_prob"].cpu().numpy(),
                                   rtol=1e-6, atol=0)


def test_noalloc_router_at_its_limit():
    """T = 32768 tokens at E = 256, k = 8: the largest call the fixed scratch
    admits (T * k at its limit, the scratch filled to within a few KiB), on
    the router kernel that large batches use. Bit-exact against the
    workspace router; one token more is rejected before any launch."""
    import routing_grouped_gemm_score_b200 as m
    T, E, k = 32768, 256, 8
    g = torch.Generator(device="cuda").manual_seed(4242)
    logits = torch.randn((T, E), generator=g, device="cuda")
    oc = m.RouterOpts().c()
    ref = _route("moe_router_topk", logits, k, oc, True)
    got = _route("moe_router_topk_noalloc", logits, k, oc, False)
    for key in ("topk_idx", "routing_map", "counts", "offsets", "topk_prob"):
        assert torch.equal(got[key], ref[key]), key
    b = _buffers(1, E, k)
    rc = m.lib().moe_router_topk_noalloc(logits.data_ptr(), T + 1, E, k, ctypes.byref(oc),
                                         b["topk_idx"].data_ptr(), b["topk_prob"].data_ptr(), None,
                                         b["counts"].data_ptr(), b["offsets"].data_ptr(),
                                         torch.cuda.current_stream().cuda_stream)
    assert rc == 2      # MOE_ERR_UNSUPPORTED
    assert torch.all(b["counts"] == -7)


def test_noalloc_router_rejects_sizes_beyond_its_scratch():
    import routing_grouped_gemm_score_b200 as m
    l = m.lib()
    oc = m.RouterOpts().c()
    T, E, k = 40000, 8, 2          # more tokens than the fixed scratch holds
    b = _buffers(1, E, k)
    rc = l.moe_router_topk_noalloc(b["topk_prob"].data_ptr(), T, E, k, ctypes.byref(oc),
                                   b["topk_idx"].data_ptr(), b["topk_prob"].data_ptr(), None,
                                   b["counts"].data_ptr(), b["offsets"].data_ptr(),
                                   torch.cuda.current_stream().cuda_stream)
    assert rc == 2      # MOE_ERR_UNSUPPORTED, returned before any launch
    rc = l.moe_router_topk_noalloc(b["topk_prob"].data_ptr(), 20000, 128, 16, ctypes.byref(oc),
                                   b["topk_idx"].data_ptr(), b["topk_prob"].data_ptr(), None,
                                   b["counts"].data_ptr(), b["offsets"].data_ptr(),
                                   torch.cuda.current_stream().cuda_stream)
    assert rc == 2      # T * k above the limit
    assert torch.all(b["counts"] == -7)     # nothing was written
