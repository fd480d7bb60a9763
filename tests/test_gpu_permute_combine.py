"""Dispatch and combine parity on the GPU (Transformer Engine "Mixture of
Experts", Token dispatch and Token combine): permutation indices and the
permuted rows bit-exact; the weighted combine within the bf16 bound."""
import numpy as np
import pytest
import torch

import oracle
import helpers
import workloads as wl
from helpers import assert_close, assert_equal, bits, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def routed(w):
    import routing_grouped_gemm_score_b200 as m
    logits = wl.make_logits(w, "cuda")
    x = wl.make_x(w, "cuda")
    r = m.moe_router_topk(logits, w.k, m.RouterOpts(w.score, w.renormalize))
    return m, logits, x, r


@pytest.mark.parametrize("name,T,H", [("tiny", None, None), ("qwen3_30b_a3b", 4096, 2048),
                                      ("skew_t1", None, 256), ("skew_t8", None, 256),
                                      ("skew_t64", None, 2048), ("llama4_17bx16e", 1000, 5120),
                                      ("tie_t64", None, 128), ("mixtral_8x7b", 3000, 4096)])
@pytest.mark.parametrize("path", ["auto", "warp"])
def test_permute_matches_dispatch_definition(name, T, H, path, monkeypatch):
    """Both permute kernels on every shape: the default choice (the
    token-range register kernel for rows up to 4096 wide, else one warp per
    token) and the warp-per-token kernel forced."""
    helpers.force_kernels(permute=path)
    w = wl.WORKLOADS[name]
    if T is not None:
        w = w.scaled(T=T)
    if H is not None:
        w = w.scaled(H=H)
    m, logits, x, r = routed(w)
    p = m.moe_permute(x, r["topk_idx"], r["offsets"])
    torch.cuda.synchronize()
    assert m.moe_get_device_status() == 0
    st, row_of = oracle.dispatch(r["topk_idx"].cpu().numpy(), r["offsets"].cpu().numpy(), w.E)
    assert_equal(p["sorted_token"], st, "sorted_token")
    assert_equal(p["row_of"], row_of, "row_of")
    assert_equal(p["x_perm"].view(torch.int16).cpu().numpy().view(np.uint16),
                 oracle.gather_rows(bits(x), st), "x_perm")


@pytest.mark.parametrize("path", ["auto", "warp"])
def test_permute_rejects_invalid_indices_on_the_device(path, monkeypatch):
    """Bad expert indices made on the host: the kernel flags them, skips the
    rows, and the status call reports MOE_ERR_DEVICE_CHECK."""
    import routing_grouped_gemm_score_b200 as m
    helpers.force_kernels(permute=path)
    T, E, k, H = 100, 8, 2, 64
    idx = torch.randint(0, E, (T, k), dtype=torch.int32)
    idx[:, 1] = (idx[:, 0] + 1) % E
    idx[5, 0] = 11          # out of range
    idx[9, 1] = idx[9, 0]   # repeated expert
    counts = torch.bincount(idx.clamp(0, E - 1).flatten().long(), minlength=E)
    offsets = torch.zeros(E + 1, dtype=torch.int32)
    offsets[1:] = torch.cumsum(counts, 0)
    x = torch.randn((T, H), device="cuda").to(torch.bfloat16)
    p = m.moe_permute(x, idx.cuda(), offsets.cuda())
    assert m.moe_get_device_status() == 5
    ro = p["row_of"].cpu()
    assert ro[5, 0] == -1 and ro[9, 1] == -1
    assert m.moe_get_device_status() == 0          # the word was cleared


@pytest.mark.parametrize("T,k,H,shared,probs", [(64, 2, 128, False, True), (1000, 8, 2048, False, True),
                                                 (333, 1, 5120, True, True), (257, 4, 64, False, False),
                                                 (1, 8, 2048, True, True), (3000, 16, 512, True, True),
                                                 (4100, 2, 4096, False, True), (700, 8, 2112, True, True)])
def test_combine_matches_weighted_sum(T, k, H, shared, probs):
    """The warp-per-token combine on shapes from one token to 4100, k from 1
    to 16, with and without a shared row and weights; H=64 leaves most lanes
    without a chunk, and H=2112 (264 chunks) ends in a part step of the 64
    chunks a warp covers per step at k=8."""
    import routing_grouped_gemm_score_b200 as m
    g_ = torch.Generator().manual_seed(T * 7 + k)
    A = T * k
    y = torch.randn((A, H), generator=g_).to(torch.bfloat16)
    row_of = torch.randperm(A, generator=g_).to(torch.int32).reshape(T, k)
    p = torch.rand((T, k), generator=g_)
    s = torch.randn((T, H), generator=g_).to(torch.bfloat16) if shared else None
    out = m.moe_unpermute_combine(y.cuda(), row_of.cuda(), p.cuda() if probs else None,
                                  s.cuda() if shared else None)
    ref = oracle.combine(oracle.bits_to_float(bits(y)), row_of.numpy(), p.numpy() if probs else None,
                         oracle.bits_to_float(bits(s)) if shared else None)
    assert_close(out, ref, "combine")
    # bf16 output of an fp32 sum: within one bf16 rounding of the exact value
    np.testing.assert_allclose(out.double().cpu().numpy(), ref, rtol=2 ** -8, atol=1e-5)
    # deterministic: a second call gives the same bytes
    out2 = m.moe_unpermute_combine(y.cuda(), row_of.cuda(), p.cuda() if probs else None,
                                   s.cuda() if shared else None)
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
