"""The C-ABI library: it builds for sm_100a, loads without a GPU, exports
every entry point that include/moe_b200.h declares, and rejects bad
arguments before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")


@pytest.fixture(scope="session")
def built():
    from routing_grouped_gemm_score_b200 import build
    return build.build()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", text)))


def test_header_declares_the_stage_calls():
    names = declared_functions()
    for n in ("moe_router_topk", "moe_permute", "moe_grouped_mlp", "moe_unpermute_combine",
              "moe_layer_forward", "moe_grouped_mlp_backward", "moe_get_device_status",
              "moe_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(built):
    l = ctypes.CDLL(built)
    missing = [n for n in declared_functions() if not hasattr(l, n)]
    assert not missing, missing


def test_binding_covers_the_header(built):
    import routing_grouped_gemm_score_b200 as m
    assert set(m.ABI_FUNCTIONS) == set(declared_functions())
    for n in declared_functions():
        if not n.endswith("_workspace_size") and n != "moe_status_string":
            assert callable(getattr(m, n, None)) or n in ("moe_get_device_status",)


def test_status_strings(built):
    import routing_grouped_gemm_score_b200 as m
    assert m.moe_status_string(0) == "MOE_OK"
    assert "INVALID_ARG" in m.moe_status_string(1)
    assert "TIMEOUT" in m.moe_status_string(6)


def test_invalid_arguments_are_rejected_without_a_device(built):
    import routing_grouped_gemm_score_b200 as m
    l = m.lib()
    fake = 1 << 20          # a non-null, aligned, never dereferenced address
    opts = m.RouterOpts().c()
    # E out of range, k > E, k > 16, negative T
    for T, E, k in ((10, 0, 1), (10, 4, 5), (10, 300, 2), (10, 32, 17), (-1, 8, 2)):
        rc = l.moe_router_topk(fake, T, E, k, ctypes.byref(opts), fake, fake, None, fake, fake,
                               fake, 1 << 20, None)
        assert rc == 1, (T, E, k)
    # unaligned pointer
    assert l.moe_router_topk(fake + 4, 10, 8, 2, ctypes.byref(opts), fake, fake, None, fake, fake,
                             fake, 1 << 20, None) == 1
    # expert bias with a softmax score
    bad = m.RouterOpts(score_fn=m.SCORE_SOFTMAX).c()
    bad.expert_bias = fake
    assert l.moe_router_topk(fake, 10, 8, 2, ctypes.byref(bad), fake, fake, None, fake, fake,
                             fake, 1 << 20, None) == 1
    # workspace too small
    assert l.moe_router_topk(fake, 10, 8, 2, ctypes.byref(opts), fake, fake, None, fake, fake,
                             fake, 16, None) == 4
    # grouped MLP: H or I not a multiple of 8 is outside the kernels' limits
    assert l.moe_grouped_mlp(fake, 100, fake, 8, 100, 128, fake, fake, fake, None, None, fake,
                             1 << 30, None) == 2
    assert l.moe_grouped_mlp(fake, 100, fake, 8, 128, 100, fake, fake, fake, None, None, fake,
                             1 << 30, None) == 2
    # missing output
    assert l.moe_grouped_mlp(fake, 100, fake, 8, 128, 128, fake, fake, None, None, None, fake,
                             1 << 30, None) == 1
    # T * k overflowing int32
    assert l.moe_permute(fake, 1 << 29, 128, fake, 8, fake, 128, fake, fake, fake, fake, 1 << 30,
                         None) == 1
    # combine: k > 16
    assert l.moe_unpermute_combine(fake, fake, fake, 10, 17, 128, None, fake, None) == 1
    # layer: shared gate_up without shared down
    assert l.moe_layer_forward(fake, fake, 10, 128, 128, 8, 2, ctypes.byref(opts), fake, fake,
                               fake, None, fake, None, None, None, None, None, None, None, None,
                               None, fake, 1 << 30, None) == 1
    # aux loss: T = 0 (the loss divides by T^2), an unknown score function, a
    # workspace too small, no loss output
    assert l.moe_aux_loss(fake, 0, 8, 2, 0, fake, ctypes.c_float(0.01), fake, None, fake, 1 << 20, None) == 1
    assert l.moe_aux_loss(fake, 10, 8, 2, 7, fake, ctypes.c_float(0.01), fake, None, fake, 1 << 20, None) == 1
    assert l.moe_aux_loss(fake, 10, 8, 2, 0, fake, ctypes.c_float(0.01), fake, None, fake, 16, None) == 4
    assert l.moe_aux_loss(fake, 10, 8, 2, 0, fake, ctypes.c_float(0.01), None, None, fake, 1 << 20, None) == 1
    assert l.moe_aux_loss_backward(fake, 10, 8, 9, 0, fake, ctypes.c_float(0.01), None, fake, 0, None) == 1
    # backward: a missing saved tensor
    assert l.moe_grouped_mlp_backward(fake, 10, 128, 128, 8, 2, fake, fake, fake, fake, fake, fake,
                                      None, fake, fake, fake, fake, fake, fake, fake, 1 << 30,
                                      None) == 1
    # ScaledSwiGLU backward: fewer rows than assignments, a missing sorted_token,
    # a workspace too small, I not a multiple of 8
    sb = l.moe_grouped_mlp_scaled_backward
    assert sb(fake, 10, 128, 128, 8, 2, fake, fake, fake, fake, fake, fake, 19, fake, fake, fake,
              fake, fake, fake, fake, fake, 1 << 30, None) == 1
    assert sb(fake, 10, 128, 128, 8, 2, fake, fake, fake, None, fake, fake, 20, fake, fake, fake,
              fake, fake, fake, fake, fake, 1 << 30, None) == 1
    assert sb(fake, 10, 128, 128, 8, 2, fake, fake, fake, fake, fake, fake, 20, fake, fake, fake,
              fake, fake, fake, fake, fake, 16, None) == 4
    assert sb(fake, 10, 128, 100, 8, 2, fake, fake, fake, fake, fake, fake, 20, fake, fake, fake,
              fake, fake, fake, fake, fake, 1 << 30, None) == 2


def test_workspace_sizes_are_consistent(built):
    import routing_grouped_gemm_score_b200 as m
    l = m.lib()
    assert l.moe_router_workspace_size(4096, 128, 8) > 4096 * 8 * 4
    assert l.moe_router_workspace_size(10, 0, 1) == 0
    # aux loss: E fp32 values per block (one block per 32 tokens, at most 1024
    # blocks) and a ticket
    assert l.moe_aux_loss_workspace_size(4096, 128) >= 128 * 128 * 4
    assert l.moe_aux_loss_workspace_size(1 << 24, 256) <= 1024 * 256 * 4 + 512
    assert l.moe_aux_loss_workspace_size(0, 8) == 0
    a = l.moe_layer_forward_workspace_size(4096, 2048, 768, 128, 8, 0)
    b = l.moe_layer_forward_workspace_size(4096, 2048, 768, 128, 8, 1)
    A = 4096 * 8
    assert a >= A * 2048 * 2 * 2 + A * 768 * 2
    assert b > a
    assert l.moe_grouped_mlp_backward_workspace_size(4096, 2048, 768, 128, 8) >= A * (2048 * 4 + 1536 * 2)
    # dy, dgu, dx_perm and the fp32 partials of dprob (one per 64 columns of I)
    assert l.moe_grouped_mlp_scaled_backward_workspace_size(A, 2048, 768) >= A * (2048 * 4 + 1536 * 2 + 12 * 4)
    assert l.moe_grouped_mlp_scaled_backward_workspace_size(A, 2048, 100) == 0
