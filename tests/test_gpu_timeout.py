"""Failure detection on the GPU without a fault: the bounded wait that every
pipeline barrier of the GEMM kernels uses runs out on a barrier that nothing
arrives on (moe_testing_wait_timeout, a limit of a few milliseconds). The
kernel must record MOE_ERR_TIMEOUT in the device error word and return; the
status call reports it once, and the next calls run normally."""
import time

import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from helpers import assert_close, bits, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def test_bounded_wait_runs_out_and_the_context_stays_usable():
    import routing_grouped_gemm_score_b200 as m
    l = m.lib()
    stream = torch.cuda.current_stream().cuda_stream
    assert m.moe_get_device_status() == m.MOE_OK
    assert l.moe_testing_wait_timeout(0, stream) == m.MOE_ERR_INVALID_ARG
    assert l.moe_testing_wait_timeout(2_000_000_000, stream) == m.MOE_ERR_INVALID_ARG
    t0 = time.perf_counter()
    assert l.moe_testing_wait_timeout(5_000_000, stream) == m.MOE_OK      # 5 ms
    assert m.moe_get_device_status() == m.MOE_ERR_TIMEOUT
    elapsed = time.perf_counter() - t0
    assert elapsed < 1.0, elapsed          # it gave up at its limit, not at the kernels' 2 s
    assert m.moe_get_device_status() == m.MOE_OK                            # read once, then cleared
    # the context is usable: a whole layer runs and matches the oracle
    w = wl.WORKLOADS["tiny"]
    d = wl.make_inputs(w, "cuda")
    out = m.moe_layer_forward(d["logits"], d["x"], d["w_gate_up"], d["w_down"], w.k)
    assert m.moe_get_device_status() == m.MOE_OK
    ref = oracle.moe_forward_tokens(bits(d["x"]), d["logits"].cpu().numpy(), bits(d["w_gate_up"]),
                                    bits(d["w_down"]), w.k)
    assert_close(out, ref, "tiny layer after the timeout")
