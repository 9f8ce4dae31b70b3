"""Failure detection on the GPU without a fault (the layer's bounded waits).

Every wait in the kernels gives up after a bounded time, records a timeout in
the workspace's error word and returns; moe_device_status reports it.  The
self-test kernel runs two waits that nothing satisfies (an mbarrier without
arrivals, a flag nothing sets) through the same primitives; here the report,
its clearing, and a correct forward on the same context afterwards are checked.
"""
import time

import pytest
import torch

import oracle
import mixture_experts_layer_logits_b200 as moe
from mixture_experts_layer_logits_b200 import workloads as wl

from parity import assert_out_close, host_bits, host_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_lib():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for -m gpu tests")
    from mixture_experts_layer_logits_b200 import build

    build.build()
    moe.load_library()


def test_bounded_wait_reports_timeout_and_context_survives():
    w = wl.WORKLOADS["tiny"]
    ws = moe.workspace(w.T, w.E, w.k, w.H, w.I)
    assert moe.moe_device_status(ws) in (moe.MOE_OK, moe.MOE_ERR_DEVICE_TIMEOUT)  # clear
    t0 = time.perf_counter()
    moe.moe_selftest_wait_timeout(ws, limit_us=20000)
    status = moe.moe_device_status(ws)
    elapsed = time.perf_counter() - t0
    assert status == moe.MOE_ERR_DEVICE_TIMEOUT
    assert elapsed < 2.0                      # gave up after ~20 ms, did not hang
    assert moe.moe_device_status(ws) == moe.MOE_OK  # reading the status cleared it

    # the context and the workspace are still good for the real layer
    d = wl.make_inputs(w, seed=21, device="cuda")
    out = moe.moe_forward(d["x"], d["logits"], d["w13"], d["w2"], w.k, ws=ws)
    assert moe.moe_device_status(ws) == moe.MOE_OK
    ref = oracle.forward(host_bits(d["x"]), host_f32(d["logits"]), host_bits(d["w13"]),
                         host_bits(d["w2"]), w.k)
    assert_out_close(out, ref["out"])
