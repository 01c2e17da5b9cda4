"""Failure detection on the GPU without a fault: every mbarrier wait in the tensor-core
kernel is bounded. The test hook ttq_debug_inject_stall makes the MMA thread wait on a
barrier that nothing arrives at, with a 1 ms limit; the kernel must then record
TTQ_ERR_TIMEOUT in the device error word, drain its own copies, free its tensor memory
and return, leaving the context usable for the next call."""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import online_activation_aware_b200 as ttq
from online_activation_aware_b200 import synthetic

pytestmark = pytest.mark.gpu

TIMEOUT = -6


def test_bounded_wait_reports_timeout_and_context_survives():
    T, d, d_out, q, g = 256, 1024, 512, 4, 64
    X, W = synthetic.draw_layer(T, d, d_out, seed=5)
    Xb, Wb = synthetic.as_bf16(X).cuda(), synthetic.as_bf16(W).cuda()
    cfg = ttq.make_config(q, g, 0.5, 0.4)
    good = ttq.linear_prefill(Xb, Wb, cfg)
    assert ttq.device_status() == 0
    Y_ref = good["Y"].clone()
    try:
        ttq.set_wait_limit_ns(1_000_000)
        ttq.debug_inject_stall(True)
        ttq.linear_decode(Xb, good["s"], good["codes"], good["scale"], good["zero"], cfg, d_out)
        status = ttq.device_status()
    finally:
        ttq.debug_inject_stall(False)
        ttq.set_wait_limit_ns(0)  # back to the default limit
    assert status == TIMEOUT
    assert ttq.device_status() == 0  # reading the status cleared it
    # the context still works and gives the same answer as before
    again = ttq.linear_prefill(Xb, Wb, cfg)
    assert ttq.device_status() == 0
    assert torch.equal(again["Y"], Y_ref)
