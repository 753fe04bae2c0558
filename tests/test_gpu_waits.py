"""Bounded in-kernel waits on the GPU: with the host-side fault hook the
GEMM's producer never fills one ring slot, so the MMA thread's wait for it
runs out after the (shortened) limit; every role of the kernel gives up its
own wait, drains its in-flight copies, frees its tensor memory and returns.
The host then reads SVDQ_ERR_DEVICE_TIMEOUT, and the context stays usable:
a normal call right after gives the right answer.  Nothing traps or faults."""
import numpy as np
import pytest
import torch

import workloads
from oracle import svdq as osv
from tests._gpu import assert_gemm_close, f32, needs_gpu, prepared, u8, weights_from_layer

import svdquant_w4a4_gemm_b200 as sv

pytestmark = [pytest.mark.gpu, needs_gpu]


def test_gemm_wait_times_out_cleanly_and_context_survives():
    case = workloads.small_case(256, 512, 512, 32, seed=21)
    d, L = prepared(case)
    out = osv.svdq_forward(d["x"], L)
    w = weights_from_layer(L)
    args = (u8(out["packed"]), u8(out["sf_swizzled"]), f32([out["gs"]]), f32(out["xl"]), w)
    sv.check_device_errors()                      # start clean
    prev_t = sv.set_wait_timeout_ns(50_000_000)   # 50 ms
    prev_f = sv.lib().svdq_debug_set_fault(1)
    try:
        sv.w4a4_linear(*args)
        with pytest.raises(sv.SvdqError) as e:
            sv.check_device_errors()
        assert e.value.status == sv.DEVICE_TIMEOUT
    finally:
        sv.lib().svdq_debug_set_fault(prev_f)
        sv.set_wait_timeout_ns(prev_t)
    sv.check_device_errors()                      # the word was cleared
    y = sv.w4a4_linear(*args)
    torch.cuda.synchronize()
    assert_gemm_close(y, out["y"], "after a timed-out launch")
