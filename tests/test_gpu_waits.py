"""Bounded in-kernel waits on the GPU: with the host-side fault hook the
GEMM's producer never fills one ring slot, so the MMA thread's wait for it
runs out after the (shortened) limit; every role of the kernel gives up its
own wait, drains its in-flight copies, frees its tensor memory and returns.
The host then reads SVDQ_ERR_DEVICE_TIMEOUT, and the context stays usable:
a normal call right after gives the right answer.  The same for the grid
barrier of the single-pass dynamic quantize: the first CTA skips its
arrival and the others' bounded waits run out.  Nothing traps or faults."""
import numpy as np
import pytest
import torch

import workloads
from oracle import svdq as osv
from tests._gpu import assert_gemm_close, bf16, f32, needs_gpu, prepared, u8, weights_from_layer

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


def test_grid_barrier_wait_times_out_cleanly_and_context_survives():
    rng = np.random.default_rng(8)
    x = bf16(workloads.to_bf16(rng.standard_normal((1024, 1024)).astype(np.float32)))
    L1t = bf16(workloads.to_bf16(rng.standard_normal((32, 1024)).astype(np.float32) * 0.05))
    sv.check_device_errors()
    prev_t = sv.set_wait_timeout_ns(50_000_000)   # 50 ms
    prev_f = sv.lib().svdq_debug_set_fault(2)
    try:
        sv.quantize_act_dynamic(x, None, L1t)
        with pytest.raises(sv.SvdqError) as e:
            sv.check_device_errors()
        assert e.value.status == sv.DEVICE_TIMEOUT
        word = int(str(e.value).split("device error word ")[1].split()[0], 16)
        assert word & 16, hex(word)                # the grid barrier gave up
    finally:
        sv.lib().svdq_debug_set_fault(prev_f)
        sv.set_wait_timeout_ns(prev_t)
    sv.check_device_errors()
    q, sf, lora, gs = sv.quantize_act_dynamic(x, None, L1t)
    base = sv.quantize_act(x, None, L1t, None)
    torch.cuda.synchronize()
    assert torch.equal(q, base[0]) and torch.equal(sf, base[1]) and gs.item() == base[3].item()
