"""Boundary behaviour on the GPU: errors before launch leave outputs
untouched, calls are capturable in a CUDA graph and replay to the same
result, and the device error word starts clear."""
import numpy as np
import pytest
import torch

import workloads
from oracle import svdq as osv
from tests._gpu import bf16, f32, needs_gpu, prepared, weights_from_layer

import svdquant_w4a4_gemm_b200 as sv

pytestmark = [pytest.mark.gpu, needs_gpu]


def test_error_word_clear_after_normal_calls():
    case = workloads.small_case(128, 256, 256, 32, seed=1)
    d, L = prepared(case)
    sv.svdq_linear(bf16(d["x"]), weights_from_layer(L), None)
    sv.check_device_errors()


def test_invalid_call_writes_nothing():
    x = torch.randn(64, 128, device="cuda").to(torch.bfloat16)
    q = torch.full((64, 64), 0xAB, dtype=torch.uint8, device="cuda")
    sf = torch.full((sv.scale_bytes(64, 128),), 0xCD, dtype=torch.uint8, device="cuda")
    gs = torch.ones(1, device="cuda")
    with pytest.raises(sv.SvdqError) as e:
        sv.quantize_act(x, None, torch.zeros(24, 128, dtype=torch.bfloat16, device="cuda"), gs,
                        out=(q, sf, torch.zeros(64, 24, device="cuda"), gs))
    assert e.value.status == sv.INVALID_ARG
    torch.cuda.synchronize()
    assert (q == 0xAB).all() and (sf == 0xCD).all()


def test_misaligned_operand_is_rejected():
    x = torch.randn(64, 136, device="cuda").to(torch.bfloat16)[:, 4:132]   # 8-byte offset
    with pytest.raises(sv.SvdqError) as e:
        sv.quantize_act(x, None, None, torch.ones(1, device="cuda"))
    assert e.value.status in (sv.MISALIGNED, sv.INVALID_ARG)


def test_cuda_graph_capture_and_replay():
    case = workloads.small_case(256, 512, 512, 32, seed=2)
    d, L = prepared(case)
    w = weights_from_layer(L)
    x = bf16(d["x"])
    gs = f32([osv.act_tensor_scale(d["x"], L["s"])])
    y_eager = sv.svdq_linear(x, w, gs).clone()
    M, K, N, r = 256, 512, 512, 32
    q = torch.empty(M, K // 2, dtype=torch.uint8, device="cuda")
    sf = torch.empty(sv.scale_bytes(M, K), dtype=torch.uint8, device="cuda")
    lora = torch.empty(M, r, device="cuda")
    gso = torch.empty(1, device="cuda")
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):   # warm-up on the capture stream
        sv.quantize_act(x, w.smooth, w.L1t, gs, out=(q, sf, lora, gso))
        sv.w4a4_linear(q, sf, gso, lora, w, y=y)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        sv.quantize_act(x, w.smooth, w.L1t, gs, out=(q, sf, lora, gso))
        sv.w4a4_linear(q, sf, gso, lora, w, y=y)
    y.zero_()
    g.replay()
    torch.cuda.synchronize()
    # the down-projection's K-split partial sums meet in fp32 atomics, so
    # the order can differ between runs: compare within fp32 noise
    assert torch.allclose(y.float(), y_eager.float(), rtol=1e-2, atol=1e-3)
    del g
