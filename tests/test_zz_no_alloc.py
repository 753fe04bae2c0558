"""svdq_quantize_act_dynamic_noalloc through the C ABI.

This entry point serves callers that cannot allocate device memory when they
call the library (an inference-engine plugin whose enqueue step must not
allocate, a runtime that plans all of its memory ahead): they have no
workspace to give svdq_quantize_act_dynamic, so this variant keeps the
kernel's scratch in a static device array.  Its outputs are checked against
svdq_quantize_act_dynamic with a caller workspace, on two calls in a row:
codes, scales and gs_a bit-exact, xl within the 1e-5 relative Frobenius
bound the other single-pass tests use (fp32 atomics across CTAs).

The file name makes pytest collect it last; it passes alone in a fresh
process as well as after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads
from tests._gpu import bf16, f32, needs_gpu

import svdquant_w4a4_gemm_b200 as sv

pytestmark = [pytest.mark.gpu, needs_gpu]


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(x, s, L1t):
    M, K = x.shape
    r = 0 if L1t is None else L1t.shape[0]
    q = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
    sf = torch.empty((sv.scale_bytes(M, K),), dtype=torch.uint8, device="cuda")
    lora = torch.empty((M, r), dtype=torch.float32, device="cuda") if r else None
    gs = torch.empty((1,), dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = sv.lib().svdq_quantize_act_dynamic_noalloc(_p(x), M, K, x.stride(0), _p(s), _p(L1t), r, _p(gs),
                                                    _p(q), _p(sf), _p(lora), stream)
    assert st == sv.OK, sv.lib().svdq_last_error_detail()
    return q, sf, lora, gs


@pytest.mark.parametrize("M,K,r", [(4096, 3072, 32), (333, 1024, 0), (1000, 12288, 128)])
def test_noalloc_matches_the_workspace_entry_point_twice(M, K, r):
    rng = np.random.default_rng(M + K + r)
    x = workloads.to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    x[rng.integers(0, M), rng.integers(0, K)] = -51.0
    xt = bf16(x)
    s = f32(rng.uniform(0.5, 4.0, K).astype(np.float32))
    L1t = bf16(workloads.to_bf16(rng.standard_normal((r, K)).astype(np.float32) * 0.05)) if r else None
    ref = sv.quantize_act_dynamic(xt, s, L1t)
    got = [_noalloc(xt, s, L1t) for _ in range(2)]
    torch.cuda.synchronize()
    sv.check_device_errors()
    for q, sf, lora, gs in got:
        assert gs.item() == ref[3].item()
        assert torch.equal(q, ref[0])
        assert torch.equal(sf, ref[1])
        if r:
            assert (lora.double() - ref[2].double()).norm() <= 1e-5 * ref[2].double().norm()
