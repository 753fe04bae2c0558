"""Programmatic dependent launch (svdq_set_pdl, on by default): a kernel of
the library may be scheduled while the previous one on the stream is still
finishing, and waits for it (griddepcontrol.wait) before it touches global
memory.  These chains put every hazard that could break on the overlapped
launches, through the C ABI:
  * K1 -> K2 -> K1 -> ... on one set of q / scale / xl buffers: K2 reads what
    K1 wrote (read after write) and the next K1 overwrites what K2 is reading
    (write after read);
  * AWQ layers with N = K, each reading the previous one's output.
With r = 0 and for AWQ the kernels are deterministic, so the chains must give
the same bytes with PDL on and off; with the low-rank branch, xl is summed
with float atomics in an order that varies from run to run, so each output
is held to the oracle's result instead.
"""
import numpy as np
import pytest
import torch

import workloads
from oracle import prep, svdq as osv
from tests._gpu import assert_gemm_close, bf16, f16, f32, needs_gpu, prepared, weights_from_layer

import svdquant_w4a4_gemm_b200 as sv

pytestmark = [pytest.mark.gpu, needs_gpu]


def _inputs(d, n):
    """n different activations of the layer's distribution (column rolls)."""
    return [np.roll(d["x"], 17 * i, axis=1) for i in range(n)]


def _svdq_chain(case, pdl, xs):
    d, L = prepared(case)
    w = weights_from_layer(L)
    M, K, r = case.M, case.K, case.r
    gss = [f32([osv.act_tensor_scale(x, L["s"])]) for x in xs]   # each input's static scale
    q = torch.empty(M, K // 2, dtype=torch.uint8, device="cuda")
    sf = torch.empty(sv.scale_bytes(M, K), dtype=torch.uint8, device="cuda")
    xl = torch.empty(M, r, device="cuda") if r else None
    gso = torch.empty(1, device="cuda")
    xs_dev = [bf16(x) for x in xs]
    torch.cuda.synchronize()
    prev = sv.set_pdl(pdl)
    try:
        ys = []
        for x, gs in zip(xs_dev, gss):
            sv.quantize_act(x, w.smooth, w.L1t if r else None, gs, out=(q, sf, xl, gso))
            ys.append(sv.w4a4_linear(q, sf, gso, xl, w))
        torch.cuda.synchronize()
    finally:
        sv.set_pdl(prev)
    sv.check_device_errors()
    return ys, L


def test_set_pdl_returns_the_previous_setting():
    prev = sv.set_pdl(False)
    try:
        assert sv.set_pdl(True) is False
        assert sv.set_pdl(True) is True
    finally:
        sv.set_pdl(prev)


def test_quantize_gemm_chain_without_low_rank_is_identical_with_and_without_pdl():
    case = workloads.small_case(512, 1024, 768, 0, seed=31)
    d, _ = prepared(case)
    xs = _inputs(d, 6)
    on, _ = _svdq_chain(case, True, xs)
    off, _ = _svdq_chain(case, False, xs)
    for i, (a, b) in enumerate(zip(on, off)):
        assert torch.equal(a, b), f"step {i}: PDL changed the output"


def test_quantize_gemm_chain_with_low_rank_matches_the_oracle_under_pdl():
    case = workloads.small_case(384, 1024, 576, 32, seed=32)
    d, _ = prepared(case)
    xs = _inputs(d, 4)
    ys, L = _svdq_chain(case, True, xs)
    for i, (x, y) in enumerate(zip(xs, ys)):
        assert_gemm_close(y, osv.svdq_forward(x, L)["y"], f"PDL chain step {i}")


def _awq_chain(pdl, layers, x):
    prev = sv.set_pdl(pdl)
    try:
        outs, h = [], x
        for (ainv, qw, sc, z, b) in layers:
            h = sv.awq_w4a16_linear(h, ainv, qw, sc, z, b)
            outs.append(h)
        torch.cuda.synchronize()
    finally:
        sv.set_pdl(prev)
    sv.check_device_errors()
    return outs


@pytest.mark.parametrize("M,K", [(1, 1024), (6, 3072), (3, 320)])
def test_awq_layer_chain_is_identical_with_and_without_pdl(M, K):
    """Each layer reads the previous layer's output (N = K): the streaming
    kernel (K = 1024, 3072) and the register-streaming kernel (K = 320)."""
    layers = []
    for i in range(4):
        d = workloads.draw_awq(workloads.AwqCase(f"chain {i}", M, K, K, seed=60 + i))
        L = prep.prepare_awq_layer(d["x_cal"], d["W"], d["bias"])
        layers.append((f32(L["act_scale_inv"]), torch.from_numpy(L["qweight"].view(np.int32)).cuda(),
                       f16(L["sc"]), f16(L["z"]), bf16(L["bias"])))
    x = bf16(workloads.draw_awq(workloads.AwqCase("chain x", M, K, K, seed=59))["x"])
    on = _awq_chain(True, layers, x)
    off = _awq_chain(False, layers, x)
    for i, (a, b) in enumerate(zip(on, off)):
        assert torch.isfinite(a.float()).all()
        assert torch.equal(a, b), f"layer {i}: PDL changed the output"
