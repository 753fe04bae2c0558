"""svdq_quantize_act (smoothing + NVFP4 quantization + low-rank down-projection)
against the oracle, through the C ABI.

Bar: E2M1 codes and E4M3 scales (the whole 128x4-layout buffer, padding
included) are bit-exact.  The down-projection x̂·L1 is compared with the
oracle's exact fp64 sum of the same bf16 products: the kernel accumulates in
fp32 (tensor-core order, then fp32 atomics across K splits), so
|err| <= K·2^-24·Σ|terms| in the worst case; the test asks for
||err||_F <= 1e-4·||ref||_F and max|err| <= 1e-3·rms(ref), a few times the
typical sqrt(K)·2^-24 and far below anything a wrong index or sign gives.
"""
import numpy as np
import pytest
import torch

import workloads
from oracle import svdq as osv
from tests._gpu import bf16, describe_byte_mismatch, f32, needs_gpu, prepared

import svdquant_w4a4_gemm_b200 as sv

pytestmark = [pytest.mark.gpu, needs_gpu]


def _run(x, L, r, dynamic, gs_val, rows=None):
    xt = bf16(x)
    s = None if L["s"] is None else f32(L["s"])
    L1t = bf16(L["L1t"][:r]) if r else None
    gs_in = None if dynamic else f32([gs_val])
    q, sf, lora, gs = sv.quantize_act(xt, s, L1t, gs_in)
    torch.cuda.synchronize()
    return q.cpu().numpy(), sf.cpu().numpy(), None if lora is None else lora.cpu().numpy(), gs.cpu().numpy()[0]


def _check(case, r, smooth=True, dynamic=False, sample_rows=None):
    d, L = prepared(case, smooth=smooth)
    x = d["x"]
    gs_ref = osv.act_tensor_scale(x, L["s"])
    q, sf, lora, gs = _run(x, L, r, dynamic, gs_ref)
    assert gs == gs_ref, (gs, gs_ref)
    ref = osv.quantize_act(x, L["s"], gs_ref)
    assert np.array_equal(sf, ref["sf_swizzled"]), "scales: " + describe_byte_mismatch(sf, ref["sf_swizzled"])
    assert np.array_equal(q, ref["packed"]), "codes: " + describe_byte_mismatch(q.ravel(), ref["packed"].ravel())
    if r:
        rows = np.arange(x.shape[0]) if sample_rows is None else sample_rows
        xl_ref = osv.lora_down(x[rows], L["s"], L["L1t"][:r])
        err = lora[rows].astype(np.float64) - xl_ref
        rms = np.sqrt(np.mean(xl_ref ** 2))
        assert np.linalg.norm(err) <= 1e-4 * np.linalg.norm(xl_ref), np.linalg.norm(err) / np.linalg.norm(xl_ref)
        assert np.abs(err).max() <= 1e-3 * rms


SMALL = [
    # (M, K, N, r, smooth, dynamic)
    (256, 512, 64, 32, True, False),      # the tiny workload's activation side
    (200, 512, 64, 16, True, True),       # ragged M, dynamic scale
    (333, 1024, 64, 64, False, False),    # no smoothing, 3 row blocks, ragged
    (128, 64, 64, 0, True, False),        # one K block, no low-rank branch
    (1, 128, 64, 128, True, True),        # a single row
    (130, 3072, 64, 32, True, False),     # one row past a block, long K
]


@pytest.mark.parametrize("M,K,N,r,smooth,dynamic", SMALL)
def test_quantize_small(M, K, N, r, smooth, dynamic):
    case = workloads.small_case(M, K, N, max(r, 16), seed=M + K)
    _check(case, r, smooth, dynamic)


def test_quantize_attn_full_size():
    _check(workloads.ATTN, 32, dynamic=False)


def test_quantize_dynamic_scale_full_size():
    _check(workloads.ATTN, 32, dynamic=True, sample_rows=np.arange(0, 4096, 17))


def test_quantize_mlp_down_full_size_sampled():
    case = workloads.MLP_DOWN
    d = workloads.draw_svdq(case)
    # the down-projection's input: only the activation side matters here, and
    # the oracle prep of a 3072 x 12288 weight is not needed for it
    rng = np.random.default_rng(0)
    s = rng.uniform(0.5, 4.0, case.K).astype(np.float32)
    L1t = workloads.to_bf16(rng.standard_normal((32, case.K)).astype(np.float32) * 0.05)
    L = dict(s=s, L1t=L1t)
    gs_ref = osv.act_tensor_scale(d["x"], s)
    q, sf, lora, gs = _run(d["x"], L, 32, False, gs_ref)
    rows = np.arange(0, case.M, 13)
    ref = osv.quantize_act(d["x"][rows], s, gs_ref)
    assert np.array_equal(q[rows], ref["packed"])
    from oracle import codecs
    got_sf = codecs.unswizzle_scales(sf, case.M, case.K // 16)[rows]
    assert np.array_equal(got_sf, ref["sf"])
    xl_ref = osv.lora_down(d["x"][rows], s, L1t)
    assert np.linalg.norm(lora[rows] - xl_ref) <= 1e-4 * np.linalg.norm(xl_ref)


# the ring depth follows K and r (as many 16 KB sub-tiles as shared memory
# holds, rounded down to an even count, at most 8): 8 at K=3072 for r <= 64,
# 6 at r=128; 6 and 4 at K=12288 for r = 64 and 128.  Repeated runs must give the same bytes every
# time: a sub-tile quantized from a slot that does not yet hold it changes
# the codes of that run only.
@pytest.mark.parametrize("M,K,r", [(4608, 3072, 128), (4608, 3072, 32), (4096, 12288, 64),
                                   (4096, 12288, 128), (1000, 3072, 0)])
def test_quantize_repeatable_at_every_ring_depth(M, K, r):
    rng = np.random.default_rng(M + K + r)
    x = workloads.to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    s = rng.uniform(0.5, 4.0, K).astype(np.float32)
    L1t = workloads.to_bf16(rng.standard_normal((max(r, 16), K)).astype(np.float32) * 0.05)
    L = dict(s=s, L1t=L1t)
    gs_ref = osv.act_tensor_scale(x, s)
    q0, sf0, lora0, _ = _run(x, L, r, False, gs_ref)
    for _ in range(8):
        q, sf, lora, _ = _run(x, L, r, False, gs_ref)
        assert np.array_equal(q, q0), "codes: " + describe_byte_mismatch(q.ravel(), q0.ravel())
        assert np.array_equal(sf, sf0), "scales: " + describe_byte_mismatch(sf, sf0)
        if r:
            assert np.abs(lora - lora0).max() <= 1e-4 * np.sqrt(np.mean(lora0.astype(np.float64) ** 2))
    rows = np.arange(0, M, 7)
    ref = osv.quantize_act(x[rows], s, gs_ref)
    assert np.array_equal(q0[rows], ref["packed"])
    from oracle import codecs
    assert np.array_equal(codecs.unswizzle_scales(sf0, M, K // 16)[rows], ref["sf"])
    if r:
        xl_ref = osv.lora_down(x[rows], s, L1t[:r])
        assert np.linalg.norm(lora0[rows] - xl_ref) <= 1e-4 * np.linalg.norm(xl_ref)


# single-pass dynamic scale: the max, a grid barrier and the quantization in
# one launch.  It must give the same bytes as the max pass + quantize path
# and the oracle's dynamic scale: small and ragged shapes, one row, several
# sub-tiles per CTA at every ring depth, and two calls in a row on one
# workspace (the call clears it).
@pytest.mark.parametrize("M,K,r,smooth", [(200, 512, 16, True), (1, 128, 128, True), (333, 1024, 0, False),
                                          (4096, 3072, 32, True), (4608, 3072, 128, True),
                                          (1000, 12288, 64, True)])
def test_single_pass_dynamic_scale(M, K, r, smooth):
    rng = np.random.default_rng(M * 3 + K + r)
    x = workloads.to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    x[rng.integers(0, M), rng.integers(0, K)] = 37.5          # one outlier sets the max
    s = rng.uniform(0.5, 4.0, K).astype(np.float32) if smooth else None
    L1t = workloads.to_bf16(rng.standard_normal((max(r, 16), K)).astype(np.float32) * 0.05)[:r] if r else None
    xt = bf16(x)
    st = None if s is None else f32(s)
    lt = bf16(L1t) if r else None
    ws = torch.empty(sv.QUANTIZE_WORKSPACE_BYTES, dtype=torch.uint8, device="cuda")
    two = [sv.quantize_act_dynamic(xt, st, lt, workspace=ws) for _ in range(2)]
    base = sv.quantize_act(xt, st, lt, None)
    torch.cuda.synchronize()
    sv.check_device_errors()
    gs_ref = osv.act_tensor_scale(x, s)
    for q, sf, lora, gs in two:
        assert gs.item() == gs_ref == base[3].item()
        assert torch.equal(q, base[0]), "codes: " + describe_byte_mismatch(q.cpu().numpy().ravel(),
                                                                          base[0].cpu().numpy().ravel())
        assert torch.equal(sf, base[1])
        if r:
            ref = base[2].double()
            assert (lora.double() - ref).norm() <= 1e-5 * ref.norm()
    rows = np.arange(0, M, 11)
    ref = osv.quantize_act(x[rows], s, gs_ref)
    assert np.array_equal(two[0][0].cpu().numpy()[rows], ref["packed"])


def test_single_pass_dynamic_scale_two_workspaces_two_streams():
    rng = np.random.default_rng(5)
    xs = [bf16(workloads.to_bf16(rng.standard_normal((2048, 3072)).astype(np.float32) * (1 + i)))
          for i in range(2)]
    streams = [torch.cuda.Stream() for _ in range(2)]
    wss = [torch.zeros(sv.QUANTIZE_WORKSPACE_BYTES, dtype=torch.uint8, device="cuda") for _ in range(2)]
    outs = [None, None]
    torch.cuda.synchronize()
    for i in range(2):
        with torch.cuda.stream(streams[i]):
            outs[i] = sv.quantize_act_dynamic(xs[i], None, None, workspace=wss[i])
    torch.cuda.synchronize()
    sv.check_device_errors()
    for i in range(2):
        base = sv.quantize_act(xs[i], None, None, None)
        torch.cuda.synchronize()
        assert torch.equal(outs[i][0], base[0]) and outs[i][3].item() == base[3].item()


def test_quantize_strided_rows_and_gs_copy():
    case = workloads.small_case(160, 256, 64, 32, seed=5)
    d, L = prepared(case)
    wide = np.zeros((160, 320), np.float32)
    wide[:, :256] = d["x"]
    xt = bf16(wide)[:, :256]
    gs_ref = osv.act_tensor_scale(d["x"], L["s"])
    gs_in = f32([gs_ref])
    gs_out = torch.zeros(1, device="cuda")
    q, sf, lora, gs = sv.quantize_act(xt, f32(L["s"]), bf16(L["L1t"]), gs_in,
                                      out=(torch.empty(160, 128, dtype=torch.uint8, device="cuda"),
                                           torch.empty(sv.scale_bytes(160, 256), dtype=torch.uint8, device="cuda"),
                                           torch.empty(160, 32, device="cuda"), gs_out))
    ref = osv.quantize_act(d["x"], L["s"], gs_ref)
    assert np.array_equal(q.cpu().numpy(), ref["packed"])
    assert gs_out.item() == gs_ref


def test_signed_zero_and_saturation_codes():
    # groups that exercise: all-zero group (scale 0, signed zeros), tiny
    # negatives that round to zero, exact E2M1 midpoints, the amax group
    x = np.zeros((128, 64), np.float32)
    x[0, :16] = -0.0
    x[1, :16] = np.linspace(-1, 1, 16)
    x[1, 3] = -1e-3
    x[2, :16] = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, 6, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5, -6]
    x[3, 16:32] = 1e-30
    x = workloads.to_bf16(x)
    L = dict(s=None, L1t=np.zeros((16, 64), np.float32))
    for gs in (np.float32(448.0), np.float32(1.0), np.float32(3.5)):
        q, sf, _, _ = _run(x, L, 0, False, gs)
        ref = osv.quantize_act(x, None, gs)
        assert np.array_equal(sf, ref["sf_swizzled"]), describe_byte_mismatch(sf, ref["sf_swizzled"])
        assert np.array_equal(q, ref["packed"]), describe_byte_mismatch(q.ravel(), ref["packed"].ravel())


@pytest.mark.parametrize("M,K,r", [(1024, 4096, 32), (640, 3072, 128), (1000, 2048, 0)])
def test_quantize_many_units_per_cta(M, K, r):
    # more 128x64 sub-tiles than SMs: every CTA walks a range that crosses
    # row blocks, so the down-projection accumulators alternate
    rng = np.random.default_rng(M + K + r)
    x = workloads.to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    s = rng.uniform(0.5, 2.0, K).astype(np.float32)
    L1t = workloads.to_bf16(rng.standard_normal((max(r, 16), K)).astype(np.float32) * 0.05)[:r]
    L = dict(s=s, L1t=L1t)
    gs_ref = osv.act_tensor_scale(x, s)
    q, sf, lora, gs = _run(x, L, r, False, gs_ref)
    ref = osv.quantize_act(x, s, gs_ref)
    assert np.array_equal(sf, ref["sf_swizzled"]), describe_byte_mismatch(sf, ref["sf_swizzled"])
    assert np.array_equal(q, ref["packed"]), describe_byte_mismatch(q.ravel(), ref["packed"].ravel())
    if r:
        xl_ref = osv.lora_down(x, s, L1t)
        assert np.linalg.norm(lora - xl_ref) <= 1e-4 * np.linalg.norm(xl_ref)
