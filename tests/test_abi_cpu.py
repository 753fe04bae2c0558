"""CPU-side checks of the C ABI: the library loads, exports every function
that include/svdq.h declares, and its host-only paths (validation, the
device-capability check override, the scale-size helper) behave as the
header says.  No kernel is launched here."""
import ctypes
import os
import re

import pytest

import svdquant_w4a4_gemm_b200 as sv
from oracle import codecs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "svdq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(\w+)\s*\(", src)) - {"defined"})


def test_library_exports_every_declared_function():
    L = sv.lib()
    names = _declared_functions()
    assert {"svdq_quantize_act", "svdq_w4a4_linear", "svdq_w4a4_linear_act",
            "awq_w4a16_linear"} <= set(names)
    for n in names:
        assert hasattr(L, n), n


def test_every_declared_function_has_its_doc_comment():
    # the header is the boundary's documentation: each entry point comes right
    # after the comment that states its operation, layouts, ownership and errors
    lines = open(os.path.join(ROOT, "include", "svdq.h")).read().splitlines()
    in_comment, seen = False, set()
    for i, line in enumerate(lines):
        if in_comment:
            in_comment = "*/" not in line
            continue
        if line.lstrip().startswith("/*"):
            in_comment = "*/" not in line
            continue
        m = re.match(r"^[A-Za-z_].*?\b((?:svdq|awq)_\w+)\s*\(", line)
        if not m or line.startswith("#"):
            continue
        j = i - 1
        while j >= 0 and (not lines[j].strip() or lines[j].startswith("#define") or lines[j].startswith("enum")):
            j -= 1
        assert lines[j].rstrip().endswith("*/"), f"{m.group(1)} has no doc comment"
        seen.add(m.group(1))
    assert set(_declared_functions()) <= seen


def test_binding_types_every_declared_function():
    # a ctypes call without argtypes would pass 64-bit pointers and sizes as C ints
    assert set(_declared_functions()) <= set(sv._SIGNATURES)


def test_status_strings_and_version():
    L = sv.lib()
    assert L.svdq_version() >= 100
    for s in range(7):
        assert L.svdq_status_string(s)
    assert L.svdq_status_string(99) == b"unknown status"


@pytest.mark.parametrize("rows,K", [(1, 64), (128, 64), (129, 128), (4096, 3072), (300, 12288)])
def test_scale_bytes_matches_layout(rows, K):
    assert sv.scale_bytes(rows, K) == codecs.scale_buffer_bytes(rows, K // 16)


def _q(**kw):
    a = dict(x=16, M=4, K=64, ldx=64, s=None, L1t=None, r=0, gs=16, gso=None, q=16, sf=16, lora=None)
    a.update(kw)
    v = lambda p: None if p is None else ctypes.c_void_p(p)
    return sv.lib().svdq_quantize_act(v(a["x"]), a["M"], a["K"], a["ldx"], v(a["s"]), v(a["L1t"]), a["r"],
                                      v(a["gs"]), v(a["gso"]), v(a["q"]), v(a["sf"]), v(a["lora"]), None)


def test_quantize_validation_is_host_side():
    assert _q(x=None) == sv.INVALID_ARG
    assert _q(K=96) == sv.INVALID_ARG
    assert _q(M=0) == sv.INVALID_ARG
    assert _q(ldx=60) == sv.INVALID_ARG
    assert _q(r=24) == sv.INVALID_ARG
    assert _q(r=32) == sv.INVALID_ARG          # needs L1t and lora
    assert _q(gs=None) == sv.INVALID_ARG       # dynamic needs gs_out
    assert _q(K=96) == sv.INVALID_ARG
    assert b"K=96" in sv.lib().svdq_last_error_detail()
    assert _q(x=24) == sv.MISALIGNED
    assert b"aligned" in sv.lib().svdq_last_error_detail()
    assert _q(s=18) == sv.MISALIGNED           # smooth_s: 4-byte alignment, as the header states


def test_smooth_s_needs_only_4_byte_alignment(monkeypatch):
    # a forced unsupported capability stops the call at the device check,
    # after validation and before any launch, on any machine
    monkeypatch.setenv("SVDQ_TEST_FORCE_CC", "9.0")
    assert _q(s=20) == sv.UNSUPPORTED_DEVICE
    assert _q(s=18) == sv.MISALIGNED


# The largest K the quantize call accepts at each rank (its kernel's shared
# memory), as include/svdq.h states them.
QUANT_KMAX = {0: 47360, 16: 46336, 32: 45312, 64: 43264, 128: 39168}


@pytest.mark.parametrize("r", sorted(QUANT_KMAX))
def test_quantize_k_limit_per_rank_is_the_headers(r, monkeypatch):
    # a forced unsupported capability stops a valid call at the device check
    monkeypatch.setenv("SVDQ_TEST_FORCE_CC", "9.0")
    kmax = QUANT_KMAX[r]
    lr = dict(L1t=16, lora=16) if r else {}
    assert _q(K=kmax, ldx=kmax, r=r, **lr) == sv.UNSUPPORTED_DEVICE
    assert _q(K=kmax + 64, ldx=kmax + 64, r=r, **lr) == sv.INVALID_ARG
    assert f"K <= {kmax} at r={r}".encode() in sv.lib().svdq_last_error_detail()
    with open(os.path.join(ROOT, "include", "svdq.h")) as f:
        assert str(kmax) in f.read()


def test_size_ceilings_are_validated(monkeypatch):
    monkeypatch.setenv("SVDQ_TEST_FORCE_CC", "9.0")
    assert _q(M=1 << 30) == sv.UNSUPPORTED_DEVICE
    assert _q(M=(1 << 30) + 1) == sv.INVALID_ARG
    L = sv.lib()
    v = ctypes.c_void_p

    def lin(M, N, K):
        return L.svdq_w4a4_linear(v(16), v(16), v(16), None, v(16), v(16), v(16), None, 0, None,
                                  M, N, K, v(16), N, None)
    assert lin(4, 32, 1 << 20) == sv.UNSUPPORTED_DEVICE
    assert lin(4, 32, (1 << 20) + 64) == sv.INVALID_ARG
    assert lin((1 << 30) + 1, 32, 64) == sv.INVALID_ARG
    assert lin(4, (1 << 30) + 16, 64) == sv.INVALID_ARG


def test_single_pass_dynamic_quantize_validation_is_host_side():
    L = sv.lib()
    v = ctypes.c_void_p
    st = L.svdq_quantize_act_dynamic(v(16), 4, 64, 64, None, None, 0, v(16), None, v(16), v(16), None, None)
    assert st == sv.INVALID_ARG and b"workspace" in L.svdq_last_error_detail()
    st = L.svdq_quantize_act_dynamic(v(16), 4, 64, 64, None, None, 0, None, v(16), v(16), v(16), None, None)
    assert st == sv.INVALID_ARG
    st = L.svdq_quantize_act_dynamic(v(16), 4, 64, 64, None, None, 0, v(16), v(24), v(16), v(16), None, None)
    assert st == sv.MISALIGNED
    st = L.svdq_quantize_act_dynamic(v(16), 4, 96, 96, None, None, 0, v(16), v(16), v(16), v(16), None, None)
    assert st == sv.INVALID_ARG  # K % 64
    st = L.svdq_quantize_act_dynamic_noalloc(v(16), 4, 64, 64, None, None, 0, None, v(16), v(16), None, None)
    assert st == sv.INVALID_ARG and b"act_gscale_out" in L.svdq_last_error_detail()


def test_linear_and_awq_validation_is_host_side():
    L = sv.lib()
    v = ctypes.c_void_p
    st = L.svdq_w4a4_linear(v(16), v(16), v(16), None, v(16), v(16), v(16), None, 0, None,
                            4, 24, 64, v(16), 24, None)
    assert st == sv.INVALID_ARG  # N % 16
    st = L.svdq_w4a4_linear(v(16), v(16), v(16), None, v(16), v(16), v(16), None, 0, None,
                            4, 32, 64, v(16), 30, None)
    assert st == sv.INVALID_ARG  # ldy % 8
    st = L.svdq_w4a4_linear_act(v(16), v(16), v(16), None, v(16), v(16), v(16), None, 0, None,
                                4, 32, 64, v(16), 32, 2, None)
    assert st == sv.INVALID_ARG  # unknown activation
    assert b"activation=2" in L.svdq_last_error_detail()
    ys = (v * 3)(v(16), v(16), v(16))
    st = L.svdq_w4a4_linear_split(v(16), v(16), v(16), None, v(16), v(16), v(16), None, 0, None,
                                  4, 384, 64, 4, ctypes.cast(ys, v), 128, 0, None)
    assert st == sv.INVALID_ARG and b"parts=4" in L.svdq_last_error_detail()
    st = L.svdq_w4a4_linear_split(v(16), v(16), v(16), None, v(16), v(16), v(16), None, 0, None,
                                  4, 192, 64, 3, ctypes.cast(ys, v), 64, 0, None)
    assert st == sv.INVALID_ARG and b"multiple of 128" in L.svdq_last_error_detail()
    ys_null = (v * 3)(v(16), None, v(16))
    st = L.svdq_w4a4_linear_split(v(16), v(16), v(16), None, v(16), v(16), v(16), None, 0, None,
                                  4, 384, 64, 3, ctypes.cast(ys_null, v), 128, 0, None)
    assert st == sv.INVALID_ARG and b"y_parts[1]" in L.svdq_last_error_detail()
    st = L.svdq_w4a4_linear_split(v(16), v(16), v(16), None, v(16), v(16), v(16), None, 0, None,
                                  4, 384, 64, 3, ctypes.cast(ys, v), 120, 0, None)
    assert st == sv.INVALID_ARG  # ldy < N/parts
    st = L.awq_w4a16_linear(v(16), 9, 64, None, v(16), v(16), v(16), 64, None, 32, v(16), None)
    assert st == sv.INVALID_ARG  # M > 8
    st = L.awq_w4a16_linear(v(16), 1, 64, None, v(16), v(16), v(16), 128, None, 32, v(16), None)
    assert st == sv.INVALID_ARG  # group
    st = L.awq_w4a16_linear(v(16), 8, 8192, None, v(16), v(16), v(16), 64, None, 32, v(16), None)
    assert st == sv.INVALID_ARG  # K too large for the B table at M > 4
    assert b"K=8192" in L.svdq_last_error_detail()
    st = L.awq_w4a16_linear(v(16), 4, 14464, None, v(16), v(16), v(16), 64, None, 32, v(16), None)
    assert st == sv.INVALID_ARG  # K over the M <= 4 limit


def test_unsupported_device_is_a_clear_error(monkeypatch):
    monkeypatch.setenv("SVDQ_TEST_FORCE_CC", "9.0")
    assert _q() == sv.UNSUPPORTED_DEVICE
    assert b"9.0" in sv.lib().svdq_last_error_detail()
    monkeypatch.setenv("SVDQ_TEST_FORCE_CC", "7.0")
    st = sv.lib().awq_w4a16_linear(ctypes.c_void_p(16), 1, 64, None, ctypes.c_void_p(16), ctypes.c_void_p(16),
                                   ctypes.c_void_p(16), 64, None, 32, ctypes.c_void_p(16), None)
    assert st == sv.UNSUPPORTED_DEVICE


def test_wait_timeout_setter_round_trips():
    L = sv.lib()
    prev = L.svdq_set_wait_timeout_ns(12345)
    assert L.svdq_set_wait_timeout_ns(0) == 12345
    # 0 restores the documented default of 2 s
    assert L.svdq_set_wait_timeout_ns(prev) == 2_000_000_000


def test_launch_switches_round_trip_and_normalise():
    """svdq_set_pdl and svdq_set_gemm_pairs are host-only: they return the
    previous setting and store any non-zero value as 1 (defaults: PDL on,
    pairs off)."""
    L = sv.lib()
    for setter, default in ((L.svdq_set_pdl, 1), (L.svdq_set_gemm_pairs, 0)):
        prev = setter(7)
        try:
            assert prev == default
            assert setter(0) == 1
            assert setter(0) == 0
        finally:
            setter(prev)
    # the Python wrappers report booleans
    prev = sv.set_pdl(False)
    try:
        assert sv.set_pdl(True) is False
    finally:
        sv.set_pdl(prev)
