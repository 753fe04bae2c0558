"""Python binding of libsvdq.so, the B200 (sm_100a) SVDQuant W4A4 / AWQ W4A16
linear library.  Argument marshalling only: every step of the layer runs in
the library's CUDA kernels; torch provides device memory and the stream.

    q, sf, lora, gs = quantize_act(x, smooth, L1t, gscale)    # one pass over x
    q, sf, lora, gs = quantize_act_dynamic(x, smooth, L1t)    # gs_a from x, same launch
    y = w4a4_linear(q, sf, gs, lora, layer)                   # FP4 GEMM + low-rank + bias
    h = w4a4_linear(q, sf, gs, lora, up_layer, act="gelu")    # ... + GELU(tanh) epilogue
    q_, k_, v_ = w4a4_linear_split(q, sf, gs, lora, qkv_layer, parts=3)  # fused QKV
    y = awq_w4a16_linear(x, act_scale_inv, qweight, scales, zeros, bias)

The C ABI (include/svdq.h) is also exposed raw as ``lib()`` for callers that
manage their own buffers.  Importing this module never falls back to another
implementation: if the library is missing, ``lib()`` raises.
"""
import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libsvdq.so")

OK, INVALID_ARG, MISALIGNED, UNSUPPORTED_DEVICE, CUDA, DEVICE_TIMEOUT, NOT_IMPLEMENTED = range(7)

_lib = None

_vp, _i64, _int, _sz, _u64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint64

_SIGNATURES = {
    "svdq_version": (_int, []),
    "svdq_status_string": (ctypes.c_char_p, [_int]),
    "svdq_last_error_detail": (ctypes.c_char_p, []),
    "svdq_nvfp4_scale_bytes": (_sz, [_i64, _i64]),
    "svdq_quantize_act": (_int, [_vp, _i64, _i64, _i64, _vp, _vp, _int, _vp, _vp, _vp, _vp, _vp, _vp]),
    "svdq_quantize_act_dynamic": (_int, [_vp, _i64, _i64, _i64, _vp, _vp, _int, _vp, _vp, _vp, _vp,
                                         _vp, _vp]),
    "svdq_quantize_act_dynamic_noalloc": (_int, [_vp, _i64, _i64, _i64, _vp, _vp, _int, _vp, _vp,
                                                 _vp, _vp, _vp]),
    "svdq_w4a4_linear": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _int, _vp,
                                _i64, _i64, _i64, _vp, _i64, _vp]),
    "svdq_w4a4_linear_act": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _int, _vp,
                                    _i64, _i64, _i64, _vp, _i64, _int, _vp]),
    "svdq_w4a4_linear_split": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _int, _vp,
                                      _i64, _i64, _i64, _int, _vp, _i64, _int, _vp]),
    "awq_w4a16_linear": (_int, [_vp, _i64, _i64, _vp, _vp, _vp, _vp, _int, _vp, _i64, _vp, _vp]),
    "svdq_check_device_errors": (_int, [_vp]),
    "svdq_set_wait_timeout_ns": (_u64, [_u64]),
    "svdq_set_gemm_pairs": (_int, [_int]),
    "svdq_set_pdl": (_int, [_int]),
    "svdq_debug_set_fault": (_int, [_int]),
}


class SvdqError(RuntimeError):
    def __init__(self, status, detail):
        super().__init__(f"svdq status {status}: {detail}")
        self.status = status
        self.detail = detail


def lib():
    """The loaded libsvdq.so (built by ``svdquant_w4a4_gemm_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m svdquant_w4a4_gemm_b200.build` "
                               "(there is no fallback implementation)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(status):
    if status != OK:
        raise SvdqError(status, lib().svdq_last_error_detail().decode())


def _require(cond, what):
    # argument checks the C ABI cannot make (dtypes, strides); explicit, so
    # that they hold under ``python -O`` too
    if not cond:
        raise ValueError(what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def scale_bytes(rows, K):
    return int(lib().svdq_nvfp4_scale_bytes(rows, K))


def check_device_errors(device=None):
    _check(lib().svdq_check_device_errors(_stream(device)))


def set_wait_timeout_ns(ns):
    return int(lib().svdq_set_wait_timeout_ns(ns))


def set_gemm_pairs(enable):
    """SM-pair (2-CTA, 256-row) tiles for the W4A4 GEMM where the shape allows
    (default off: one-SM tiles measured faster on B200); returns the previous
    setting."""
    return bool(lib().svdq_set_gemm_pairs(1 if enable else 0))


def set_pdl(enable):
    """Programmatic dependent launch for later launches (default on: a kernel
    sets up while the previous one finishes, then waits for it before touching
    any operand); returns the previous setting."""
    return bool(lib().svdq_set_pdl(1 if enable else 0))


def quantize_act(x, smooth=None, L1t=None, gscale=None, *, out=None):
    """Smoothing + NVFP4 quantization + low-rank down-projection of x [M, K] bf16.

    smooth: [K] fp32 s (or None); L1t: [r, K] bf16 (or None); gscale: fp32
    scalar tensor (static) or None (dynamic).  Returns (q [M, K/2] uint8,
    sf (scale bytes) uint8, lora [M, r] fp32 or None, gs fp32 [1]).
    ``out`` may pass preallocated (q, sf, lora, gs).
    """
    _require(x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1,
             "x must be a 2-D bf16 tensor with unit column stride")
    M, K = x.shape
    r = 0 if L1t is None else L1t.shape[0]
    dev = x.device
    if out is None:
        q = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
        sf = torch.empty((scale_bytes(M, K),), dtype=torch.uint8, device=dev)
        lora = torch.empty((M, r), dtype=torch.float32, device=dev) if r else None
        gs = torch.empty((1,), dtype=torch.float32, device=dev)
    else:
        q, sf, lora, gs = out
    _check(lib().svdq_quantize_act(_ptr(x), M, K, x.stride(0), _ptr(smooth), _ptr(L1t), r,
                                   _ptr(gscale), _ptr(gs), _ptr(q), _ptr(sf), _ptr(lora), _stream(dev)))
    return q, sf, lora, gs


QUANTIZE_WORKSPACE_BYTES = 16


def quantize_act_dynamic(x, smooth=None, L1t=None, *, out=None, workspace=None):
    """quantize_act with the dynamic tensor scale computed in the same kernel
    (one cooperative launch with a grid barrier).  ``workspace``: a device
    buffer of at least QUANTIZE_WORKSPACE_BYTES bytes, 16-byte aligned (one is
    allocated if None); calls that may overlap on the GPU need their own."""
    _require(x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1,
             "x must be a 2-D bf16 tensor with unit column stride")
    M, K = x.shape
    r = 0 if L1t is None else L1t.shape[0]
    dev = x.device
    if out is None:
        q = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
        sf = torch.empty((scale_bytes(M, K),), dtype=torch.uint8, device=dev)
        lora = torch.empty((M, r), dtype=torch.float32, device=dev) if r else None
        gs = torch.empty((1,), dtype=torch.float32, device=dev)
    else:
        q, sf, lora, gs = out
    if workspace is None:
        workspace = torch.empty((QUANTIZE_WORKSPACE_BYTES,), dtype=torch.uint8, device=dev)
    _require(workspace.numel() * workspace.element_size() >= QUANTIZE_WORKSPACE_BYTES,
             f"workspace must hold at least {QUANTIZE_WORKSPACE_BYTES} bytes")
    _check(lib().svdq_quantize_act_dynamic(_ptr(x), M, K, x.stride(0), _ptr(smooth), _ptr(L1t), r,
                                           _ptr(gs), _ptr(workspace), _ptr(q), _ptr(sf), _ptr(lora),
                                           _stream(dev)))
    return q, sf, lora, gs


@dataclass
class SvdqWeights:
    """Prepared weights of one W4A4 layer (all on the device)."""
    q_w: torch.Tensor          # [N, K/2] uint8 E2M1 codes of the residual
    sf_w: torch.Tensor         # scale bytes, 128x4 block layout
    gs_w: torch.Tensor         # fp32 [1]
    L1t: torch.Tensor          # [r, K] bf16 (or [0, K])
    L2t: torch.Tensor          # [N, r] bf16 (or [N, 0])
    smooth: torch.Tensor       # [K] fp32 or None
    bias: torch.Tensor         # [N] bf16 or None

    @property
    def rank(self):
        return self.L1t.shape[0]

    @property
    def N(self):
        return self.q_w.shape[0]

    @property
    def K(self):
        return self.q_w.shape[1] * 2


ACT_NONE, ACT_GELU_TANH = 0, 1
_ACTS = {None: ACT_NONE, "gelu": ACT_GELU_TANH}


def w4a4_linear(q, sf, gs_a, lora, w: SvdqWeights, *, y=None, act=None):
    """y [M, N] bf16 = act(dec(q)·dec(W)ᵀ + lora·L2 + bias); act None or "gelu" (tanh form)."""
    _require(act in _ACTS, f"act={act!r} must be None or 'gelu'")
    M, K = q.shape[0], q.shape[1] * 2
    N, r = w.N, w.rank
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=q.device)
    _check(lib().svdq_w4a4_linear_act(_ptr(q), _ptr(sf), _ptr(gs_a), _ptr(lora) if r else None,
                                      _ptr(w.q_w), _ptr(w.sf_w), _ptr(w.gs_w),
                                      _ptr(w.L2t) if r else None, r, _ptr(w.bias), M, N, K,
                                      _ptr(y), y.stride(0), _ACTS[act], _stream(q.device)))
    return y


def w4a4_linear_split(q, sf, gs_a, lora, w: SvdqWeights, parts=3, *, ys=None, act=None):
    """The fused projection stored as ``parts`` outputs [M, N/parts] bf16 (Q, K, V of a
    fused QKV projection): columns [i·N/parts, (i+1)·N/parts) of y go to ys[i]."""
    _require(act in _ACTS, f"act={act!r} must be None or 'gelu'")
    M, K = q.shape[0], q.shape[1] * 2
    N, r = w.N, w.rank
    n_part = N // parts
    if ys is None:
        ys = [torch.empty((M, n_part), dtype=torch.bfloat16, device=q.device) for _ in range(parts)]
    ys = list(ys)
    ldy = ys[0].stride(0)
    _require(len(ys) == parts and all(t.stride(0) == ldy and t.stride(1) == 1 for t in ys),
             "ys must be `parts` row-major tensors with one leading dimension")
    arr = (_vp * parts)(*[_ptr(t) for t in ys])
    _check(lib().svdq_w4a4_linear_split(_ptr(q), _ptr(sf), _ptr(gs_a), _ptr(lora) if r else None,
                                        _ptr(w.q_w), _ptr(w.sf_w), _ptr(w.gs_w),
                                        _ptr(w.L2t) if r else None, r, _ptr(w.bias), M, N, K, parts,
                                        ctypes.cast(arr, _vp), ldy, _ACTS[act], _stream(q.device)))
    return tuple(ys)


def svdq_linear(x, w: SvdqWeights, gscale=None, act=None):
    """The whole layer: quantize_act then w4a4_linear (two kernels, same stream)."""
    q, sf, lora, gs = quantize_act(x, w.smooth, w.L1t if w.rank else None, gscale)
    return w4a4_linear(q, sf, gs, lora, w, act=act)


def awq_w4a16_linear(x, act_scale_inv, qweight, scales, zeros, bias=None, *, y=None, group=64):
    """y [M, N] bf16 for x [M <= 8, K] bf16 and int4 weights [N, K/8] uint32 (as int32)."""
    _require(x.dtype == torch.bfloat16 and x.is_contiguous(), "x must be a contiguous bf16 tensor")
    M, K = x.shape
    N = qweight.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _check(lib().awq_w4a16_linear(_ptr(x), M, K, _ptr(act_scale_inv), _ptr(qweight), _ptr(scales),
                                  _ptr(zeros), group, _ptr(bias), N, _ptr(y), _stream(x.device)))
    return y
