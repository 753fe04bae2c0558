"""SVDQuant W4A4 (NVFP4) linear, step by step on the CPU.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The method, as the pages state it ("Bringing Nunchaku 4-bit Diffusion
Inference to Diffusers"; blog.margrop.com "技术细节 §1", the SVDQuant list;
ainews.surl.tw paragraph 2):

1. activation outliers are moved into the weights: the activation is
   divided channel-wise by a smoothing vector s and the weight multiplied
   by it, so the layer computes x·diag(1/s) against diag(s)·W;
2. the hardest part of the smoothed weight is a 16-bit rank-r branch
   L1·L2 (down-projection L1, up-projection L2);
3. the residual R = smoothed weight − L1·L2 is quantized to 4 bits, and so
   is the smoothed activation (W4A4; NVFP4 on Blackwell);
4. the down-projection x̂·L1 runs beside the activation quantization and
   the up-projection (x̂·L1)·L2 is added to the 4-bit product.

So y = Q4(x̂)·Q4(R)ᵀ + (x̂·L1)·L2 + b with x̂ = x·diag(1/s).

Readings where the pages are silent:
* smoothing multiplies by inv_s = RN_fp32(1/s) rather than dividing per
  element (the same operator, one rounding fewer per element);
* the activation tensor scale is gs_a = 2688 / amax(x̂) = 448·6/amax
  (1 when amax is 0); static: passed in;
* the down-projection contracts bf16(x̂) with the bf16 factor (16-bit
  branch) and accumulates exactly here (fp64);
* every quantization step is a separate IEEE fp32 operation, in this order:
  a = max|x̂| over 16 elements; t = (a / 6) · gs; sf = E4M3(t);
  d = dec(sf); if d == 0 every code is a signed zero, otherwise
  inv = gs / d and code = E2M1(x̂ · inv).
"""

import numpy as np

from . import codecs

GROUP = 16
E4M3_MAX = np.float32(448.0)
E2M1_MAX = np.float32(6.0)
TENSOR_SCALE_NUM = np.float32(448.0 * 6.0)  # 2688


def inv_smooth(s, K):
    """RN_fp32(1/s_k); None means no smoothing (all ones)."""
    if s is None:
        return np.ones(K, dtype=np.float32)
    s = np.asarray(s, dtype=np.float32)
    return (np.float32(1.0) / s).astype(np.float32)


def smooth(x, s):
    """x̂ = fp32(x) · inv_s, one fp32 rounding per element."""
    x = np.asarray(x, dtype=np.float32)
    return (x * inv_smooth(s, x.shape[-1])[None, :]).astype(np.float32)


def tensor_scale(amax):
    """gs = 2688 / amax in fp32, or 1 when amax == 0."""
    amax = np.float32(amax)
    if amax == 0:
        return np.float32(1.0)
    with np.errstate(over="ignore", divide="ignore"):
        return np.float32(TENSOR_SCALE_NUM / amax)


def act_tensor_scale(x, s):
    """The dynamic activation scale: 2688 / max|x̂| over the whole tensor."""
    xh = smooth(x, s)
    return tensor_scale(np.abs(xh).max() if xh.size else np.float32(0))


def nvfp4_quantize(xh, gs):
    """Quantize fp32 rows [R, K] (K % 16 == 0) with tensor scale gs.

    Returns (codes [R, K] uint8 unpacked, sf [R, K/16] uint8 E4M3 codes).
    """
    xh = np.asarray(xh, dtype=np.float32)
    gs = np.float32(gs)
    R, K = xh.shape
    assert K % GROUP == 0
    g = xh.reshape(R, K // GROUP, GROUP)
    a = np.abs(g).max(axis=-1).astype(np.float32)             # group amax
    t = ((a / np.float32(6.0)).astype(np.float32) * gs).astype(np.float32)
    sf = codecs.e4m3_encode(t)                                # E4M3 RNE sat
    d = codecs.e4m3_decode(sf).astype(np.float32)             # exact
    with np.errstate(divide="ignore", invalid="ignore"):
        inv = np.where(d == 0, np.float32(0), (gs / d)).astype(np.float32)
    v = (g * inv[..., None]).astype(np.float32)
    codes = codecs.e2m1_encode(v)
    # zero scale: every code is a zero that keeps the input's sign
    zero = np.where(np.signbit(g), np.uint8(8), np.uint8(0)).astype(np.uint8)
    codes = np.where((d == 0)[..., None], zero, codes).astype(np.uint8)
    return codes.reshape(R, K), sf


def nvfp4_dequantize(codes, sf, gs):
    """codes [R, K], sf [R, K/16] -> fp64 values e2m1·dec(sf)/gs."""
    codes = np.asarray(codes, dtype=np.uint8)
    R, K = codes.shape
    val = codecs.e2m1_decode(codes).reshape(R, K // GROUP, GROUP)
    scale = codecs.e4m3_decode(sf)[..., None]
    return (val * scale / np.float64(np.float32(gs))).reshape(R, K)


def quantize_act(x, s, gs=None):
    """The activation side of the layer (the quantize call).

    x: [M, K] bf16 values (as float32); s: [K] smoothing vector or None;
    gs: fp32 tensor scale or None for the dynamic one.
    Returns dict(codes, sf, packed, sf_swizzled, gs, xh).
    """
    xh = smooth(x, s)
    if gs is None:
        gs = tensor_scale(np.abs(xh).max() if xh.size else np.float32(0))
    codes, sf = nvfp4_quantize(xh, gs)
    return dict(codes=codes, sf=sf, packed=codecs.pack_nibbles(codes),
                sf_swizzled=codecs.swizzle_scales(sf), gs=np.float32(gs), xh=xh)


def lora_down(x, s, L1t):
    """x̂·L1 with bf16(x̂) and the bf16 factor L1ᵀ [r, K], exact in fp64."""
    xh16 = codecs.bf16_round(smooth(x, s)).astype(np.float64)
    return xh16 @ np.asarray(L1t, dtype=np.float64).T


def gelu_tanh(v):
    """GELU in its tanh form, 0.5·v·(1 + tanh(√(2/π)·(v + 0.044715·v³))), in fp64.

    The MLP up-projection of a DiT block is followed by GELU(tanh); the
    original engine fuses it into the GEMM (blog.margrop.com "技术细节 §2",
    its per-architecture GELU/MLP fusion), which saves one round trip of
    the layer's output through HBM.
    """
    v = np.asarray(v, dtype=np.float64)
    return 0.5 * v * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (v + 0.044715 * v * v * v)))


def svdq_linear(codes_a, sf_a, gs_a, xl, codes_w, sf_w, gs_w, L2t, bias, act=None):
    """y = act(deq(A)·deq(W)ᵀ + xl·L2 + b), all in fp64; act None or "gelu".

    codes_a [M, K], sf_a [M, K/16]; codes_w [N, K], sf_w [N, K/16];
    xl [M, r] (fp64 or fp32); L2t = L2ᵀ stored [N, r]; bias [N] or None.
    """
    A = nvfp4_dequantize(codes_a, sf_a, gs_a)
    W = nvfp4_dequantize(codes_w, sf_w, gs_w)
    y = A @ W.T
    if L2t is not None and np.asarray(L2t).size:
        y = y + np.asarray(xl, dtype=np.float64) @ np.asarray(L2t, dtype=np.float64).T
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    if act == "gelu":
        y = gelu_tanh(y)
    elif act is not None:
        raise ValueError(f"unknown activation {act!r}")
    return y


def svdq_forward(x, layer, gs_a=None, act=None):
    """Whole layer from a bf16 activation: quantize, down-proj, GEMM (+ act).

    ``layer`` is the dict that ``oracle.prep.prepare_svdq_layer`` returns.
    """
    q = quantize_act(x, layer["s"], gs_a)
    r = layer["L1t"].shape[0]
    xl = lora_down(x, layer["s"], layer["L1t"]) if r else np.zeros((x.shape[0], 0))
    y = svdq_linear(q["codes"], q["sf"], q["gs"], xl, layer["codes_w"], layer["sf_w"],
                    layer["gs_w"], layer["L2t"] if r else None, layer["bias"], act=act)
    return dict(y=y, xl=xl, **q)
