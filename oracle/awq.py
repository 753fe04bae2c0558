"""AWQ W4A16 linear (int4 weights, 16-bit activations), on the CPU.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The pages use this kernel family for the modulation (adaLN) layers, which
are precision-sensitive or memory-bound (ainews.surl.tw paragraph 2;
app.hamidun.com "Что такое Nunchaku и SVDQuant"; keryc.com "Nunchaku Lite:
integración y modelo de ejecución", awq_w4a16 family).  They do not give the
arithmetic; the plain reading used here:

* weights are asymmetric int4 per (output row n, group of 64 along K):
  w ≈ (q − z)·sc with sc, z stored in fp16 (z holds an integer 0..15);
* the AWQ per-input-channel scale a is folded into the weights offline
  (W̃ = W·diag(a)) and undone on the activation at run time (x·diag(1/a));
* y = (x·diag(1/a))·deq(W̃)ᵀ + b.
"""

import numpy as np

GROUP = 64


def int4_quantize(w, group=GROUP):
    """Asymmetric int4 per (row, group): returns q [N,K] uint8, sc, z [N,K/g] fp16.

    sc = fp16((max − min)/15) (1 when max == min or when that rounds to 0);
    z = fp16(clamp(rint(−min/sc), 0, 15)); q = clamp(rint(w/sc) + z, 0, 15);
    rint is round-half-even; the divisions use sc's fp16 value.
    """
    w = np.asarray(w, dtype=np.float64)
    N, K = w.shape
    assert K % group == 0
    g = w.reshape(N, K // group, group)
    mn = g.min(axis=-1)
    mx = g.max(axis=-1)
    sc = ((mx - mn) / 15.0).astype(np.float16)
    sc = np.where((mx == mn) | (sc == 0), np.float16(1.0), sc).astype(np.float16)
    sc64 = sc.astype(np.float64)
    z = np.clip(np.rint(-mn / sc64), 0, 15).astype(np.float16)
    q = np.clip(np.rint(g / sc64[..., None]) + z.astype(np.float64)[..., None], 0, 15)
    return q.astype(np.uint8).reshape(N, K), sc, z


def int4_dequantize(q, sc, z, group=GROUP):
    q = np.asarray(q, dtype=np.float64)
    N, K = q.shape
    g = q.reshape(N, K // group, group)
    out = (g - z.astype(np.float64)[..., None]) * sc.astype(np.float64)[..., None]
    return out.reshape(N, K)


def pack_int4_words(q):
    """[N, K] nibbles -> [N, K/8] uint32, nibble j of a word is k % 8 == j."""
    q = np.asarray(q, dtype=np.uint32)
    N, K = q.shape
    assert K % 8 == 0
    g = q.reshape(N, K // 8, 8)
    shifts = (4 * np.arange(8, dtype=np.uint32))[None, None, :]
    return np.bitwise_or.reduce(g << shifts, axis=-1).astype(np.uint32)


def unpack_int4_words(words, K):
    w = np.asarray(words, dtype=np.uint32)
    shifts = (4 * np.arange(8, dtype=np.uint32))[None, None, :]
    return ((w[..., None] >> shifts) & 0xF).astype(np.uint8).reshape(w.shape[0], K)


def awq_linear(x, act_scale_inv, q, sc, z, bias, group=GROUP):
    """y = (x ⊙ act_scale_inv)·deq(q, sc, z)ᵀ + b in fp64.

    x: [M, K] bf16 values; act_scale_inv: [K] (the fp32 values the kernel
    receives) or None; q: [N, K] nibbles; sc, z: [N, K/group] fp16.
    """
    xf = np.asarray(x, dtype=np.float64)
    if act_scale_inv is not None:
        xf = xf * np.asarray(act_scale_inv, dtype=np.float32).astype(np.float64)[None, :]
    y = xf @ int4_dequantize(q, sc, z, group).T
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    return y
