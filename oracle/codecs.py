"""Number formats used by the method, written out from their definitions.

TEST INFRASTRUCTURE ONLY (see the package docstring).

* E2M1 (the NVFP4 element): 1 sign bit, 2 exponent bits, 1 mantissa bit.
  Magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6} are codes 0..7; bit 3 is the sign.
  Encoding rounds to the nearest magnitude, ties to the even code, and
  saturates at 6 (OCP MX v1.0 "FP4 E2M1"; NVIDIA NVFP4).  The sign bit is the
  sign of the input, so a negative value that rounds to zero encodes as 0x8.
* E4M3 "fn" (the NVFP4 block scale): bias 7, no infinities, 0x7F/0xFF are
  NaN, largest finite 448, subnormal step 2**-9 (OCP 8-bit float spec).
  Encoding rounds to nearest, ties to even, and saturates to 448.
* bf16: the upper 16 bits of an IEEE fp32 after round-to-nearest-even.
* Nibble packing: byte = code[even k] | code[odd k] << 4.
* Scale layout: the 128x4 "swizzled" block layout that cuBLAS documents for
  1-D block scaling factors and that the tcgen05 block-scaled MMA consumes:
  rows padded to 128, scale columns padded to 4, one 512-byte block per
  (128-row block, 4-column block), blocks ordered column-block fastest.
"""

import numpy as np

E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)


# ---------------------------------------------------------------- E2M1 ----
def e2m1_decode(codes):
    """Codes (uint8, low 4 bits used) -> exact float64 values."""
    codes = np.asarray(codes, dtype=np.uint8)
    mag = E2M1_MAGNITUDES[codes & 0x7]
    return np.where(codes & 0x8, -mag, mag)


def _nearest_code(a, mags):
    """Index of the nearest entry of the ascending table ``mags`` to each
    non-negative ``a`` (float64); on an exact tie the even index wins.
    Values beyond the last entry map to the last entry (saturation)."""
    hi = np.clip(np.searchsorted(mags, a, side="left"), 1, len(mags) - 1)
    lo = hi - 1
    d_lo = a - mags[lo]
    d_hi = mags[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    return np.where(a >= mags[-1], len(mags) - 1, idx)


def e2m1_encode(v):
    """float32 values -> E2M1 codes (uint8 in 0..15).

    Nearest magnitude in {0,...,6}; on an exact tie the candidate with the
    even code wins; magnitudes above 6 saturate to 6; sign bit copied from
    the input (so -0.0 and small negatives give 0x8).
    """
    v = np.asarray(v, dtype=np.float32)
    a = np.abs(v.astype(np.float64))
    code = _nearest_code(a, E2M1_MAGNITUDES).astype(np.uint8)
    sign = np.signbit(v)
    return (code | np.where(sign, np.uint8(8), np.uint8(0))).astype(np.uint8)


# ---------------------------------------------------------------- E4M3 ----
def e4m3_decode(codes):
    """E4M3fn codes -> float64 (NaN for 0x7F / 0xFF)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s = (c >> 7) & 1
    e = (c >> 3) & 0xF
    m = c & 0x7
    sub = m * 2.0 ** -9                      # e == 0: m/8 * 2^(1-7)
    nor = (1.0 + m / 8.0) * np.power(2.0, e - 7)
    val = np.where(e == 0, sub, nor)
    val = np.where((e == 0xF) & (m == 0x7), np.nan, val)
    return np.where(s == 1, -val, val)


_E4M3_POS = e4m3_decode(np.arange(0x7F, dtype=np.uint8))  # codes 0..126, finite


def e4m3_encode(v):
    """float32 values -> E4M3fn codes, round-to-nearest-even, saturating.

    Non-negative codes are in value order, so "even" is the code's low bit
    (the mantissa's last bit).  |v| >= 448 saturates to 448 (0x7E).
    """
    v = np.asarray(v, dtype=np.float32)
    a = np.abs(v.astype(np.float64))
    code = _nearest_code(a, _E4M3_POS).astype(np.uint8)
    neg = np.signbit(v) & (code != 0)
    return (code | np.where(neg, np.uint8(0x80), np.uint8(0))).astype(np.uint8)


# ---------------------------------------------------------------- bf16 ----
def bf16_round(x):
    """float32 -> float32 holding the nearest bf16 value (ties to even)."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    r = np.where(np.isnan(x), u | 0x400000, r)  # keep NaN a NaN
    return r.astype(np.uint32).view(np.float32)


def bf16_bits(x):
    """float32 holding bf16 values -> uint16 bit patterns."""
    x = np.ascontiguousarray(bf16_round(x))
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def bf16_from_bits(b):
    b = np.ascontiguousarray(np.asarray(b, dtype=np.uint16))
    return (b.astype(np.uint32) << 16).view(np.float32)


# ------------------------------------------------------------- packing ----
def pack_nibbles(codes):
    """[rows, K] codes -> [rows, K/2] bytes, even k in the low nibble."""
    codes = np.asarray(codes, dtype=np.uint8)
    assert codes.shape[-1] % 2 == 0
    lo = codes[..., 0::2] & 0xF
    hi = codes[..., 1::2] & 0xF
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_nibbles(packed):
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = packed & 0xF
    out[..., 1::2] = packed >> 4
    return out


# -------------------------------------------------------- scale layout ----
def scale_buffer_bytes(rows, n_scale_cols):
    return (-(-rows // 128) * 128) * (-(-n_scale_cols // 4) * 4)


def scale_offset(row, col, n_scale_cols):
    """Byte offset of scale (row, col) in the 128x4 block layout."""
    row = np.asarray(row, dtype=np.int64)
    col = np.asarray(col, dtype=np.int64)
    col_blocks = -(-n_scale_cols // 4)
    block = (row // 128) * col_blocks + col // 4
    inner = (row % 32) * 16 + ((row % 128) // 32) * 4 + (col % 4)
    return block * 512 + inner


def swizzle_scales(sf):
    """[rows, C] scale codes -> flat padded buffer (padding bytes zero)."""
    sf = np.asarray(sf, dtype=np.uint8)
    rows, cols = sf.shape
    out = np.zeros(scale_buffer_bytes(rows, cols), dtype=np.uint8)
    r, c = np.meshgrid(np.arange(rows), np.arange(cols), indexing="ij")
    out[scale_offset(r, c, cols)] = sf
    return out


def unswizzle_scales(buf, rows, cols):
    buf = np.asarray(buf, dtype=np.uint8)
    r, c = np.meshgrid(np.arange(rows), np.arange(cols), indexing="ij")
    return buf[scale_offset(r, c, cols)]
