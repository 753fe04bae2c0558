"""Pins for oracle/codecs.py: format tables, brute force, library routines."""
import math

import numpy as np
import pytest
import torch

from oracle import codecs
from tests._golden import rows


# ---------------------------------------------------------------- E2M1 ----
def test_e2m1_decode_matches_printed_table():
    for code, val in rows("e2m1_table.txt"):
        got = codecs.e2m1_decode(np.array([int(code, 16)], np.uint8))[0]
        assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val))


def test_e2m1_value_set_is_the_nvfp4_set():
    mags = codecs.e2m1_decode(np.arange(8, dtype=np.uint8))
    assert list(mags) == [0, 0.5, 1, 1.5, 2, 3, 4, 6]


def test_e2m1_ties_and_saturation_match_printed_table():
    for v, code in rows("e2m1_ties.txt"):
        got = codecs.e2m1_encode(np.array([float(v)], np.float32))[0]
        assert got == int(code, 16), (v, got, code)


def test_e2m1_encode_brute_force_grid():
    # every multiple of 2^-8 in [-8, 8]: the chosen value is a nearest
    # representable one, exact ties go to the even code, beyond 6 saturates
    v = (np.arange(-8 * 256, 8 * 256 + 1) / 256.0).astype(np.float32)
    codes = codecs.e2m1_encode(v)
    got = codecs.e2m1_decode(codes)
    table = np.concatenate([codecs.E2M1_MAGNITUDES, -codecs.E2M1_MAGNITUDES])
    for vi, ci, gi in zip(v.astype(np.float64), codes, got):
        if abs(vi) > 6:
            assert abs(gi) == 6 and np.sign(gi) == np.sign(vi)
            continue
        dist = np.abs(table - vi)
        assert abs(gi - vi) == dist.min()
        n_near = len(set(np.abs(table[dist == dist.min()])))
        if n_near == 2:  # exact tie between two magnitudes
            assert (ci & 0x7) % 2 == 0
        assert bool(ci & 0x8) == bool(np.signbit(np.float32(vi)))


def test_e2m1_round_trip_and_signed_zero():
    codes = np.arange(16, dtype=np.uint8)
    vals = codecs.e2m1_decode(codes).astype(np.float32)
    back = codecs.e2m1_encode(vals)
    assert np.array_equal(back, codes)
    assert codecs.e2m1_encode(np.array([-1e-3, -0.0, 1e-3], np.float32)).tolist() == [8, 8, 0]


# ---------------------------------------------------------------- E4M3 ----
def test_e4m3_decode_matches_printed_points():
    for code, val in rows("e4m3_points.txt"):
        got = codecs.e4m3_decode(np.array([int(code, 16)], np.uint8))[0]
        if val == "nan":
            assert np.isnan(got)
        else:
            assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val))


def test_e4m3_decode_exhaustive_structure():
    v = codecs.e4m3_decode(np.arange(256, dtype=np.uint8))
    assert np.isnan(v).sum() == 2
    pos = v[:127]
    assert np.all(np.diff(pos) > 0)                       # strictly increasing
    assert np.array_equal(v[128:255], -pos)               # sign symmetry
    assert np.all(np.diff(pos[:8]) == 2.0 ** -9)          # subnormal step


def test_e4m3_round_trip_all_finite_codes():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF, 0x80)], np.uint8)
    vals = codecs.e4m3_decode(codes).astype(np.float32)
    assert np.array_equal(codecs.e4m3_encode(vals), codes)


def test_e4m3_encode_matches_torch_cast_in_range():
    rng = np.random.default_rng(5)
    v = np.concatenate([
        rng.uniform(0, 448, 20000), rng.uniform(0, 2 ** -6, 5000),   # normals, subnormals
        np.exp(rng.uniform(np.log(2 ** -12), np.log(448), 20000)),
        # exact midpoints between neighbouring codes (ties)
        (codecs.e4m3_decode(np.arange(0, 126)) + codecs.e4m3_decode(np.arange(1, 127))) / 2,
    ]).astype(np.float32)
    v = v[v <= 448]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codecs.e4m3_encode(v), ref)


def test_e4m3_saturates():
    assert codecs.e4m3_encode(np.array([448, 449, 464, 480, 1e30], np.float32)).tolist() == [0x7E] * 5


# ---------------------------------------------------------------- bf16 ----
def test_bf16_round_matches_torch_cast():
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.standard_normal(100000) * 10.0 ** rng.integers(-30, 30, 100000),
                        [0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 3.3895e38]]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(codecs.bf16_round(v).view(np.uint32), ref.view(np.uint32))


# ------------------------------------------------------------- packing ----
def test_nibble_order_even_k_low():
    assert codecs.pack_nibbles(np.array([[0x1, 0x2, 0xF, 0x0]], np.uint8)).tolist() == [[0x21, 0x0F]]
    c = np.random.default_rng(0).integers(0, 16, (7, 64)).astype(np.uint8)
    assert np.array_equal(codecs.unpack_nibbles(codecs.pack_nibbles(c)), c)


# -------------------------------------------------------- scale layout ----
@pytest.mark.parametrize("rows_,cols", [(128, 4), (256, 32), (300, 8), (4096, 192), (1, 4)])
def test_scale_layout_is_a_bijection_onto_padded_blocks(rows_, cols):
    n = codecs.scale_buffer_bytes(rows_, cols)
    rp, cp = -(-rows_ // 128) * 128, -(-cols // 4) * 4
    assert n == rp * cp
    r, c = np.meshgrid(np.arange(rp), np.arange(cp), indexing="ij")
    off = codecs.scale_offset(r, c, cols).ravel()
    assert np.array_equal(np.sort(off), np.arange(n))
    # one 512-byte block holds exactly one (128-row, 4-column) block, and the
    # 4 scales of one row inside a block are 4 consecutive bytes
    blk = off.reshape(rp, cp) // 512
    for rb in range(rp // 128):
        for cb in range(cp // 4):
            assert len(np.unique(blk[rb * 128:(rb + 1) * 128, cb * 4:(cb + 1) * 4])) == 1
    o = off.reshape(rp, cp)
    assert np.all(np.diff(o[:, :4], axis=1) == 1)
    # column blocks are the fastest-varying blocks
    if cp >= 8:
        assert o[0, 4] - o[0, 0] == 512


def test_scale_layout_matches_documented_offsets():
    """Hand-worked byte offsets from the cuBLASLt description of the 1x16
    block-scale layout (tests/golden/nvfp4_scale_layout.txt): they single out
    the order of rows inside a 16-byte line (row % 32 picks the line, row //
    32 the 4-byte word), the order of tiles (scale columns first) and the
    padding of ragged shapes, which a bijection check cannot tell apart."""
    pts = rows("nvfp4_scale_layout.txt")
    assert len(pts) >= 15
    for n_rows, n_cols, r, c, off in pts:
        got = int(codecs.scale_offset(int(r), int(c), int(n_cols)))
        assert got == int(off), (n_rows, n_cols, r, c, got, off)
        assert got < codecs.scale_buffer_bytes(int(n_rows), int(n_cols))


def test_swizzle_round_trip_and_zero_padding():
    sf = np.random.default_rng(2).integers(1, 255, (130, 12)).astype(np.uint8)
    buf = codecs.swizzle_scales(sf)
    assert np.array_equal(codecs.unswizzle_scales(buf, 130, 12), sf)
    assert (buf != 0).sum() == sf.size
