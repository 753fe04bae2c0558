"""Pins for oracle/awq.py and the AWQ part of oracle/prep.py."""
import numpy as np
import pytest

import workloads
from oracle import awq, prep


def test_q_equal_z_gives_bias_only():
    N, K, M = 8, 128, 3
    q = np.full((N, K), 9, np.uint8)
    z = np.full((N, K // 64), 9, np.float16)
    sc = np.random.default_rng(0).uniform(0.001, 1, (N, K // 64)).astype(np.float16)
    x = np.random.default_rng(1).standard_normal((M, K)).astype(np.float32)
    b = np.arange(N, dtype=np.float32)
    y = awq.awq_linear(x, None, q, sc, z, b)
    assert np.array_equal(y, np.broadcast_to(b.astype(np.float64), (M, N)))


def test_gemv_equals_double_loop():
    rng = np.random.default_rng(2)
    M, K, N = 2, 128, 3
    q = rng.integers(0, 16, (N, K)).astype(np.uint8)
    sc = rng.uniform(0.001, 0.1, (N, 2)).astype(np.float16)
    z = rng.integers(0, 16, (N, 2)).astype(np.float16)
    x = workloads.to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    ainv = rng.uniform(0.5, 2, K).astype(np.float32)
    b = rng.standard_normal(N).astype(np.float32)
    y = awq.awq_linear(x, ainv, q, sc, z, b)
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += float(x[m, k]) * float(ainv[k]) * (int(q[n, k]) - float(z[n, k // 64])) * float(sc[n, k // 64])
            assert y[m, n] == pytest.approx(acc + float(b[n]), rel=1e-12, abs=1e-12)


def test_int4_quantization_error_bound_and_range():
    w = np.random.default_rng(3).standard_normal((16, 256)) * 0.02
    q, sc, z = awq.int4_quantize(w)
    assert q.max() <= 15 and np.all(z.astype(np.float64) == np.rint(z.astype(np.float64)))
    deq = awq.int4_dequantize(q, sc, z)
    step = np.repeat(sc.astype(np.float64), 64, axis=1)
    # within half a step, plus the fp16 rounding of the step and the zero
    # point's clamp to [0, 15] can cost at most one more step at the edges
    assert np.all(np.abs(deq - w) <= 1.01 * step)
    assert np.mean(np.abs(deq - w) <= 0.5 * step + 1e-12) > 0.95


def _awq_groups_by_hand():
    from tests._golden import rows
    groups, cur = [], None
    for r in rows("awq_groups_by_hand.txt"):
        if r[0] == "case":
            kv = dict(t.split("=", 1) for t in r[2:])
            cur = dict(name=r[1], sc=float(kv["sc"]), z=int(kv["z"]), w=[], q=[])
            groups.append(cur)
        else:
            cur["w"].append(float(r[0]))
            cur["q"].append(int(r[1]))
    return groups


@pytest.mark.parametrize("g", _awq_groups_by_hand(), ids=lambda g: g["name"])
def test_int4_quantize_matches_hand_quantized_groups(g):
    # a scale exact in fp16 with ties in both directions, and one that fp16
    # rounds (moving a value off a tie): pins the zero point's sign, the
    # half-to-even rounding and that the divisions use the stored fp16 scale
    w = np.zeros((1, 64))
    n = len(g["w"])
    w[0, :n] = g["w"]
    q, sc, z = awq.int4_quantize(w)
    assert float(sc[0, 0]) == g["sc"] and float(z[0, 0]) == g["z"]
    assert q[0, :n].tolist() == g["q"]
    assert np.all(q[0, n:] == g["z"])


def test_constant_group_uses_unit_scale():
    w = np.full((1, 64), 3.0)
    q, sc, z = awq.int4_quantize(w)
    assert sc[0, 0] == 1.0 and z[0, 0] == 0 and np.all(q == 3)
    assert np.all(awq.int4_dequantize(q, sc, z) == 3.0)


def test_word_packing_nibble_j_is_k_mod_8():
    q = np.zeros((1, 16), np.uint8)
    q[0, 3] = 0xA
    q[0, 8] = 0x5
    words = awq.pack_int4_words(q)
    assert words.tolist() == [[0xA000, 0x5]]
    rq = np.random.default_rng(4).integers(0, 16, (5, 64)).astype(np.uint8)
    assert np.array_equal(awq.unpack_int4_words(awq.pack_int4_words(rq), 64), rq)


def test_awq_scale_folding_preserves_the_layer():
    case = workloads.AwqCase("t", 2, 256, 64)
    d = workloads.draw_awq(case)
    L = prep.prepare_awq_layer(d["x_cal"], d["W"], d["bias"])
    a = L["a"]
    assert np.sqrt(a.max() * a.min()) == pytest.approx(1.0)
    y = awq.awq_linear(d["x"], L["act_scale_inv"], L["q"], L["sc"], L["z"], L["bias"])
    exact = d["x"].astype(np.float64) @ d["W"].T.astype(np.float64) + d["bias"]
    rel = np.linalg.norm(y - exact) / np.linalg.norm(exact)
    assert rel < 0.15   # int4 weight-only error level
