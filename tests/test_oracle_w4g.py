"""Pins for the oracle's W4A16 path ([VQ] notes.devxops.cn vLLM runtime quantisation §4.2, §5).

Checked against hand-worked values, exact ties, exhaustive nibble enumeration and exact
rational dot products.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle as O


def test_hand_worked_group(golden):
    case = golden["w4g_group"]
    W = np.zeros((1, 128), np.float32)
    W[0, :4] = case["w_first4_f32"]
    qw, s = O.w4g_quantize_pack(W)
    assert int(s[0, 0]) == case["scale_bits"]
    assert int(qw.view(np.uint32)[0, 0]) == case["word0_u32"]
    assert np.all(qw.view(np.uint32)[0, 1:] == 0x88888888)
    What = O.w4g_unpack(qw, s)
    q = np.rint(What[0, :4] / O.f16_bits_to_f64(s)[0, 0]).astype(int)
    assert q.tolist() == case["q_first4"]


def test_quotient_ties_go_to_even():
    s0 = 0.0999755859375                     # fp16 0x2E66
    W = np.zeros((1, 128), np.float64)
    W[0, :6] = [7 * s0, 2.5 * s0, 3.5 * s0, -2.5 * s0, 0.5 * s0, -0.5 * s0]
    qw, s = O.w4g_quantize_pack(W.astype(np.float32))
    assert int(s[0, 0]) == 0x2E66            # fp16(7 s0 / 7) = s0
    What = O.w4g_unpack(qw, s)
    assert (What[0, :6] / s0).tolist() == [7, 2, 4, -2, 0, 0]


def test_nibble_order_and_layout():
    # k = 8j + i lives in bits 4i..4i+3 of word j; groups are 128 wide along K.
    s0 = 0.25
    q = np.array([7, -7, 1, 2, 3, -1, -2, 0] * 32, np.float64)   # 256 = 2 groups
    W = (q * s0).astype(np.float32)[None, :]
    qw, s = O.w4g_quantize_pack(W)
    assert qw.shape == (1, 32) and s.shape == (1, 2)
    w0 = int(qw.view(np.uint32)[0, 0])
    u = [(w0 >> (4 * i)) & 0xF for i in range(8)]
    assert u == [15, 1, 9, 10, 11, 7, 6, 8]
    assert np.array_equal(O.w4g_unpack(qw, s), W.astype(np.float64))


def test_all_nibbles_round_trip():
    s_bits = np.array([[0x2E66]], np.uint16)
    for u in range(1, 16):                     # q = u - 8 in [-7, 7]
        word_vals = [u] * 8
        word = sum(v << (4 * i) for i, v in enumerate(word_vals))
        qw = np.full((1, 16), word, np.uint32)
        qw[0, 0] = (word & ~0xF) | 15          # put a q = 7 in the group so max|w| = 7 s
        qw = qw.view(np.int32)
        What = O.w4g_unpack(qw, s_bits)
        qw2, s2 = O.w4g_quantize_pack(What.astype(np.float32))
        assert np.array_equal(qw2, qw) and np.array_equal(s2, s_bits)


def test_zero_group_and_minus_eight_by_clamping():
    W = np.zeros((2, 128), np.float32)
    # row 1: tiny values so that s = fp16(max/7) is the smallest subnormal 2^-24 and the
    # quotient -9.6 clamps to -8 (the only way to reach u = 0)
    W[1, 0] = np.float32(9.6 * 2.0 ** -24)
    W[1, 1] = -np.float32(9.6 * 2.0 ** -24)
    qw, s = O.w4g_quantize_pack(W)
    assert int(s[0, 0]) == 0 and np.all(qw.view(np.uint32)[0] == 0x88888888)
    assert int(s[1, 0]) == 0x0001
    w0 = int(qw.view(np.uint32)[1, 0])
    assert (w0 & 0xF) == 15 and ((w0 >> 4) & 0xF) == 0   # q = +7 (clamped), q = -8 (clamped)


def test_exact_dot_products():
    rng = np.random.default_rng(21)
    N, K, M = 3, 256, 4
    u = rng.integers(0, 16, size=(N, K))
    words = np.zeros((N, K // 8), np.int64)
    for i in range(8):
        words |= u[:, i::8] << (4 * i)
    qw = words.astype(np.uint32).view(np.int32)
    s_bits = O.f64_to_f16_bits(rng.uniform(0.001, 0.05, (N, 2)))
    sv = O.f16_bits_to_f64(s_bits)
    x = rng.integers(-8, 9, size=(M, K)).astype(np.float16)
    y, _ = O.w4g_gemm(x, qw, s_bits, None, K)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(int(x[m, k])) * Fraction(sv[n, k // 128]) * (int(u[n, k]) - 8)
                        for k in range(K))
            assert y[m, n] == float(exact)


def test_rejects_k_not_multiple_of_group():
    with pytest.raises(ValueError):
        O.w4g_quantize_pack(np.zeros((1, 100), np.float32))


def test_gemm_reference_orientation_and_bias():
    # non-square What catches a transposed operand; bias is per output column n
    What = np.array([[1.0, 0.0, 2.0], [0.0, -1.0, 0.5]])
    x = np.array([[1.0, 2.0, 4.0]], np.float16)
    bias = np.array([0.5, -0.25], np.float16)
    y, bound = O.gemm_reference(x, What, bias)
    assert y.tolist() == [[1 + 8 + 0.5, -2 + 2 - 0.25]]
    assert np.allclose(bound, 1e-3 + 2e-3 * np.array([[9.0, 4.0]]), rtol=1e-15)
