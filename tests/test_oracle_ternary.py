"""Pins for the oracle's ternary path ([TQ] wzjinhao.cn/news/47283 §1, §3.1-3.3, §4).

Each test checks the oracle against something other than itself: hand-worked values derived
from the article's rules, exhaustive enumeration, integer arithmetic, closed forms and
statistics of the normal distribution.
"""
import itertools
import math

import numpy as np
import pytest

import oracle as O


def _row(case):
    return np.array([case["w_f32"]], np.float32)


@pytest.mark.parametrize("name", ["ternary_row", "ternary_zero_row", "ternary_alternating_row",
                                  "ternary_ragged_row"])
def test_hand_worked_rows(golden, name):
    case = golden[name]
    p, s = O.tq_quantize_pack(_row(case))
    assert p[0].tolist() == case["packed"]
    assert int(s[0]) == case["scale_bits"]


def test_hand_worked_gemm(golden):
    case = golden["ternary_row"]
    p = np.array([case["packed"]], np.uint8)
    s = np.array([case["scale_bits"]], np.uint16)
    x = np.array([case["x_f16"]], np.float16)
    y, bound = O.tq_gemm(x, p, s, None, 4)
    assert y[0, 0] == case["y"]
    # bound = 1e-3 + 2e-3 * sum |x * What| = 1e-3 + 2e-3 * 0.7001953125 * (1 + 3)
    assert bound[0, 0] == pytest.approx(1e-3 + 2e-3 * 0.7001953125 * 4, rel=1e-15)


def test_code_bit_order():
    # element 4j+k sits at bits 2k..2k+1 of byte j: codes [0,1,2,1] -> 0b01_10_01_00
    assert O.pack_codes(np.array([0, 1, 2, 1])).tolist() == [0x64]
    assert O.unpack_codes(np.array([[0x64]], np.uint8), 4).tolist() == [[0, 1, 2, 1]]


def test_threshold_comparisons_are_strict():
    t = 0.25
    w = np.array([0.25, -0.25, np.nextafter(0.25, 1), -np.nextafter(0.25, 1), 0.0])
    assert O.ternary_codes(w, t).tolist() == [1, 1, 2, 0, 1]


def test_threshold_uses_mean_not_std():
    # [TQ] §3.1: mean(|w|)*0.7 is the statistic; std would give a different code here.
    w = np.array([1.0, 1.0, 1.0, 0.5, 0.0, 0.0, 0.0, 0.0], np.float32)
    t = O.ternary_threshold(w)
    assert t == 0.7 * (3.5 / 8)                 # 0.30625
    assert O.ternary_codes(w, t)[3] == 2        # 0.5 > 0.30625
    t_std = 0.7 * float(np.std(np.abs(w)))       # ~0.334: the wrong statistic
    assert t_std != t


def test_scale_is_mean_abs_of_nonzero_codes():
    w = np.array([[0.3, -0.5, 0.01, 0.02, 0.0, 0.7, -0.02, 0.0]], np.float32)
    p, s = O.tq_quantize_pack(w)
    # S = 1.55, t = 0.7 * 1.55 / 8 = 0.135625 -> nonzero: 0.3, -0.5, 0.7 -> mean 0.5
    assert O.f16_bits_to_f64(s)[0] == 0.5
    assert O.unpack_codes(p, 8)[0].tolist() == [2, 0, 1, 1, 1, 2, 1, 1]


def test_ragged_padding_is_zero_code():
    rng = np.random.default_rng(3)
    for K in (1, 2, 3, 5, 6, 7, 9, 4095):
        w = rng.standard_normal((3, K)).astype(np.float32)
        p, _ = O.tq_quantize_pack(w)
        assert p.shape == (3, (K + 3) // 4)
        full = O.unpack_codes(p, p.shape[1] * 4)
        assert np.all(full[:, K:] == 1)


def test_round_trip_all_81_bytes():
    # pack(unpack(P)) == P for every byte whose 4 codes are valid, with a nonzero fp16 scale.
    s = np.array([0x2E66], np.uint16)  # 0.0999755859375
    n = 0
    for codes in itertools.product([0, 1, 2], repeat=4):
        P = O.pack_codes(np.array(codes))[None, :]
        What = O.tq_unpack(P, s, 4)
        p2, s2 = O.tq_quantize_pack(What.astype(np.float32))
        assert p2.tolist() == P.tolist()
        assert int(s2[0]) == (0 if codes == (1, 1, 1, 1) else 0x2E66)
        n += 1
    assert n == 81


def test_unpack_rejects_code_11():
    with pytest.raises(O.InvalidCode):
        O.tq_unpack(np.array([[0b11]], np.uint8), np.array([0x3C00], np.uint16), 4)
    # a 0b11 in the padding beyond K is ignored
    O.tq_unpack(np.array([[0b11_000000]], np.uint8), np.array([0x3C00], np.uint16), 3)


@pytest.mark.parametrize("N,K", [(1, 8), (2, 4), (4, 2), (8, 1)])
def test_brute_force_all_code_matrices(N, K):
    # every one of the 3^(N*K) code matrices: y must equal the integer dot product times scale
    rng = np.random.default_rng(N * 10 + K)
    x = rng.integers(-7, 8, size=(3, K)).astype(np.float16)
    xi = x.astype(np.int64)
    scale_bits = O.f64_to_f16_bits(rng.uniform(0.01, 2.0, N))
    sc = O.f16_bits_to_f64(scale_bits)
    for codes in itertools.product([0, 1, 2], repeat=N * K):
        c = np.array(codes, np.int64).reshape(N, K)
        P = O.pack_codes(c)
        y, _ = O.tq_gemm(x, P, scale_bits, None, K)
        dot = xi @ (c - 1).T                       # independent integer dot product
        assert np.array_equal(y, dot * sc[None, :])


def test_all_plus_one_codes_give_row_sums():
    rng = np.random.default_rng(11)
    K, N = 96, 5
    x = rng.standard_normal((4, K)).astype(np.float16)
    P = O.pack_codes(np.full((N, K), 2))
    y, _ = O.tq_gemm(x, P, np.full(N, 0x3C00, np.uint16), None, K)
    rs = np.array([math.fsum(r) for r in x.astype(np.float64)])
    assert np.allclose(y, rs[:, None], rtol=0, atol=1e-12)


def test_identity_pattern_gives_scaled_x():
    K = 12
    c = np.ones((K, K), np.int64) + np.eye(K, dtype=np.int64)   # diagonal +1, rest 0
    P = O.pack_codes(c)
    s_bits = np.full(K, 0x3800, np.uint16)                       # 0.5
    x = np.arange(2 * K, dtype=np.float16).reshape(2, K)
    bias = np.full(K, 0x3C00, np.uint16).view(np.float16)        # 1.0
    y, _ = O.tq_gemm(x, P, s_bits, bias, K)
    assert np.array_equal(y, 0.5 * x.astype(np.float64) + 1.0)


def test_normal_weights_statistics():
    # For N(0, s): t = 0.7 * s * sqrt(2/pi) = 0.5585 s, P(|w| <= t) = erf(0.5585/sqrt 2) = 0.4235,
    # and the scale = E[|w| | |w| > t] = s * phi(a) / Q(a) with a = t / s.
    from scipy.stats import norm
    rng = np.random.default_rng(5)
    sigma = 0.02
    W = (rng.standard_normal((64, 8192)) * sigma).astype(np.float32)
    p, s = O.tq_quantize_pack(W)
    codes = O.unpack_codes(p, 8192)
    a = 0.7 * math.sqrt(2 / math.pi)
    p0 = math.erf(a / math.sqrt(2))
    assert abs((codes == 1).mean() - p0) < 0.005
    assert abs((codes == 0).mean() - (1 - p0) / 2) < 0.005
    expect_scale = sigma * norm.pdf(a) / norm.sf(a)
    assert abs(O.f16_bits_to_f64(s).mean() / expect_scale - 1) < 0.01


def test_fp16_input_matches_fp32_of_same_values():
    rng = np.random.default_rng(9)
    W16 = (rng.standard_normal((8, 200)) * 0.02).astype(np.float16)
    pa, sa = O.tq_quantize_pack(W16)
    pb, sb = O.tq_quantize_pack(W16.astype(np.float32))
    assert np.array_equal(pa, pb) and np.array_equal(sa, sb)


def test_quant_check_fields():
    ref = np.array([[1.0, 2.0]])
    test = np.array([[1.0, 2.5]], np.float16)
    r = O.quant_check(ref, test, bound=np.array([[0.1, 0.1]]))
    assert r["ok"] is False and r["max_abs"] == 0.5 and r["mean_abs"] == 0.25 and r["finite"]
    r = O.quant_check(ref, test, atol=0.6, rtol=0)
    assert r["ok"] is True
