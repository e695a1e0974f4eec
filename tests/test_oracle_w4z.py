"""Pins for the oracle's INT4 variants: asymmetric zero-points and activation order
([VQ] notes.devxops.cn vLLM runtime quantisation §5: weight_zp per group of 128, optional g_idx;
[TQ] §2.1: AWQ's qweight / scales / zeros).

Checked against hand-worked groups (tests/golden/w4z_hand_worked.json), the round-to-nearest
error bound, exact zero representation, exact rational dot products, and the permutation
invariant x . What^T = (x P) . (What P)^T that ties the activation-order form to the contiguous
one."""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden", "w4z_hand_worked.json")


def test_hand_worked_groups():
    with open(GOLD) as f:
        d = json.load(f)
    for c in d["cases"]:
        W = np.zeros((1, 256), np.float32)
        W[0, 132:256] = c.get("fill", 0.0)
        W[0, 128:132] = c["w_first4_f32"]           # second group; the first is all zero
        qw, s, z, g_idx = O.w4z_quantize_pack(W)
        assert int(s[0, 1]) == c["scale_bits"], c["name"]
        assert int(z[0, 1]) == c["zero"], c["name"]
        q = O.unpack_nibbles(qw)[0]
        assert q[128:132].tolist() == c["q_first4"], c["name"]
        assert (q[132:] == c["q_rest"]).all(), c["name"]
        assert int(s[0, 0]) == 0 and int(z[0, 0]) == 0 and (q[:128] == 0).all()
        assert g_idx.tolist() == [k // 128 for k in range(256)]


def test_nibble_pack_round_trip_and_order():
    rng = np.random.default_rng(1)
    u = rng.integers(0, 16, (5, 64))
    assert (O.unpack_nibbles(O.pack_nibbles(u)) == u).all()
    word = O.pack_nibbles(np.arange(8)[None, :])   # element 8j + i at bits 4i..4i+3
    assert int(word.view(np.uint32)[0, 0]) == 0x76543210


def test_rounding_error_bound_and_exact_zero():
    rng = np.random.default_rng(2)
    W = (rng.standard_normal((16, 512)) * 0.02).astype(np.float32)
    W[3, :128] = np.abs(W[3, :128])                    # one-sided groups
    W[4, 128:256] = -np.abs(W[4, 128:256])
    W[5, 256:384] *= 100.0
    qw, s, z, _ = O.w4z_quantize_pack(W)
    What = O.w4z_unpack(qw, s, z)
    sf = O.f16_bits_to_f64(s)
    step = np.repeat(sf, 128, axis=1)
    # round to nearest on the grid s * (q - z): within half a step, plus the widening of the grid
    # by the fp16 rounding of s (the extreme element may sit one rounding away from the grid end)
    lo = np.minimum(0, W.reshape(16, 4, 128).min(axis=2)).astype(np.float64)
    hi = np.maximum(0, W.reshape(16, 4, 128).max(axis=2)).astype(np.float64)
    slack = np.repeat(np.abs((hi - lo) - 15 * sf) + 0.5 * sf, 128, axis=1)
    assert (np.abs(What - W.astype(np.float64)) <= slack * (1 + 1e-12)).all()
    # 0 lies inside [lo, hi] and z is an integer: a zero weight dequantises to exactly 0
    W0 = W.copy()
    W0[:, ::7] = 0.0
    qw0, s0, z0, _ = O.w4z_quantize_pack(W0)
    assert (O.w4z_unpack(qw0, s0, z0)[:, ::7] == 0.0).all()


def test_zero_point_range():
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((8, 1024)) * 0.05 + rng.standard_normal((8, 1)) * 0.05).astype(np.float32)
    _, s, z, _ = O.w4z_quantize_pack(W)
    assert z.min() >= 0 and z.max() <= 15
    q = O.unpack_nibbles(O.w4z_quantize_pack(W)[0])
    assert q.min() >= 0 and q.max() <= 15


def test_gemm_exact_dot_products():
    rng = np.random.default_rng(4)
    W = (rng.standard_normal((3, 256)) * 0.3).astype(np.float32)
    qw, s, z, _ = O.w4z_quantize_pack(W)
    x = rng.integers(-3, 4, (2, 256)).astype(np.float16)
    b = np.array([0.5, -0.25, 1.0], np.float16)
    y, bound = O.w4z_gemm(x, qw, s, z, b, 256)
    q = O.unpack_nibbles(qw)
    for m in range(2):
        for n in range(3):
            acc = Fraction(0)
            for k in range(256):
                g = k // 128
                acc += Fraction(float(x[m, k])) * Fraction(float(O.f16_bits_to_f64(s[n, g]))) * (int(q[n, k]) - int(z[n, g]))
            acc += Fraction(float(b[n]))
            assert abs(float(acc) - y[m, n]) <= 1e-12 * max(1.0, abs(float(acc)))
    assert (bound >= 1e-3).all()


@pytest.mark.parametrize("seed", [5, 6])
def test_act_order_groups_follow_the_permutation(seed):
    rng = np.random.default_rng(seed)
    K = 512
    W = (rng.standard_normal((4, K)) * 0.02).astype(np.float32)
    perm = rng.permutation(K)
    qw, s, z, g_idx = O.w4z_quantize_pack(W, perm)
    # every group holds 128 columns, exactly perm[128 g .. 128 g + 127]
    assert np.bincount(g_idx, minlength=K // 128).tolist() == [128] * (K // 128)
    for gi in range(K // 128):
        assert sorted(np.nonzero(g_idx == gi)[0].tolist()) == sorted(perm[128 * gi:128 * (gi + 1)].tolist())
    # the perm-indexed quantiser equals the contiguous one applied to the permuted matrix
    qp, sp, zp, _ = O.w4z_quantize_pack(W[:, perm])
    assert (s == sp).all() and (z == zp).all()
    assert (O.unpack_nibbles(qw)[:, perm] == O.unpack_nibbles(qp)).all()
    # symmetric activation order: each group's scale is the w4g rule on its own members
    qs, ss, gs = O.w4g_quantize_pack_actorder(W, perm)
    assert (gs == g_idx).all()
    for gi in range(K // 128):
        cols = perm[128 * gi:128 * (gi + 1)]
        mx = np.abs(W[:, cols].astype(np.float64)).max(axis=1)
        assert (ss[:, gi] == O.f64_to_f16_bits(mx / 7.0)).all()


def test_act_order_gemm_is_the_permuted_contiguous_gemm():
    # x . What^T summed over k in any order: permuting the contraction index by P changes nothing
    rng = np.random.default_rng(7)
    K = 384
    W = (rng.standard_normal((5, K)) * 0.02).astype(np.float32)
    perm = rng.permutation(K)
    x = rng.standard_normal((3, K)).astype(np.float16)
    qw, s, g_idx = O.w4g_quantize_pack_actorder(W, perm)
    y1, _ = O.w4g_gemm_actorder(x, qw, s, g_idx, None, K)
    qc, sc = O.w4g_quantize_pack(W[:, perm])
    y2, _ = O.w4g_gemm(x[:, perm], qc, sc, None, K)
    assert np.allclose(y1, y2, rtol=1e-12, atol=1e-12)
    qz, sz, zz, gz = O.w4z_quantize_pack(W, perm)
    y3, _ = O.w4z_gemm(x, qz, sz, zz, None, K, g_idx=gz)
    qz2, sz2, zz2, _ = O.w4z_quantize_pack(W[:, perm])
    y4, _ = O.w4z_gemm(x[:, perm], qz2, sz2, zz2, None, K)
    assert np.allclose(y3, y4, rtol=1e-12, atol=1e-12)
