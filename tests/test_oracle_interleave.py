"""Pins for the oracle's pair-interleaved ternary layout (tq_interleave / tq_deinterleave)."""
import json
import os

import numpy as np
import pytest

import oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))


def test_hand_worked_word():
    g = json.load(open(os.path.join(HERE, "golden", "tq_interleave_hand_worked.json")))
    codes = np.array([g["codes"]], np.int64)
    canon = O.pack_codes(codes)
    assert canon.tolist() == [g["canonical_bytes"]]
    assert O.tq_interleave(canon).tolist() == [g["interleaved_bytes"]]
    assert O.tq_deinterleave(np.array([g["interleaved_bytes"]], np.uint8)).tolist() == [g["canonical_bytes"]]


def test_slot_definition_by_bit_extraction():
    # every slot of every interleaved word, read back with explicit shifts of the 32-bit word,
    # holds the canonical code that the layout assigns to it
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 3, size=(5, 64))
    il = O.tq_interleave(O.pack_codes(codes))
    words = il.view("<u4") if il.flags["C_CONTIGUOUS"] else np.ascontiguousarray(il).view("<u4")
    for n in range(5):
        for q in range(4):
            w = int(words[n, q])
            for j in range(8):
                assert (w >> (2 * j)) & 3 == codes[n, 16 * q + 2 * j]
                assert (w >> (16 + 2 * j)) & 3 == codes[n, 16 * q + 2 * j + 1]


def test_round_trip_and_gemm_invariance():
    rng = np.random.default_rng(5)
    N, K, M = 37, 512, 3
    W = rng.normal(0, 0.02, size=(N, K)).astype(np.float32)
    p, s = O.tq_quantize_pack(W)
    il = O.tq_interleave(p)
    assert np.array_equal(O.tq_deinterleave(il), p)
    assert not np.array_equal(il, p)  # the layout really moves codes
    x = rng.normal(0, 1, size=(M, K)).astype(np.float16)
    y0, b0 = O.tq_gemm(x, p, s, None, K)
    y1, b1 = O.tq_gemm(x, O.tq_deinterleave(il), s, None, K)
    assert np.array_equal(y0, y1) and np.array_equal(b0, b1)


def test_rejects_partial_words():
    with pytest.raises(ValueError):
        O.tq_interleave(np.zeros((2, 6), np.uint8))
    with pytest.raises(ValueError):
        O.tq_deinterleave(np.zeros((2, 6), np.uint8))
