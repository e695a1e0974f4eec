"""CPU fp64 oracle for the weight-only low-bit linear layer.

TEST INFRASTRUCTURE.  Only the test suite, the smoke check in ``__graft_entry__`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this module.  The product
path (``bit_weight_only_tq_b200``) never imports it and shares no code with it: this file is a
plain, slow, obviously-correct restatement of what the method computes, written from the sources
below, in float64 numpy (plus exact rational / integer arithmetic where the definition asks for an
exact quantity).

Sources (short tags used in the docstrings):
  [TQ]  "Squeezing ternary-quantised models into vLLM: reverse engineering, reconciliation and
        kernel optimisation" (wzjinhao.cn/news/47283); section numbers are the article's.
  [VQ]  "Model quantisation - the vLLM runtime quantisation architecture" (notes.devxops.cn).
  [QS]  "10.6 Quantisation selection and vLLM in practice" (jennyma11.github.io/infra/ch10-06).

Readings adopted where the sources are silent or garbled (each is repeated at its function):
  * ternarisation comparisons are strict: +1 if w > t, -1 if w < -t, 0 if |w| <= t;
  * the threshold statistic is 0.7 * mean|w| over the row, with the mean taken from the EXACT sum
    of |w| rounded once to fp64 (so it does not depend on summation order);
  * the row scale is the mean |w| over the nonzero codes (exact sum rounded once to fp64, divided
    by the count in fp64), rounded to fp16 with ties-to-even; 0 if the row has no nonzero code;
  * the 2-bit code table is 00 -> -1, 01 -> 0, 10 -> +1; 11 is invalid;
  * INT4: s = fp16(max|w| / 7) per (row, group of 128 along K); q = clamp(rint(w / s), -8, 7)
    using the stored fp16 s, ties-to-even; nibble i of int32 word j holds q + 8 for k = 8j + i;
  * asymmetric INT4: lo = min(0, min w), hi = max(0, max w) over the group, s = fp16((hi-lo)/15),
    z = clamp(rint(-lo/s), 0, 15), q = clamp(rint(w/s) + z, 0, 15); zeros stored one byte per group;
  * activation order: a given column permutation perm defines the groups (g_idx[perm[j]] =
    j // 128); packed weights stay in the original column order.

Every function here is pinned by tests in ``tests/test_oracle_*.py`` against values derived by
hand from the sources, exact rational arithmetic, exhaustive enumeration and library routines.
Nothing here is "parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "f16_table",
    "f64_to_f16_bits",
    "f16_bits_to_f64",
    "exact_abs_sum",
    "ternary_threshold",
    "ternary_codes",
    "pack_codes",
    "unpack_codes",
    "tq_quantize_pack",
    "tq_unpack",
    "tq_gemm",
    "tq_interleave",
    "tq_deinterleave",
    "w4g_quantize_pack",
    "w4g_unpack",
    "w4g_gemm",
    "pack_nibbles",
    "unpack_nibbles",
    "w4z_quantize_group",
    "w4z_quantize_pack",
    "w4z_unpack",
    "w4z_gemm",
    "w4g_quantize_pack_actorder",
    "w4g_gemm_actorder",
    "gemm_reference",
    "quant_check",
    "InvalidCode",
]


class InvalidCode(ValueError):
    """Packed ternary data held the unused code 0b11 ([TQ] §3.1 maps only 00, 01, 10)."""


# ----------------------------------------------------------------------------------------------
# IEEE 754 binary16, built from the format definition
# ----------------------------------------------------------------------------------------------
def f16_table() -> np.ndarray:
    """Values of every non-negative finite binary16 bit pattern 0x0000..0x7BFF, in fp64.

    Format definition (IEEE 754-2008 binary16): 1 sign bit, 5 exponent bits (bias 15),
    10 fraction bits; exponent field 0 encodes subnormals f * 2^-24, fields 1..30 encode
    (1024 + f) * 2^(e - 25).  The table is strictly increasing in the bit pattern.
    """
    bits = np.arange(0x7C00, dtype=np.int64)
    e = bits >> 10
    f = bits & 0x3FF
    sub = f.astype(np.float64) * 2.0 ** -24
    nor = (1024 + f).astype(np.float64) * np.exp2((e - 25).astype(np.float64))
    return np.where(e == 0, sub, nor)


_F16 = f16_table()


def f16_bits_to_f64(bits) -> np.ndarray:
    """Exact fp64 value of binary16 bit patterns (any shape, uint16 or int)."""
    b = np.asarray(bits).astype(np.int64) & 0xFFFF
    mag = b & 0x7FFF
    out = np.empty(b.shape, np.float64)
    fin = mag < 0x7C00
    out[fin] = _F16[mag[fin]]
    inf = mag == 0x7C00
    out[inf] = np.inf
    out[(mag > 0x7C00)] = np.nan
    return np.where(b & 0x8000, -out, out)


def f64_to_f16_bits(d) -> np.ndarray:
    """Round fp64 values to the nearest binary16, ties to the even bit pattern; return uint16.

    Round-to-nearest by definition: locate the two neighbouring binary16 values lo <= |d| < hi
    in the table, take the nearer one, and on a tie the one whose bit pattern is even.  Above
    the largest finite value 65504 the next candidate is 2^16 (even pattern 0x7C00), so
    |d| >= 65520 overflows to infinity as IEEE 754 round-to-nearest requires.
    Both differences |d| - lo and hi - |d| are exact in fp64 (Sterbenz: lo <= |d| <= hi <= 2*lo
    for lo > 0, and |d| - 0 is exact), so the comparison is exact.
    """
    d = np.asarray(d, dtype=np.float64)
    a = np.abs(d)
    ext = np.append(_F16, 65536.0)  # candidate above 65504 is "2^16", i.e. infinity
    idx = np.searchsorted(ext, a, side="right") - 1  # ext[idx] <= a < ext[idx+1]
    idx = np.clip(idx, 0, 0x7C00)
    lo = ext[idx]
    hi = ext[np.minimum(idx + 1, 0x7C00)]
    dlo = a - lo
    dhi = hi - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (idx % 2 == 1))
    res = np.where(pick_hi, idx + 1, idx).astype(np.int64)
    res = np.where(a >= 65536.0, 0x7C00, res)  # beyond the last candidate: infinity
    res = np.where(np.isnan(d), 0x7E00, res)
    sign = np.where(np.signbit(d), 0x8000, 0)
    return (res | sign).astype(np.uint16)


# ----------------------------------------------------------------------------------------------
# Exact sums
# ----------------------------------------------------------------------------------------------
def exact_abs_sum(values) -> float:
    """The exact sum of |v| over finite values, rounded once to fp64 (ties to even).

    ``math.fsum`` returns the correctly rounded sum of its inputs; the inputs here are the fp64
    images of fp32 / fp16 weights, which are exact.  (Pinned against Fraction arithmetic.)
    """
    v = np.abs(np.asarray(values, dtype=np.float64)).ravel()
    return math.fsum(v.tolist())


# ----------------------------------------------------------------------------------------------
# Ternary ([TQ] §1, §3.1, §4)
# ----------------------------------------------------------------------------------------------
def ternary_threshold(w_row) -> float:
    """t = 0.7 * mean|w| for one row ([TQ] §3.1: the statistic is mean(|w|) * 0.7, not std).

    Reading: mean = S / K in fp64 where S is the exact sum of |w| rounded once to fp64; then
    t = 0.7 * mean in fp64 (0.7 = the fp64 literal nearest 0.7).
    """
    w = np.asarray(w_row)
    K = w.shape[-1]
    S = exact_abs_sum(w)
    return 0.7 * (S / K)


def ternary_codes(w_row, t: float) -> np.ndarray:
    """Codes of one row given its threshold ([TQ] §1: sign(w) * [|w| above threshold]).

    Reading of the garbled comparison: code 0b00 (-1) if w < -t, 0b10 (+1) if w > t, and
    0b01 (0) otherwise, i.e. when |w| <= t.  Comparisons are made in fp64 on the exact values.
    """
    w = np.asarray(w_row).astype(np.float64)
    return np.where(w < -t, 0, np.where(w > t, 2, 1)).astype(np.uint8)


def pack_codes(codes) -> np.ndarray:
    """Pack a row of 2-bit codes, 4 per byte: element 4j+i goes to bits 2i..2i+1 of byte j
    ([TQ] §3.1 dequant_ternary reads (byte >> 2k) & 3 for element 4j+k).  A partial last byte is
    padded with code 0b01 (value 0), so the row is ceil(K/4) bytes ([TQ] §3.2-3.3)."""
    c = np.asarray(codes, dtype=np.int64)
    K = c.shape[-1]
    KB = (K + 3) // 4
    padded = np.ones(c.shape[:-1] + (KB * 4,), np.int64)
    padded[..., :K] = c
    q = padded.reshape(c.shape[:-1] + (KB, 4))
    byte = q[..., 0] | (q[..., 1] << 2) | (q[..., 2] << 4) | (q[..., 3] << 6)
    return byte.astype(np.uint8)


def unpack_codes(packed, K: int) -> np.ndarray:
    """Inverse of pack_codes for the first K codes of each row: code = (byte >> 2i) & 3."""
    p = np.asarray(packed, dtype=np.int64)
    shifts = np.array([0, 2, 4, 6], np.int64)
    codes = (p[..., :, None] >> shifts) & 3
    codes = codes.reshape(p.shape[:-1] + (p.shape[-1] * 4,))
    return codes[..., :K].astype(np.uint8)


# The pair-interleaved layout: a post-load relayout of the packed codes (the repack step that
# [VQ] §4.3 describes for GPTQ/AWQ checkpoints, applied here to the ternary format).  It is a
# layout of this library, not of the pages: the same bytes per row, the codes of every group of
# 16 moved so that the two fp16 halves of a 32-bit word read at one bit position hold the codes
# of two consecutive k.
IL_SOURCE = np.array([0, 2, 4, 6, 8, 10, 12, 14, 1, 3, 5, 7, 9, 11, 13, 15], np.int64)


def tq_interleave(packed) -> np.ndarray:
    """Canonical packed rows [N, KB] (KB % 4 == 0: whole 32-bit words of 16 codes) to the
    pair-interleaved layout.  Code slot s of a little-endian word (bits 2s..2s+1) holds, in the
    canonical layout, code k = 16q + s; in the interleaved layout slot j (j < 8) holds
    k = 16q + 2j and slot 8 + j holds k = 16q + 2j + 1."""
    p = np.asarray(packed, np.uint8)
    N, KB = p.shape
    if KB % 4:
        raise ValueError("the interleaved layout needs whole 32-bit words (K a multiple of 16)")
    codes = unpack_codes(p, KB * 4).reshape(N, KB // 4, 16)
    return pack_codes(codes[:, :, IL_SOURCE].reshape(N, KB * 4))


def tq_deinterleave(packed_il) -> np.ndarray:
    """Inverse of tq_interleave."""
    p = np.asarray(packed_il, np.uint8)
    N, KB = p.shape
    if KB % 4:
        raise ValueError("the interleaved layout needs whole 32-bit words (K a multiple of 16)")
    il = unpack_codes(p, KB * 4).reshape(N, KB // 4, 16)
    codes = np.empty_like(il)
    codes[:, :, IL_SOURCE] = il
    return pack_codes(codes.reshape(N, KB * 4))


def tq_quantize_pack(W):
    """Ternarise and pack a weight matrix W[N,K] (fp32 or fp16).

    Returns (packed uint8 [N, ceil(K/4)], scale uint16 fp16-bits [N]).
    Per row ([TQ] §1 ternarisation, §3.1 threshold and storage, §2.1 uint8 weight + fp16 scale):
      S = exact sum |w| (rounded once to fp64);  t = 0.7 * (S / K)
      codes by ternary_codes;  nz = #codes != 1;  A = exact sum of |w| where code != 1
      scale = fp16(A / nz) (fp64 division, then round to binary16, ties-to-even); 0 if nz == 0
    Reading: the pages give the scale's dtype and shape but no formula; the mean |w| over the
    nonzero codes (the Ternary Weight Networks rule) is taken.
    """
    W = np.asarray(W)
    if W.dtype not in (np.float32, np.float16):
        raise TypeError("W must be float32 or float16")
    N, K = W.shape
    if K <= 0:
        raise ValueError("K must be positive")
    KB = (K + 3) // 4
    packed = np.zeros((N, KB), np.uint8)
    scale = np.zeros(N, np.uint16)
    for n in range(N):
        w = W[n].astype(np.float64)
        t = ternary_threshold(w)
        codes = ternary_codes(w, t)
        nzm = codes != 1
        nz = int(nzm.sum())
        if nz > 0:
            A = exact_abs_sum(w[nzm])
            scale[n] = f64_to_f16_bits(A / nz)
        packed[n] = pack_codes(codes)
    return packed, scale


def tq_unpack(packed, scale_bits, K: int) -> np.ndarray:
    """What[n,k] = scale[n] * (code - 1) in fp64 ([TQ] §3.1 dequant_ternary; §4 (c - 1)).

    The stored fp16 scale is used ([TQ] §3.1 compares against scale.half().float()).
    Raises InvalidCode if any of the first K codes of a row is 0b11.
    """
    codes = unpack_codes(packed, K).astype(np.int64)
    if np.any(codes == 3):
        raise InvalidCode("packed data holds code 0b11")
    s = f16_bits_to_f64(scale_bits)
    return s[:, None] * (codes - 1).astype(np.float64)


def gemm_reference(x_f16, What, bias_f16=None):
    """y_ref = x . What^T (+ bias) in fp64, and the per-element acceptance bound
    1e-3 + 2e-3 * sum_k |x[m,k] * What[n,k]|.

    x_f16: numpy float16 [M,K] (or uint16 bit patterns); What: fp64 [N,K]; bias: fp16 [N] or None.
    """
    x = _as_f64_from_f16(x_f16)
    y = x @ What.T
    if bias_f16 is not None:
        y = y + _as_f64_from_f16(bias_f16)[None, :]
    bound = 1e-3 + 2e-3 * (np.abs(x) @ np.abs(What).T)
    return y, bound


def tq_gemm(x_f16, packed, scale_bits, bias_f16, K: int):
    """Ternary linear layer reference: dequantise, then matmul ([TQ] §2.3 apply_weights, §4)."""
    return gemm_reference(x_f16, tq_unpack(packed, scale_bits, K), bias_f16)


# ----------------------------------------------------------------------------------------------
# W4A16, group size 128 ([VQ] §4.2, §5)
# ----------------------------------------------------------------------------------------------
GROUP = 128


def w4g_quantize_pack(W):
    """Symmetric INT4 with one fp16 scale per (row, group of 128 along K), no act-order.

    [VQ] §5 gives the checkpoint config {"bits": 4, "group_size": 128, "desc_act": false,
    "sym": true} and §4.2 / §5 the layout: 8 INT4 values per int32, weight [d_out, d_in/8],
    weight_scale [d_out, d_in/128].  The calibration-based GPTQ solve is not reproduced; the
    round-to-nearest reading is used:
      s = fp16(max|w| / 7)  (fp64 division, then binary16 ties-to-even)
      q = 0 if s == 0 else clamp(rint(w / s), -8, 7), fp64 quotient by the stored fp16 s,
          rint = round half to even
      nibble i (bits 4i..4i+3) of word j holds u = q + 8 for k = 8j + i.
    Returns (qweight int32 [N, K/8], scales uint16 fp16-bits [N, K/128]).
    """
    W = np.asarray(W)
    if W.dtype not in (np.float32, np.float16):
        raise TypeError("W must be float32 or float16")
    N, K = W.shape
    if K % GROUP != 0 or K <= 0:
        raise ValueError("K must be a positive multiple of 128")
    G = K // GROUP
    w = W.astype(np.float64).reshape(N, G, GROUP)
    mx = np.abs(w).max(axis=2)
    s_bits = f64_to_f16_bits(mx / 7.0)
    s = f16_bits_to_f64(s_bits)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.rint(w / s[:, :, None])
    q = np.where(s[:, :, None] == 0.0, 0.0, q)
    q = np.clip(q, -8, 7).astype(np.int64)
    u = (q + 8).reshape(N, K // 8, 8)
    word = np.zeros((N, K // 8), np.int64)
    for i in range(8):
        word |= u[:, :, i] << (4 * i)
    return word.astype(np.uint32).view(np.int32), s_bits.astype(np.uint16)


def w4g_unpack(qweight, scales_bits) -> np.ndarray:
    """What[n,k] = s[n, k/128] * (u - 8) in fp64, u = nibble k%8 of word k/8."""
    qw = np.asarray(qweight).view(np.uint32).astype(np.int64)
    N, KW = qw.shape
    K = KW * 8
    u = np.stack([(qw >> (4 * i)) & 0xF for i in range(8)], axis=2).reshape(N, K)
    s = f16_bits_to_f64(scales_bits)
    return np.repeat(s, GROUP, axis=1) * (u - 8).astype(np.float64)


def w4g_gemm(x_f16, qweight, scales_bits, bias_f16, K: int):
    """W4A16 linear layer reference: dequantise, then matmul ([VQ] §5 forward)."""
    What = w4g_unpack(qweight, scales_bits)
    assert What.shape[1] == K
    return gemm_reference(x_f16, What, bias_f16)


# ----------------------------------------------------------------------------------------------
# INT4 variants ([VQ] §5): asymmetric zero-points and activation ordering (g_idx)
# ----------------------------------------------------------------------------------------------
def w4z_quantize_group(w_group, order_of_zero=True):
    """Asymmetric INT4 of one group (the weight_zp / GroupQuantZeroPointParameter of [VQ] §5's
    GPTQ-Marlin create_weights; the qweight / scales / zeros triple of an AWQ checkpoint, [TQ] §2.1).

    The pages name the zero-point but give no formula; the min-max rule that keeps 0 inside the
    range is read here:
      lo = min(0, min w), hi = max(0, max w)            (fp64, exact)
      s  = fp16(( hi - lo ) / 15)                        (fp64 division, binary16 ties-to-even)
      s == 0 (an all-zero group): z = 0, every q = 0
      else z = clamp(rint(-lo / s), 0, 15) and q = clamp(rint(w / s) + z, 0, 15), both with the
           STORED fp16 s, fp64 quotients, rint = round half to even
    Returns (q int64 array, s bits uint16, z int).
    """
    w = np.asarray(w_group, dtype=np.float64)
    lo = min(0.0, float(w.min()))
    hi = max(0.0, float(w.max()))
    s_bits = f64_to_f16_bits((hi - lo) / 15.0)
    s = float(f16_bits_to_f64(s_bits))
    if s == 0.0:
        return np.zeros(w.shape, np.int64), np.uint16(s_bits), 0
    z = int(np.clip(np.rint(-lo / s), 0, 15))
    q = np.clip(np.rint(w / s) + z, 0, 15).astype(np.int64)
    return q, np.uint16(s_bits), z


def pack_nibbles(u):
    """u int64 [N, K] in 0..15 -> int32 [N, K/8], nibble i of word j = element 8j + i."""
    N, K = u.shape
    u = u.reshape(N, K // 8, 8)
    word = np.zeros((N, K // 8), np.int64)
    for i in range(8):
        word |= u[:, :, i] << (4 * i)
    return word.astype(np.uint32).view(np.int32)


def unpack_nibbles(qweight):
    qw = np.asarray(qweight).view(np.uint32).astype(np.int64)
    N, KW = qw.shape
    return np.stack([(qw >> (4 * i)) & 0xF for i in range(8)], axis=2).reshape(N, KW * 8)


def w4z_quantize_pack(W, perm=None):
    """Asymmetric INT4, group 128 along K, optionally in activation order.

    perm (optional int array [K], a permutation of 0..K-1): the order in which GPTQ with
    desc_act processes the input columns ([VQ] §5: "optional g_idx (activation ordering)"); here it
    is an input (the pages' Hessian order needs calibration data).  Column perm[j] belongs to
    group j // 128, i.e. g_idx[perm[j]] = j // 128.  Without perm, g_idx[k] = k // 128.
    The packed weights stay in the ORIGINAL column order (nibble i of word j = column 8j + i, the
    checkpoint layout); scales and zeros are [N, K/128] by group.
    Returns (qweight int32 [N, K/8], scales uint16 fp16-bits [N, K/128], zeros uint8 [N, K/128],
    g_idx int32 [K]).
    """
    W = np.asarray(W)
    if W.dtype not in (np.float32, np.float16):
        raise TypeError("W must be float32 or float16")
    N, K = W.shape
    if K % GROUP != 0 or K <= 0:
        raise ValueError("K must be a positive multiple of 128")
    perm = np.arange(K) if perm is None else np.asarray(perm, dtype=np.int64)
    if sorted(perm.tolist()) != list(range(K)):
        raise ValueError("perm must be a permutation of 0..K-1")
    G = K // GROUP
    g_idx = np.empty(K, np.int32)
    g_idx[perm] = np.arange(K) // GROUP
    q = np.zeros((N, K), np.int64)
    scales = np.zeros((N, G), np.uint16)
    zeros = np.zeros((N, G), np.uint8)
    Wd = W.astype(np.float64)
    for n in range(N):
        for g in range(G):
            cols = perm[g * GROUP:(g + 1) * GROUP]
            qg, sb, z = w4z_quantize_group(Wd[n, cols])
            q[n, cols] = qg
            scales[n, g] = sb
            zeros[n, g] = z
    return pack_nibbles(q), scales, zeros, g_idx


def w4z_unpack(qweight, scales_bits, zeros, g_idx=None) -> np.ndarray:
    """What[n,k] = s[n, g_idx[k]] * (q[n,k] - z[n, g_idx[k]]) in fp64 (g_idx default k // 128)."""
    q = unpack_nibbles(qweight)
    N, K = q.shape
    g = (np.arange(K) // GROUP) if g_idx is None else np.asarray(g_idx, dtype=np.int64)
    s = f16_bits_to_f64(scales_bits)
    z = np.asarray(zeros, dtype=np.int64)
    return s[:, g] * (q - z[:, g]).astype(np.float64)


def w4z_gemm(x_f16, qweight, scales_bits, zeros, bias_f16, K: int, g_idx=None):
    """Asymmetric / act-order W4A16 linear layer reference: dequantise, then matmul."""
    What = w4z_unpack(qweight, scales_bits, zeros, g_idx)
    assert What.shape[1] == K
    return gemm_reference(x_f16, What, bias_f16)


def w4g_quantize_pack_actorder(W, perm):
    """Symmetric INT4 ([VQ] §5 sym=true) with activation ordering: the rule of w4g_quantize_pack
    applied to the columns of each group perm[128 g .. 128 g + 127].  Returns (qweight [N, K/8]
    in the original column order, scales [N, K/128], g_idx [K])."""
    W = np.asarray(W)
    N, K = W.shape
    perm = np.asarray(perm, dtype=np.int64)
    if sorted(perm.tolist()) != list(range(K)) or K % GROUP != 0:
        raise ValueError("perm must be a permutation of 0..K-1, K % 128 == 0")
    qw_p, s = w4g_quantize_pack(W[:, perm])            # contiguous groups in processing order
    u_p = unpack_nibbles(qw_p)
    u = np.empty_like(u_p)
    u[:, perm] = u_p                                   # back to the original column order
    g_idx = np.empty(K, np.int32)
    g_idx[perm] = np.arange(K) // GROUP
    return pack_nibbles(u), s, g_idx


def w4g_gemm_actorder(x_f16, qweight, scales_bits, g_idx, bias_f16, K: int):
    """What[n,k] = s[n, g_idx[k]] * (u[n,k] - 8); then y = x . What^T (+ bias)."""
    u = unpack_nibbles(qweight)
    s = f16_bits_to_f64(scales_bits)
    g = np.asarray(g_idx, dtype=np.int64)
    What = s[:, g] * (u - 8).astype(np.float64)
    return gemm_reference(x_f16, What, bias_f16)


# ----------------------------------------------------------------------------------------------
# Numerics report ([QS] 10.6.3 quant_check: ok, max_abs, mean_abs, finite)
# ----------------------------------------------------------------------------------------------
def quant_check(y_ref, y_test, bound=None, atol=None, rtol=None):
    """The fields of the pages' quant_check, plus the per-element bound used by this library.

    ok is all(|y_test - y_ref| <= bound) when a bound array is given, else allclose(atol, rtol).
    """
    yr = np.asarray(y_ref, dtype=np.float64)
    yt = _as_f64_from_f16(y_test) if np.asarray(y_test).dtype in (np.float16, np.uint16) \
        else np.asarray(y_test, dtype=np.float64)
    diff = np.abs(yr - yt)
    finite = bool(np.isfinite(yt).all())
    if bound is not None:
        ok = bool(np.all(diff <= bound)) and finite
        worst = float(np.max(diff / bound)) if diff.size else 0.0
    else:
        ok = bool(np.allclose(yr, yt, atol=atol, rtol=rtol)) and finite
        worst = None
    return {
        "ok": ok,
        "max_abs": float(diff.max()) if diff.size else 0.0,
        "mean_abs": float(diff.mean()) if diff.size else 0.0,
        "finite": finite,
        "worst_bound_ratio": worst,
    }


def _as_f64_from_f16(a) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype == np.float16:
        return a.astype(np.float64)
    if a.dtype == np.uint16:
        return f16_bits_to_f64(a)
    raise TypeError("expected float16 values or uint16 fp16 bit patterns")

