"""tq_quantize_pack / w4g_quantize_pack on the GPU must equal the oracle bit for bit."""
import numpy as np
import pytest
import torch

import bit_weight_only_tq_b200 as tq
import oracle as O
import tq_inputs as I
from gpu_util import bits, gpu, need_cuda

pytestmark = gpu


def _check_tq(w_cpu, rows=None, offset=0):
    need_cuda()
    if offset:
        buf = torch.zeros(w_cpu.numel() + offset, dtype=w_cpu.dtype, device="cuda")
        buf[offset:] = w_cpu.reshape(-1).cuda()
        wg = buf[offset:].view(w_cpu.shape)
    else:
        wg = w_cpu.cuda()
    p, s = tq.tq_quantize_pack(wg)
    torch.cuda.synchronize()
    wn = w_cpu.numpy()
    idx = np.arange(wn.shape[0]) if rows is None else np.asarray(rows)
    pr, sr = O.tq_quantize_pack(wn[idx])
    assert np.array_equal(p.cpu().numpy()[idx], pr), "packed bytes differ"
    assert np.array_equal(bits(s)[idx], sr), "scales differ"


def test_pack_config0_fp32_1024x1024():
    _check_tq(I.weights(1024, 1024, I.seed_for(0, 0, 0)))


def test_pack_fp16_rows():
    _check_tq(I.weights(300, 3584, I.seed_for(4, 0, 1), dtype=torch.float16))


# fp16 rows on each pack kernel: one row per warp (K = 6912: four warps' rows in 55 KB), one row
# per CTA (K = 7040, just past that), rows too long for shared memory (K = 65536, streamed)
@pytest.mark.parametrize("K", [6912, 7040, 65536])
def test_pack_fp16_kernel_boundaries(K):
    _check_tq(I.weights(37, K, 90 + K, dtype=torch.float16, outlier_frac=0.001))


@pytest.mark.parametrize("K", [1, 2, 3, 5, 63, 65, 1001, 4095])
def test_pack_ragged_k(K):
    _check_tq(I.weights(17, K, 77 + K))
    _check_tq(I.weights(9, K, 78 + K, dtype=torch.float16))


def test_pack_unaligned_input():
    _check_tq(I.weights(33, 4096, 5), offset=1)
    _check_tq(I.weights(33, 4096, 6, dtype=torch.float16), offset=3)


# K = 2048: one row per warp; K = 18944: one row per CTA (long rows); both from shared memory
@pytest.mark.parametrize("K", [2048, 18944])
def test_pack_adversarial_rows(K):
    g = torch.Generator().manual_seed(11)
    rows = []
    rows.append(torch.zeros(K))                                           # all zero
    rows.append(torch.full((K,), 0.02))                                   # constant
    e = torch.randint(-140, 100, (K,), generator=g).float()
    rows.append(torch.randn(K, generator=g) * torch.exp2(e))              # huge exponent range
    sub = torch.randint(1, 2 ** 23, (K,), generator=g, dtype=torch.int32).view(torch.float32)
    rows.append(sub)                                                      # fp32 subnormals only
    one = torch.zeros(K)
    one[777] = -3.0
    rows.append(one)                                                      # a single nonzero
    q = torch.randn(K, generator=g) * 0.02
    q[::3] = 1e-30
    rows.append(q)                                                        # many tiny values
    w = torch.stack(rows).float()
    _check_tq(w)
    _check_tq(w.clamp(-60000, 60000).to(torch.float16))


def test_pack_llama_gate_sampled_rows():
    need_cuda()
    w = I.weights(14336, 4096, I.seed_for(1, 0, 4), device="cuda")
    p, s = tq.tq_quantize_pack(w)
    torch.cuda.synchronize()
    rows = np.random.default_rng(0).choice(14336, 48, replace=False)
    rows = np.concatenate([rows, [0, 14335]])
    wn = w[torch.as_tensor(rows, device="cuda")].cpu().numpy()
    pr, sr = O.tq_quantize_pack(wn)
    assert np.array_equal(p.cpu().numpy()[rows], pr)
    assert np.array_equal(bits(s)[rows], sr)


def _check_w4g(w_cpu, offset=0):
    need_cuda()
    if offset:
        buf = torch.zeros(w_cpu.numel() + offset, dtype=w_cpu.dtype, device="cuda")
        buf[offset:] = w_cpu.reshape(-1).cuda()
        wg = buf[offset:].view(w_cpu.shape)
    else:
        wg = w_cpu.cuda()
    qw, s = tq.w4g_quantize_pack(wg)
    torch.cuda.synchronize()
    qr, sr = O.w4g_quantize_pack(w_cpu.numpy())
    assert np.array_equal(qw.cpu().numpy(), qr), "qweight differs"
    assert np.array_equal(bits(s), sr), "scales differ"


def test_w4g_pack_config3_outliers():
    _check_w4g(I.weights(512, 4096, I.seed_for(3, 0, 0), outlier_frac=0.001, outlier_mult=10.0))


def test_w4g_pack_fp16_and_unaligned():
    _check_w4g(I.weights(64, 1024, 9, dtype=torch.float16))
    _check_w4g(I.weights(40, 512, 10), offset=1)


def test_w4g_pack_edge_groups():
    w = torch.zeros(4, 256)
    w[1, 0] = 9.6 * 2.0 ** -24           # subnormal scale, clamping to -8 / +7
    w[1, 1] = -9.6 * 2.0 ** -24
    s0 = 0.0999755859375
    w[2, :6] = torch.tensor([7 * s0, 2.5 * s0, 3.5 * s0, -2.5 * s0, 0.5 * s0, -0.5 * s0])  # ties
    w[3] = torch.randn(256, generator=torch.Generator().manual_seed(3)) * 1e4
    _check_w4g(w)


def _near_threshold_row(K, seed, np_dtype):
    """A row whose elements include the representable values just below, at and just above its
    own threshold 0.7*mean|w| (iterated until the threshold no longer moves), both signs."""
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal(K) * 0.02).astype(np_dtype)
    for _ in range(6):
        t = O.ternary_threshold(w.astype(np.float64))
        c = np.asarray(t, dtype=np_dtype)
        lo = np.nextafter(c, np_dtype(0))
        hi = np.nextafter(c, np_dtype(np.inf))
        near = np.array([lo, c, hi, -lo, -c, -hi], dtype=np_dtype)
        w[: 6 * 16] = np.tile(near, 16)
    return w


def test_pack_threshold_boundary():
    for np_dtype, tdt in ((np.float32, torch.float32), (np.float16, torch.float16)):
        rows = [_near_threshold_row(K, 100 + K, np_dtype) for K in (512, 4096, 4099)]
        for r in rows:
            _check_tq(torch.from_numpy(r[None, :].copy()).to(tdt))


def test_pack_fp32_deep_bins_long_row():
    # K = 2^20 -> narrow exponent bins; a wide exponent spread lands values in many bins.
    g = torch.Generator().manual_seed(12)
    K = 1 << 20
    e = torch.randint(-120, 60, (3, K), generator=g).float()
    w = torch.randn(3, K, generator=g) * torch.exp2(e)
    _check_tq(w)


@pytest.mark.parametrize("K", [2048, 7168, 18944])
def test_pack_fp16_fast_sum_boundaries(K):
    # fp16 rows (16-byte aligned, K % 8 == 0) whose per-lane sums sit at the edges of the fast
    # fp32 accumulation (values up to 2^11, lane sums around 2^11, many subnormals), and rows
    # that must fall back to the fp64 sums; the result must match the oracle bit for bit
    g = torch.Generator().manual_seed(21)
    rows = []
    r = torch.full((K,), 2047.0)                       # every value just below 2^11: lane sums overflow
    rows.append(r)
    r = torch.zeros(K)
    r[::32] = 2047.0                                   # one such value per lane... and 63 more per lane
    rows.append(r)
    r = torch.zeros(K)
    r[::64] = 2040.0                                   # lane sums just below 2^11 (one value each)
    rows.append(r)
    r = torch.randn(K, generator=g) * 6e-8             # fp16 subnormals and zeros
    rows.append(r)
    r = torch.randn(K, generator=g) * 0.02
    r[::7] = 5e-5                                      # mixed normal and subnormal magnitudes
    rows.append(r)
    r = torch.randn(K, generator=g) * 30.0             # lane sums around 2^11
    rows.append(r)
    r = torch.randn(K, generator=g)
    r[5] = 65504.0                                     # the largest fp16 value
    rows.append(r)
    w = torch.stack(rows).to(torch.float16)
    _check_tq(w)


def _near_decision_edges(K, n_rows, seed, rel):
    """Rows of N(0, 0.02) fp16 weights whose threshold 0.7 mean|w| lies within 4 rel (relative)
    of an fp16 value (where the threshold's fp16 bucket changes), or whose scale mean lies within
    4 rel of a midpoint between fp16 values (where its rounding changes): there an approximate
    row sum must not decide.  Found by search; the sums here are plain fp64 sums, exact for fp16
    values with K < 2^13 (multiples of 2^-24 below 2^29)."""
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((n_rows, K)) * 0.02).astype(np.float16)
    d_t, d_s = np.empty(n_rows), np.empty(n_rows)
    for r0 in range(0, n_rows, 512):
        a = np.abs(w[r0:r0 + 512].astype(np.float64))
        t = 0.7 * (a.sum(axis=1) / K)
        tv = np.float16(t).astype(np.float64)               # nearest fp16 value
        d_t[r0:r0 + 512] = np.abs(t - tv) / t
        keep = a > t[:, None]
        nz = keep.sum(axis=1)
        m = (a * keep).sum(axis=1) / np.maximum(nz, 1)
        f = np.float16(m).astype(np.float64)
        nxt = np.where(m >= f, np.nextafter(np.float16(m), np.float16(np.inf)).astype(np.float64),
                       np.nextafter(np.float16(m), np.float16(0)).astype(np.float64))
        d_s[r0:r0 + 512] = np.abs(m - (f + nxt) / 2) / m
    return w, d_t, d_s


# K = 3584: one row per warp (14 terms per fp32 accumulator); K = 18944: one row per CTA of 256
# threads (10 terms)
@pytest.mark.parametrize("K,terms,n_rows,least", [(3584, 14, 8192, 4), (18944, 10, 4096, 2)])
def test_pack_fp16_bounded_sums_at_decision_edges(K, terms, n_rows, least):
    # the fp16 pack takes its row sums from fp32 accumulators when their error bound cannot change
    # the threshold's bucket or the scale's rounding, and sums exactly otherwise: rows right at
    # (and just beyond) those edges must still match the oracle bit for bit
    rel = 1.02 * (terms * 2.0 ** -24)                       # the kernel's bound
    w, d_t, d_s = _near_decision_edges(K, n_rows, 5, rel)
    near_t = np.argsort(d_t)[:32]
    near_s = np.argsort(d_s)[:32]
    assert (d_t[near_t] < rel).sum() >= least, "too few rows inside the threshold band"
    assert (d_s[near_s] < rel).sum() >= least, "too few rows inside the scale band"
    idx = np.unique(np.concatenate([near_t, near_s]))
    _check_tq(torch.from_numpy(w[idx]))
