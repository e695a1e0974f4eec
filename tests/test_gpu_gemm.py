"""tq_gemm / w4g_gemm on the GPU against the oracle, per path, over ragged shapes.

Pass rule (element by element): |y - y_ref| <= 1e-3 + 2e-3 * sum_k |x[m,k] * What[n,k]|.
"""
import numpy as np
import pytest
import torch

import bit_weight_only_tq_b200 as tq
import tq_inputs as I
from gpu_util import check_canaries, check_tq_gemm, check_w4g_gemm, gpu, guarded_empty, need_cuda

pytestmark = gpu


def _tq_problem(M, N, K, seed, bias=True, outlier_rows=0.0):
    w = I.weights(N, K, seed, device="cuda")
    packed, scale = tq.tq_quantize_pack(w)
    x = I.activations(M, K, seed, device="cuda", outlier_row_frac=outlier_rows)
    b = I.bias(N, seed, device="cuda") if bias else None
    return x, packed, scale, b


def _w4_problem(M, N, K, seed, bias=True):
    w = I.weights(N, K, seed, device="cuda", outlier_frac=0.001)
    qw, sc = tq.w4g_quantize_pack(w)
    x = I.activations(M, K, seed, device="cuda")
    b = I.bias(N, seed, device="cuda") if bias else None
    return x, qw, sc, b


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 7, 8, 9, 12, 13, 16])
@pytest.mark.parametrize("path", [tq.PATH_DECODE, tq.PATH_GENERIC])
def test_tq_small_m(M, path):
    need_cuda()
    x, p, s, b = _tq_problem(M, 1000, 1088, 100 + M)
    y = tq.tq_gemm(x, p, s, b, path=path)
    check_tq_gemm(x, p, s, b, y, label=f"M={M} path={path}")


@pytest.mark.parametrize("N,K", [(128, 64), (200, 14336), (256, 18944), (1024, 4096), (37, 512),
                                 (4096, 1024)])
@pytest.mark.parametrize("M", [1, 16])
def test_tq_decode_shapes(N, K, M):
    need_cuda()
    x, p, s, b = _tq_problem(M, N, K, 7 * N + K + M, bias=(M == 1))
    y = tq.tq_gemm(x, p, s, b, path=tq.PATH_DECODE)
    check_tq_gemm(x, p, s, b, y, label=f"{M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(17, 256, 64), (128, 256, 1088), (200, 1000, 1024),
                                   (300, 512, 4096), (129, 257, 128), (512, 4096, 4096)])
def test_tq_prefill(M, N, K):
    need_cuda()
    x, p, s, b = _tq_problem(M, N, K, 3 * M + N + K, outlier_rows=0.01)
    y = tq.tq_gemm(x, p, s, b, path=tq.PATH_PREFILL)
    rows = None if M * N <= 300 * 1000 else np.arange(0, M, 7)
    check_tq_gemm(x, p, s, b, y, rows=rows, label=f"prefill {M}x{N}x{K}")


@pytest.mark.parametrize("M,K", [(1, 5), (3, 1001), (20, 4095), (2, 7)])
def test_tq_generic_ragged_k(M, K):
    need_cuda()
    x, p, s, b = _tq_problem(M, 77, K, 5 + K)
    y = tq.tq_gemm(x, p, s, b)                       # AUTO must route to the generic kernel
    check_tq_gemm(x, p, s, b, y, label=f"generic K={K}")


def test_tq_unaligned_x_goes_generic():
    need_cuda()
    x, p, s, b = _tq_problem(4, 300, 512, 99)
    buf = torch.empty(x.numel() + 1, dtype=torch.float16, device="cuda")
    buf[1:] = x.reshape(-1)
    xu = buf[1:].view(x.shape)
    y = tq.tq_gemm(xu, p, s, b)
    check_tq_gemm(x, p, s, b, y)
    with pytest.raises(tq.TQError):
        tq.tq_gemm(xu, p, s, b, path=tq.PATH_DECODE)


def test_config0_auto_m1():
    need_cuda()
    w = I.weights(1024, 1024, I.seed_for(0, 0, 0), device="cuda")
    p, s = tq.tq_quantize_pack(w)
    x = I.activations(1, 1024, I.seed_for(0, 0, 0), device="cuda")
    y = tq.tq_gemm(x, p, s)
    check_tq_gemm(x, p, s, None, y, label="config 0")


@pytest.mark.parametrize("M", [1, 3, 8, 11, 16])
@pytest.mark.parametrize("path", [tq.PATH_DECODE, tq.PATH_GENERIC])
def test_w4g_small_m(M, path):
    need_cuda()
    x, qw, sc, b = _w4_problem(M, 1000, 1152, 300 + M)
    y = tq.w4g_gemm(x, qw, sc, b, path=path)
    check_w4g_gemm(x, qw, sc, b, y, label=f"w4g M={M} path={path}")


@pytest.mark.parametrize("N,K", [(200, 14336), (1024, 4096), (129, 128), (4096, 1024)])
def test_w4g_decode_shapes(N, K):
    need_cuda()
    for M in (1, 16):
        x, qw, sc, b = _w4_problem(M, N, K, N + K + M)
        y = tq.w4g_gemm(x, qw, sc, b, path=tq.PATH_DECODE)
        check_w4g_gemm(x, qw, sc, b, y, label=f"w4g {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(17, 256, 128), (256, 1000, 1024), (300, 512, 4096)])
def test_w4g_prefill(M, N, K):
    need_cuda()
    x, qw, sc, b = _w4_problem(M, N, K, 5 * M + N + K)
    y = tq.w4g_gemm(x, qw, sc, b, path=tq.PATH_PREFILL)
    check_w4g_gemm(x, qw, sc, b, y, label=f"w4g prefill {M}x{N}x{K}")


def test_validate_counts_code_11():
    need_cuda()
    p = torch.full((5, 3), 0x55, dtype=torch.uint8, device="cuda")     # K = 10 -> 3 bytes/row
    assert tq.tq_validate_packed(p, 10) == 0
    p[1, 0] = 0b11_01_01_01          # code 11 inside K
    p[3, 2] = 0b11_01_01_01          # code 11 in the padding of the last byte (k = 11 >= K): ok
    p[4, 2] = 0b01_01_01_11          # code 11 at k = 8 < K
    assert tq.tq_validate_packed(p, 10) == 2


# M > 8 has two consumer layouts (both token groups per warp, or one group per warp when every
# CTA has a single stage and there are more CTAs than SMs): cover both, with a partial second
# token group, for both formats.
@pytest.mark.parametrize("M", [9, 12, 16])
@pytest.mark.parametrize("N,K", [(4096, 4096), (1024, 4096), (4096, 14336)])
def test_decode_m_gt_8_layouts(M, N, K):
    need_cuda()
    x, p, s, b = _tq_problem(M, N, K, 700 + M + N // 64)
    y = tq.tq_gemm(x, p, s, b, path=tq.PATH_DECODE)
    check_tq_gemm(x, p, s, b, y, cols=np.arange(0, N, 7), label=f"tq decode M={M} {N}x{K}")
    xw, qw, sc, bw = _w4_problem(M, N, K, 800 + M)
    yw = tq.w4g_gemm(xw, qw, sc, bw, path=tq.PATH_DECODE)
    check_w4g_gemm(xw, qw, sc, bw, yw, cols=np.arange(0, N, 7), label=f"w4g decode M={M} {N}x{K}")


# Mid-M prefill: narrow token tiles and K split over a cluster (S = 2..8 CTAs, uneven K slices),
# reduced through distributed shared memory.
@pytest.mark.parametrize("M,N,K", [(40, 384, 1088), (100, 1000, 1152), (64, 3584, 3584), (130, 4608, 3584)])
def test_prefill_split_k(M, N, K):
    need_cuda()
    x, p, s, b = _tq_problem(M, N, K, 900 + M)
    y, buf = guarded_empty(M, N)
    tq.tq_gemm(x, p, s, b, y=y, path=tq.PATH_PREFILL)
    torch.cuda.synchronize()
    check_canaries(buf, M, N, f"split-K M={M}")
    check_tq_gemm(x, p, s, b, y, cols=np.arange(0, N, 3), label=f"tq prefill split-K M={M} {N}x{K}")
    xw, qw, sc, bw = _w4_problem(M, N, K // 128 * 128, 950 + M)
    yw, bufw = guarded_empty(M, N)
    tq.w4g_gemm(xw, qw, sc, bw, y=yw, path=tq.PATH_PREFILL)
    torch.cuda.synchronize()
    check_canaries(bufw, M, N, f"w4g split-K M={M}")
    check_w4g_gemm(xw, qw, sc, bw, yw, cols=np.arange(0, N, 3), label=f"w4g prefill split-K M={M} {N}x{K}")


# M > 16 on the decode path: token chunks of 16 over grid z (ragged last chunk, several row
# blocks and K slices per chunk), both formats; M = 16 is the single-chunk reference point.
@pytest.mark.parametrize("M", [17, 24, 32, 33, 48, 64])
@pytest.mark.parametrize("N,K", [(1000, 1088), (4096, 4096), (3584, 18944)])
def test_decode_token_chunks(M, N, K):
    need_cuda()
    cols = None if N <= 1000 else np.arange(0, N, 11)
    x, p, s, b = _tq_problem(M, N, K, 1200 + M + N // 64)
    y, buf = guarded_empty(M, N)
    tq.tq_gemm(x, p, s, b, y=y, path=tq.PATH_DECODE)
    torch.cuda.synchronize()
    check_canaries(buf, M, N, f"chunks M={M}")
    check_tq_gemm(x, p, s, b, y, cols=cols, label=f"tq decode chunks M={M} {N}x{K}")
    Kw = K // 128 * 128
    xw, qw, sc, bw = _w4_problem(M, N, Kw, 1300 + M)
    yw, bufw = guarded_empty(M, N)
    tq.w4g_gemm(xw, qw, sc, bw, y=yw, path=tq.PATH_DECODE)
    torch.cuda.synchronize()
    check_canaries(bufw, M, N, f"w4g chunks M={M}")
    check_w4g_gemm(xw, qw, sc, bw, yw, cols=cols, label=f"w4g decode chunks M={M} {N}x{Kw}")


def test_decode_token_chunks_limit():
    need_cuda()
    x, p, s, b = _tq_problem(65, 256, 512, 1400)
    with pytest.raises(tq.TQError):
        tq.tq_gemm(x, p, s, b, path=tq.PATH_DECODE)   # 64 tokens at most on the decode path
