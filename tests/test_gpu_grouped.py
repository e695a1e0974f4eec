"""Grouped decode (several linears sharing x in one launch) against the oracle."""
import numpy as np
import pytest
import torch

import bit_weight_only_tq_b200 as tq
import tq_inputs as I
from gpu_util import check_canaries, check_tq_gemm, check_w4g_gemm, gpu, guarded_empty, need_cuda

pytestmark = gpu


# M <= 16: one decode launch for all three matrices; M = 29, 32, 41: one tensor-core launch
@pytest.mark.parametrize("M", [1, 5, 16, 29, 32, 41])
def test_tq_grouped_qkv(M):
    need_cuda()
    K = 4096
    shapes = [4096, 1024, 1000]          # q, k, and a ragged third matrix
    ws = [tq.tq_quantize_pack(I.weights(N, K, 11 + i, device="cuda")) for i, N in enumerate(shapes)]
    x = I.activations(M, K, 3, device="cuda")
    biases = [I.bias(shapes[0], 1, device="cuda"), None, I.bias(shapes[2], 2, device="cuda")]
    outs = [guarded_empty(M, N) for N in shapes]
    ys = tq.tq_gemm_grouped(x, [p for p, _ in ws], [s for _, s in ws], biases, [y for y, _ in outs])
    torch.cuda.synchronize()
    for (_, buf), N in zip(outs, shapes):
        check_canaries(buf, M, N, f"grouped N={N} M={M}")
    for (p, s), b, y, N in zip(ws, biases, ys, shapes):
        cols = np.arange(0, N, 3)
        check_tq_gemm(x, p, s, b, y, cols=cols, label=f"grouped N={N} M={M}")


def test_tq_grouped_gate_up_and_prefill_fallback():
    need_cuda()
    K = 1024
    ws = [tq.tq_quantize_pack(I.weights(2048, K, 21 + i, device="cuda")) for i in range(2)]
    for M in (8, 64):                     # one decode launch, then one tensor-core prefill launch
        x = I.activations(M, K, 4 + M, device="cuda")
        ys = tq.tq_gemm_grouped(x, [p for p, _ in ws], [s for _, s in ws])
        torch.cuda.synchronize()
        for (p, s), y in zip(ws, ys):
            check_tq_gemm(x, p, s, None, y, cols=np.arange(0, 2048, 5), label=f"gate/up M={M}")


def test_w4g_grouped():
    need_cuda()
    K = 2048
    shapes = [1024, 512]
    ws = [tq.w4g_quantize_pack(I.weights(N, K, 31 + i, device="cuda")) for i, N in enumerate(shapes)]
    x = I.activations(3, K, 5, device="cuda")
    ys = tq.w4g_gemm_grouped(x, [q for q, _ in ws], [s for _, s in ws])
    torch.cuda.synchronize()
    for (q, s), y in zip(ws, ys):
        check_w4g_gemm(x, q, s, None, y, label="w4g grouped")


# Prefill-sized M: one tensor-core launch over the row tiles of every matrix (ragged N per
# matrix, an empty matrix, 2-4 matrices, token tiles of 64 / 128 / 256, K split over clusters).
@pytest.mark.parametrize("fmt,M,shapes,K", [
    ("tq", 200, [1024, 256, 130], 1024),
    ("tq", 300, [640, 0, 384], 4096),
    ("tq", 64, [384, 384, 256, 100], 1088),
    ("tq", 129, [4096, 1024, 1024], 4096),
    ("w4", 256, [512, 200, 128], 2048),
    ("w4", 100, [256, 136], 1152),
    ("tq", 4096, [4096, 4096], 256),      # more than four waves: one launch per matrix
    # 150 row tiles x one token tile: 148 in a first launch, the last 2 (the second matrix's,
    # one of them ragged) in a second launch split over K
    ("tq", 256, [9600, 9550], 1024),
    ("w4", 512, [9600], 1024),            # 75 row tiles x 2 token tiles: the last row tile apart
])
def test_grouped_prefill(fmt, M, shapes, K):
    need_cuda()
    if fmt == "tq":
        ws = [tq.tq_quantize_pack(I.weights(max(N, 1), K, 41 + i, device="cuda")) for i, N in enumerate(shapes)]
        ws = [(p[:N], s[:N]) for (p, s), N in zip(ws, shapes)]
    else:
        ws = [tq.w4g_quantize_pack(I.weights(max(N, 1), K, 51 + i, device="cuda")) for i, N in enumerate(shapes)]
        ws = [(q[:N], s[:N]) for (q, s), N in zip(ws, shapes)]
    x = I.activations(M, K, 7 + M, device="cuda", outlier_row_frac=0.01)
    biases = [I.bias(N, 3 + i, device="cuda") if i % 2 == 0 and N > 0 else None for i, N in enumerate(shapes)]
    outs = [guarded_empty(M, N) for N in shapes]
    fn = tq.tq_gemm_grouped if fmt == "tq" else tq.w4g_gemm_grouped
    ys = fn(x, [w for w, _ in ws], [s for _, s in ws], biases, [y for y, _ in outs])
    torch.cuda.synchronize()
    for (_, buf), N in zip(outs, shapes):
        check_canaries(buf, M, N, f"grouped prefill {fmt} N={N} M={M}")
    check = check_tq_gemm if fmt == "tq" else check_w4g_gemm
    for (w, s), b, y, N in zip(ws, biases, ys, shapes):
        if N == 0:
            continue
        check(x, w, s, b, y, rows=np.arange(0, M, 5 if M <= 512 else 41), cols=np.arange(0, N, 3),
              label=f"grouped prefill {fmt} N={N} M={M} K={K}")
