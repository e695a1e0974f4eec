"""Grouped decode (several linears sharing x in one launch) against the oracle."""
import numpy as np
import pytest
import torch

import bit_weight_only_tq_b200 as tq
import tq_inputs as I
from gpu_util import check_canaries, check_tq_gemm, check_w4g_gemm, gpu, guarded_empty, need_cuda

pytestmark = gpu


# M = 32 and 41 take the decode path in token chunks of 16 (the last one ragged), one launch for
# all three matrices
@pytest.mark.parametrize("M", [1, 5, 16, 32, 41])
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
    for M in (8, 64):                     # decode launch, then the per-matrix prefill fallback
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
