"""The pair-interleaved ternary layout on the GPU: tq_interleave_packed bit-exact against the
oracle's relayout, and the batch decode on interleaved weights against the oracle product."""
import numpy as np
import pytest
import torch

import bit_weight_only_tq_b200 as tq
import oracle as O
import tq_inputs as I
from gpu_util import check_canaries, check_tq_gemm, gpu, guarded_empty, need_cuda

pytestmark = gpu


@pytest.mark.parametrize("N,K", [(1, 16), (7, 64), (300, 512), (1024, 4096), (37, 14336)])
def test_interleave_matches_oracle(N, K):
    need_cuda()
    w = I.weights(N, K, 60 + N, device="cuda")
    p, _ = tq.tq_quantize_pack(w)
    il = tq.tq_interleave_packed(p)
    torch.cuda.synchronize()
    want = O.tq_interleave(p.cpu().numpy())
    assert np.array_equal(il.cpu().numpy(), want)
    # in place gives the same bytes
    q = p.clone()
    tq.tq_interleave_packed(q, out=q)
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), want)


SHAPES = [
    [(1000, 1088)],
    [(300, 512), (77, 4096), (1024, 1024), (129, 64)],
    [(4096, 4096), (1024, 4096), (1024, 4096), (4096, 4096), (14336, 4096), (14336, 4096), (4096, 14336)],
]


@pytest.mark.parametrize("M", [1, 3, 8, 9, 16])
@pytest.mark.parametrize("si", range(len(SHAPES)))
def test_batch_on_interleaved_weights(si, M):
    need_cuda()
    shapes = SHAPES[si]
    xs, ps, pil, ss, bs = [], [], [], [], []
    for i, (N, K) in enumerate(shapes):
        p, s = tq.tq_quantize_pack(I.weights(N, K, 300 + 10 * si + i, device="cuda"))
        xs.append(I.activations(M, K, 400 + 10 * si + i, device="cuda", outlier_row_frac=0.01))
        ps.append(p)
        pil.append(tq.tq_interleave_packed(p))
        ss.append(s)
        bs.append(I.bias(N, 500 + i, device="cuda") if i % 2 == 0 else None)
    out = [guarded_empty(M, N) for N, _ in shapes]
    ys, bufs = [y for y, _ in out], [b for _, b in out]
    tq.tq_gemm_batch(xs, pil, ss, bs, ys, workspace=tq.batch_workspace(), variant=tq.BATCH_MMA_SYNC, interleaved=True)
    torch.cuda.synchronize()
    assert tq.tq_device_status() == 0
    for (N, K), x, p, s, b, y, buf in zip(shapes, xs, ps, ss, bs, ys, bufs):
        check_canaries(buf, M, N, f"interleaved batch {N}x{K} M={M}")
        cols = None if N <= 4096 else np.arange(0, N, 13)
        # the oracle multiplies the canonical codes: same product
        check_tq_gemm(x, p, s, b, y, cols=cols, label=f"interleaved batch {N}x{K} M={M}")
