"""tq_gemm_batch / w4g_gemm_batch (one persistent launch over a list of independent linears)
on the GPU against the oracle, element by element, with output canaries.

The work is cut into equal ranges of stages per CTA, so a row block can be split between CTAs
and summed through the workspace; the shapes below make splits at every position (ragged N,
K that is not a multiple of a stage, items of very different sizes, more CTAs than stages)."""
import numpy as np
import pytest
import torch

import bit_weight_only_tq_b200 as tq
import tq_inputs as I
from gpu_util import check_canaries, check_tq_gemm, check_w4g_gemm, gpu, guarded_empty, need_cuda

pytestmark = gpu


def _workspace():
    return tq.batch_workspace()


def _counters_zero(ws):
    # the first bytes of the workspace are the arrival counters: every call leaves them at zero
    n = 2 * torch.cuda.get_device_properties(0).multi_processor_count
    assert int(ws[: 4 * n].view(torch.int32).abs().sum().item()) == 0


def _tq_items(shapes, M, seed, share_x=False):
    xs, ps, ss, bs = [], [], [], []
    x_shared = {}
    for i, (N, K) in enumerate(shapes):
        w = I.weights(N, K, seed + i, device="cuda")
        p, s = tq.tq_quantize_pack(w)
        if share_x and K in x_shared:
            x = x_shared[K]
        else:
            x = I.activations(M, K, seed + 100 + i, device="cuda", outlier_row_frac=0.01)
            x_shared[K] = x
        xs.append(x)
        ps.append(p)
        ss.append(s)
        bs.append(I.bias(N, seed + i, device="cuda") if i % 2 == 0 else None)
    return xs, ps, ss, bs


def _guarded_ys(M, shapes):
    out = [guarded_empty(M, N) for N, _ in shapes]
    return [y for y, _ in out], [b for _, b in out]


SHAPES = [
    [(1000, 1088)],
    [(300, 512), (77, 4096), (1024, 1024), (129, 64)],
    [(4096, 4096), (1024, 4096), (1024, 4096), (4096, 4096), (14336, 4096), (14336, 4096), (4096, 14336)],
    [(4608, 3584), (3584, 3584), (37888, 3584), (3584, 18944)],
    [(5, 64), (3, 128)],                                            # fewer stages than CTAs
]


VARIANTS = [(tq.BATCH_MMA_SYNC, M) for M in (1, 3, 8, 9, 16)] + \
           [(tq.BATCH_TENSOR_CORE, M) for M in (1, 3, 8, 16, 17, 32)]


@pytest.mark.parametrize("variant,M", VARIANTS)
@pytest.mark.parametrize("si", range(len(SHAPES)))
def test_tq_batch(si, variant, M):
    need_cuda()
    shapes = SHAPES[si]
    xs, ps, ss, bs = _tq_items(shapes, M, 40 * si + M, share_x=(si == 2))
    ys, bufs = _guarded_ys(M, shapes)
    ws = _workspace()
    tq.tq_gemm_batch(xs, ps, ss, bs, ys, workspace=ws, variant=variant)
    torch.cuda.synchronize()
    for (N, K), x, p, s, b, y, buf in zip(shapes, xs, ps, ss, bs, ys, bufs):
        check_canaries(buf, M, N, f"batch {shapes} M={M}")
        cols = None if N <= 4096 else np.arange(0, N, 13)
        check_tq_gemm(x, p, s, b, y, cols=cols, label=f"batch item {N}x{K} M={M}")
    _counters_zero(ws)
    assert tq.tq_device_status() == 0


@pytest.mark.parametrize("variant", [tq.BATCH_MMA_SYNC, tq.BATCH_TENSOR_CORE])
def test_tq_batch_deterministic_and_reusable(variant):
    need_cuda()
    shapes = SHAPES[2]
    M = 4
    xs, ps, ss, bs = _tq_items(shapes, M, 7, share_x=True)
    ws = _workspace()
    first = [y.clone() for y in tq.tq_gemm_batch(xs, ps, ss, bs, workspace=ws, variant=variant)]
    for _ in range(3):
        again = tq.tq_gemm_batch(xs, ps, ss, bs, workspace=ws, variant=variant)
        for a, b in zip(first, again):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    _counters_zero(ws)


# naming the next call (an L2 prefetch of its first weight tiles) moves no output bit: the same
# layer sequence with and without the hints, including a next call of another M, one above the
# mma.sync range (nothing prefetched), one with an empty matrix, and W4A16
@pytest.mark.parametrize("int4", [False, True])
def test_batch_next_hint_changes_nothing(int4):
    need_cuda()
    shapes = SHAPES[2]
    layers = []
    for li in range(2):
        mats = []
        for i, (N, K) in enumerate(shapes):
            w = I.weights(N, K, 60 + 7 * li + i, device="cuda")
            mats.append(tq.w4g_quantize_pack(w) if int4 else tq.tq_quantize_pack(w))
        layers.append(mats)
    ws = _workspace()
    fn = tq.w4g_gemm_batch if int4 else tq.tq_gemm_batch
    key = "next_qweight" if int4 else "next_packed"
    calls = [(1, 0, (1, 1)), (1, 1, (4, 0)), (4, 0, (16, 1)), (16, 1, (32, 0)), (4, 1, (1, 0)), (16, 0, None)]
    xs = {(M, K): I.activations(M, K, 70 + M + K, device="cuda") for M in (1, 4, 16) for K in (4096, 14336)}
    for M, li, nxt in calls:
        X = [xs[(M, K)] for _, K in shapes]
        P = [p for p, _ in layers[li]]
        S = [s for _, s in layers[li]]
        plain = [y.clone() for y in fn(X, P, S, workspace=ws)]
        if nxt is None:
            continue
        nM, nl = nxt
        named = [p for p, _ in layers[nl]]
        if nM == 4:
            named = named[:3] + [named[3][:0]] + named[4:]  # an empty matrix among the next items
        hinted = fn(X, P, S, workspace=ws, **{key: named, "next_M": nM})
        torch.cuda.synchronize()
        for a, b in zip(plain, hinted):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16)), (M, li, nxt)
    _counters_zero(ws)
    assert tq.tq_device_status() == 0


def test_tq_batch_matches_single_calls():
    need_cuda()
    shapes = SHAPES[1]
    M = 16
    xs, ps, ss, bs = _tq_items(shapes, M, 9)
    yb = tq.tq_gemm_batch(xs, ps, ss, bs, workspace=_workspace())
    for x, p, s, b, y in zip(xs, ps, ss, bs, yb):
        y1 = tq.tq_gemm(x, p, s, b, path=tq.PATH_DECODE)
        # both are within the bound of the oracle; they need not be bit-identical (different K
        # splits), but they agree closely
        d = (y.float() - y1.float()).abs().max().item()
        assert d <= 2e-2, d


@pytest.mark.parametrize("variant,M", [(tq.BATCH_MMA_SYNC, 1), (tq.BATCH_MMA_SYNC, 16), (tq.BATCH_TENSOR_CORE, 1),
                                       (tq.BATCH_TENSOR_CORE, 16), (tq.BATCH_TENSOR_CORE, 32)])
def test_tq_batch_edge_rows(variant, M):
    need_cuda()
    from test_gpu_edge_gemm import adversarial_ternary, edge_activations
    shapes = [(200, 4096), (200, 14336)]
    xs, ps, ss, bs = [], [], [], []
    for i, (N, K) in enumerate(shapes):
        p, s = tq.tq_quantize_pack(adversarial_ternary(N, K, 3 + i).cuda())
        xs.append(edge_activations(M, K, 11 + i).cuda())
        ps.append(p)
        ss.append(s)
        bs.append(I.bias(N, i, device="cuda"))
    ys, bufs = _guarded_ys(M, shapes)
    tq.tq_gemm_batch(xs, ps, ss, bs, ys, workspace=_workspace(), variant=variant)
    torch.cuda.synchronize()
    for (N, K), x, p, s, b, y, buf in zip(shapes, xs, ps, ss, bs, ys, bufs):
        check_canaries(buf, M, N)
        check_tq_gemm(x, p, s, b, y, label=f"batch edge {N}x{K} M={M} variant={variant}")


@pytest.mark.parametrize("variant,M", [(tq.BATCH_MMA_SYNC, 1), (tq.BATCH_MMA_SYNC, 5), (tq.BATCH_MMA_SYNC, 16),
                                       (tq.BATCH_TENSOR_CORE, 1), (tq.BATCH_TENSOR_CORE, 16),
                                       (tq.BATCH_TENSOR_CORE, 24)])
def test_w4g_batch(variant, M):
    need_cuda()
    shapes = [(1000, 1152), (4096, 4096), (200, 14336), (129, 128)]
    xs, qs, ss, bs = [], [], [], []
    for i, (N, K) in enumerate(shapes):
        qw, sc = tq.w4g_quantize_pack(I.weights(N, K, 60 + i, device="cuda", outlier_frac=0.001))
        xs.append(I.activations(M, K, 70 + i, device="cuda"))
        qs.append(qw)
        ss.append(sc)
        bs.append(I.bias(N, i, device="cuda") if i != 1 else None)
    ys, bufs = _guarded_ys(M, shapes)
    ws = _workspace()
    tq.w4g_gemm_batch(xs, qs, ss, bs, ys, workspace=ws, variant=variant)
    torch.cuda.synchronize()
    for (N, K), x, q, s, b, y, buf in zip(shapes, xs, qs, ss, bs, ys, bufs):
        check_canaries(buf, M, N)
        check_w4g_gemm(x, q, s, b, y, label=f"w4g batch {N}x{K} M={M}")
    _counters_zero(ws)


def test_tq_batch_in_cuda_graph():
    need_cuda()
    shapes = SHAPES[1]
    M = 8
    xs, ps, ss, bs = _tq_items(shapes, M, 5)
    ws = _workspace()
    ys = [torch.empty(M, N, dtype=torch.float16, device="cuda") for N, _ in shapes]
    tq.tq_gemm_batch(xs, ps, ss, bs, ys, workspace=ws)   # warm-up outside capture
    ref = [y.clone() for y in ys]
    for y in ys:
        y.zero_()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            tq.tq_gemm_batch(xs, ps, ss, bs, ys, workspace=ws)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    for a, b in zip(ref, ys):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    _counters_zero(ws)
