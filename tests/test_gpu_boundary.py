"""Boundary properties of the C ABI on the GPU: CUDA-graph capture ([TQ] §5.4 stateless
kernels), no temporary device allocations ([TQ] §5.5), determinism, non-default streams,
device ordinal of the caller ([TQ] §5.1), and the device status word."""
import numpy as np
import pytest
import torch

import bit_weight_only_tq_b200 as tq
import tq_inputs as I
from gpu_util import check_tq_gemm, gpu, need_cuda

pytestmark = gpu


def _problem(M, N, K, seed):
    w = I.weights(N, K, seed, device="cuda")
    p, s = tq.tq_quantize_pack(w)
    x = I.activations(M, K, seed, device="cuda")
    b = I.bias(N, seed, device="cuda")
    return x, p, s, b


@pytest.mark.parametrize("M,path", [(1, tq.PATH_DECODE), (16, tq.PATH_DECODE), (256, tq.PATH_PREFILL)])
def test_graph_capture_replays_bitwise(M, path):
    need_cuda()
    x, p, s, b = _problem(M, 2048, 4096, 41 + M)
    y_eager = tq.tq_gemm(x, p, s, b, path=path)
    y = torch.empty_like(y_eager)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        tq.tq_gemm(x, p, s, b, y=y, path=path)   # warm-up outside capture
    torch.cuda.current_stream().wait_stream(stream)
    g = torch.cuda.CUDAGraph()
    y.zero_()
    with torch.cuda.graph(g):
        tq.tq_gemm(x, p, s, b, y=y, path=path)
    y.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(y, y_eager)


def test_deterministic_and_no_allocation():
    need_cuda()
    x, p, s, b = _problem(16, 4096, 14336, 5)
    xp, pp, sp, bp = _problem(512, 1024, 4096, 6)
    qw, qs = tq.w4g_quantize_pack(I.weights(1024, 4096, 7, device="cuda"))
    y1 = torch.empty(16, 4096, dtype=torch.float16, device="cuda")
    y2 = torch.empty_like(y1)
    z1 = torch.empty(512, 1024, dtype=torch.float16, device="cuda")
    z2 = torch.empty_like(z1)
    u1 = torch.empty(16, 1024, dtype=torch.float16, device="cuda")
    for _ in range(2):  # warm-up
        tq.tq_gemm(x, p, s, b, y=y1)
        tq.tq_gemm(xp, pp, sp, bp, y=z1)
        tq.w4g_gemm(x[:, :4096].contiguous(), qw, qs, y=u1)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    xs = x[:, :4096].contiguous()
    torch.cuda.synchronize()
    alloc0 = torch.cuda.memory_allocated()
    for _ in range(5):
        tq.tq_gemm(x, p, s, b, y=y1)
        tq.tq_gemm(xp, pp, sp, bp, y=z1)
        tq.w4g_gemm(xs, qw, qs, y=u1)
    tq.tq_gemm(x, p, s, b, y=y2)
    tq.tq_gemm(xp, pp, sp, bp, y=z2)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0
    assert free1 == free0 or abs(free1 - free0) < (2 << 20)   # no library-side device allocation
    assert torch.equal(y1, y2) and torch.equal(z1, z2)


def test_non_default_stream_and_device_status():
    need_cuda()
    x, p, s, b = _problem(4, 1024, 4096, 8)
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        y = tq.tq_gemm(x, p, s, b)
    st.synchronize()
    check_tq_gemm(x, p, s, b, y)
    assert tq.tq_device_status() == 0


def test_current_device_is_used():
    need_cuda()
    dev = torch.cuda.device_count() - 1
    with torch.cuda.device(dev):
        x, p, s, b = _problem(2, 512, 1024, 9)
        y = tq.tq_gemm(x, p, s, b)
        torch.cuda.synchronize()
        assert y.device.index == dev
        check_tq_gemm(x, p, s, b, y)


def test_pack_then_gemm_back_to_back():
    # the GEMMs read weights before waiting for the previous kernel; the pack calls end with a
    # plain-order empty kernel, so a GEMM enqueued right after a pack (no sync) sees its output
    need_cuda()
    import oracle as O
    from gpu_util import bits, check_tq_gemm, check_w4g_gemm
    for trial in range(3):
        w = I.weights(4096, 4096, 70 + trial, device="cuda")
        x = I.activations(4, 4096, 71 + trial, device="cuda")
        p = torch.empty(4096, 1024, dtype=torch.uint8, device="cuda")
        s = torch.empty(4096, dtype=torch.float16, device="cuda")
        p.fill_(0x55)
        s.fill_(0)
        tq.tq_quantize_pack(w, p, s)
        y = tq.tq_gemm(x, p, s, path=tq.PATH_DECODE)
        yb = tq.tq_gemm(x.repeat(64, 1)[:200].contiguous(), p, s, path=tq.PATH_PREFILL)
        qw, sc = tq.w4g_quantize_pack(w)
        yw = tq.w4g_gemm(x, qw, sc, path=tq.PATH_DECODE)
        torch.cuda.synchronize()
        cols = np.arange(0, 4096, 17)
        check_tq_gemm(x, p, s, None, y, cols=cols)
        check_tq_gemm(x.repeat(64, 1)[:200].contiguous(), p, s, None, yb, rows=np.arange(0, 200, 13), cols=cols)
        check_w4g_gemm(x, qw, sc, None, yw, cols=cols)
