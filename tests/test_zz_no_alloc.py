"""tq_gemm_batch_noalloc: the batch call whose scratch is the library's static device array.

Collected last so that it also runs after every other test has used the library.  Two calls in
a row on the same shapes (different inputs) must each match tq_gemm_batch with a workspace of
its own within the tests' error bound, and match the oracle; the second call checks that the
shared scratch is left ready by the first."""
import numpy as np
import pytest
import torch

import bit_weight_only_tq_b200 as tq
import tq_inputs as I
from gpu_util import bits, check_canaries, check_tq_gemm, f16np, gpu, guarded_empty, need_cuda

import oracle as O

pytestmark = gpu

LLAMA_LAYER = [(4096, 4096), (1024, 4096), (1024, 4096), (4096, 4096), (14336, 4096), (14336, 4096),
               (4096, 14336)]
SMALL = [(300, 512), (77, 4096), (129, 64)]


def _items(shapes, M, seed):
    xs, ps, ss, bs = [], [], [], []
    for i, (N, K) in enumerate(shapes):
        p, s = tq.tq_quantize_pack(I.weights(N, K, seed + i, device="cuda"))
        xs.append(I.activations(M, K, seed + 100 + i, device="cuda", outlier_row_frac=0.01))
        ps.append(p)
        ss.append(s)
        bs.append(I.bias(N, seed + i, device="cuda") if i % 2 == 0 else None)
    return xs, ps, ss, bs


@pytest.mark.parametrize("M", [1, 16, 32])
@pytest.mark.parametrize("shapes", [SMALL, LLAMA_LAYER], ids=["small", "llama_layer"])
def test_noalloc_matches_workspace_call_twice(shapes, M):
    need_cuda()
    ws = tq.batch_workspace()
    for call in range(2):
        xs, ps, ss, bs = _items(shapes, M, 7000 + 97 * call + M)
        out = [guarded_empty(M, N) for N, _ in shapes]
        ys, bufs = [y for y, _ in out], [b for _, b in out]
        tq.tq_gemm_batch_noalloc(xs, ps, ss, bs, ys)
        want = tq.tq_gemm_batch(xs, ps, ss, bs, workspace=ws)
        torch.cuda.synchronize()
        assert tq.tq_device_status() == 0
        for (N, K), x, p, s, b, y, yw, buf in zip(shapes, xs, ps, ss, bs, ys, want, bufs):
            check_canaries(buf, M, N, f"noalloc call {call} {N}x{K} M={M}")
            cols = None if N <= 4096 else np.arange(0, N, 13)
            # against the call with a workspace: within the error bound of the product
            cc = np.arange(N) if cols is None else cols
            _, bound = O.tq_gemm(f16np(x), p.cpu().numpy()[cc], bits(s)[cc],
                                 None if b is None else f16np(b)[cc], K)
            d = np.abs(f16np(y)[:, cc].astype(np.float64) - f16np(yw)[:, cc].astype(np.float64))
            assert np.all(d <= bound), (call, N, K, M, float(d.max()))
            # and against the oracle itself
            check_tq_gemm(x, p, s, b, y, cols=cols, label=f"noalloc call {call} {N}x{K} M={M}")


def test_noalloc_after_failed_argument_check():
    """A call the library rejects (K not a multiple of 64, found after the scratch was cleared)
    leaves the next call correct."""
    need_cuda()
    xs, ps, ss, bs = _items(SMALL, 4, 91)
    y0 = torch.empty(4, SMALL[0][0], dtype=torch.float16, device="cuda")
    bad = (tq.TqLinear * 1)(tq.TqLinear(xs[0].data_ptr(), ps[0].data_ptr(), ss[0].data_ptr(), None,
                                        y0.data_ptr(), SMALL[0][0], 100, None))
    assert tq.lib.tq_gemm_batch_noalloc(bad, 1, 4, None) == -2
    ys = tq.tq_gemm_batch_noalloc(xs, ps, ss, bs)
    torch.cuda.synchronize()
    assert tq.tq_device_status() == 0
    for (N, K), x, p, s, b, y in zip(SMALL, xs, ps, ss, bs, ys):
        check_tq_gemm(x, p, s, b, y, label=f"noalloc after error {N}x{K}")
