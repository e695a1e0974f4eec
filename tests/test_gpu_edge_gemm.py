"""GEMM parity on the method's edge-case rows, every path, against the oracle.

Rows a uniform N(0, 0.02) matrix never produces: all-zero rows (scale 0), constant rows, rows
with one or two nonzero codes and a scale >= 1 whose other codes are all 01, wide exponent
ranges, fp32 subnormal rows (scale underflows to 0), rows of many tiny values.  The activations
carry 1 % of token rows x 20 and, at the positions of the single nonzero codes, tiny values, so
that sum_k |x * What| is small while sum_k |x| is large: a kernel that formed sum_k c x and
sum_k x separately and subtracted them would fail the bound there.

W4A16: all-zero groups (scale 0), subnormal scales with codes clamped to -8 / +7, whole
groups x 10, single-spike groups.

Pass rule, element by element: |y - y_ref| <= 1e-3 + 2e-3 * sum_k |x[m,k] * What[n,k]|.
Every output buffer carries canaries on both sides.
"""
import numpy as np
import pytest
import torch

import bit_weight_only_tq_b200 as tq
import tq_inputs as I
from gpu_util import check_canaries, check_tq_gemm, check_w4g_gemm, gpu, guarded_empty, need_cuda

pytestmark = gpu

SPIKE_K = (777, 3001)   # the positions of the sparse rows' nonzero weights


def adversarial_ternary(N, K, seed):
    """fp32 W[N,K]: N rows cycling through the edge-case kinds ([TQ] §1 / §3.1 rules)."""
    g = torch.Generator().manual_seed(seed)
    rows = []
    for n in range(N):
        kind = n % 9
        if kind == 0:
            r = torch.zeros(K)                                       # scale 0
        elif kind == 1:
            r = torch.full((K,), 0.75)                               # constant: every code +1
        elif kind == 2:                                              # one nonzero, scale 3
            r = torch.zeros(K)
            r[SPIKE_K[0]] = -3.0
        elif kind == 3:                                              # two nonzero, scale 2, noise below t
            r = torch.randn(K, generator=g) * 1e-4
            r[SPIKE_K[0]] = 2.5
            r[SPIKE_K[1]] = -1.5
        elif kind == 4:                                              # one nonzero, scale 40
            r = torch.randn(K, generator=g) * 1e-3
            r[SPIKE_K[1]] = 40.0
        elif kind == 5:                                              # wide exponent range, |w| <= ~1
            e = torch.randint(-140, 0, (K,), generator=g).float()
            r = torch.randn(K, generator=g) * torch.exp2(e)
        elif kind == 6:                                              # fp32 subnormals: scale 0
            r = torch.randint(1, 2 ** 23, (K,), generator=g, dtype=torch.int32).view(torch.float32)
        elif kind == 7:                                              # many tiny values
            r = torch.randn(K, generator=g) * 0.02
            r[::3] = 1e-30
        else:                                                        # dense, large scale
            r = torch.randn(K, generator=g) * 2.0
        rows.append(r.float())
    return torch.stack(rows)


def edge_activations(M, K, seed):
    """x ~ N(0,1) with 1 % of rows (at least one) x 20, and tiny values at the spike positions."""
    x = I.activations(M, K, seed, outlier_row_frac=0.01).float()
    x[:, SPIKE_K[0]] = 1e-3
    x[:, SPIKE_K[1]] = -2e-3
    return x.to(torch.float16)


def _run_tq(M, K, path, N=200, seed=5):
    need_cuda()
    w = adversarial_ternary(N, K, seed).cuda()
    p, s = tq.tq_quantize_pack(w)
    x = edge_activations(M, K, seed + M).cuda()
    b = I.bias(N, seed, device="cuda")
    y, buf = guarded_empty(M, N)
    tq.tq_gemm(x, p, s, b, y=y, path=path)
    torch.cuda.synchronize()
    check_canaries(buf, M, N, f"tq path={path} M={M} K={K}")
    check_tq_gemm(x, p, s, b, y, label=f"edge tq path={path} M={M} K={K}")


@pytest.mark.parametrize("K", [4096, 14336])
@pytest.mark.parametrize("M", [1, 4, 16, 40])
def test_edge_rows_decode(M, K):
    _run_tq(M, K, tq.PATH_DECODE)


@pytest.mark.parametrize("K", [4096, 14336])
@pytest.mark.parametrize("M", [16, 300])
def test_edge_rows_prefill(M, K):
    _run_tq(M, K, tq.PATH_PREFILL)


@pytest.mark.parametrize("K", [4096, 14336])
def test_edge_rows_generic(K):
    _run_tq(5, K, tq.PATH_GENERIC)


def adversarial_w4g(N, K, seed):
    """fp32 W[N,K] whose 128-wide groups cycle through the W4A16 edge cases ([VQ] §5 layout)."""
    g = torch.Generator().manual_seed(seed)
    w = torch.randn(N, K, generator=g) * 0.02
    G = K // 128
    wv = w.view(N, G, 128)
    for n in range(N):
        for gi in range(G):
            kind = (n + 3 * gi) % 6
            if kind == 0:
                wv[n, gi] = 0.0                                      # scale 0
            elif kind == 1:                                          # subnormal scale, clamps
                v = torch.randint(-12, 13, (128,), generator=g).float() * 0.8 * 2.0 ** -24
                v[0], v[1] = 9.6 * 2.0 ** -24, -9.6 * 2.0 ** -24
                wv[n, gi] = v
            elif kind == 2:
                wv[n, gi] *= 10.0                                    # outlier group
            elif kind == 3:                                          # single spike, rest tiny
                wv[n, gi] = torch.randn(128, generator=g) * 1e-5
                wv[n, gi, 17] = 5.0
    return w


@pytest.mark.parametrize("K", [4096, 14336])
@pytest.mark.parametrize("M,path", [(1, tq.PATH_DECODE), (16, tq.PATH_DECODE), (40, tq.PATH_DECODE),
                                    (16, tq.PATH_PREFILL), (300, tq.PATH_PREFILL), (3, tq.PATH_GENERIC)])
def test_edge_groups_w4g(M, K, path):
    need_cuda()
    N = 136
    w = adversarial_w4g(N, K, 21).cuda()
    qw, sc = tq.w4g_quantize_pack(w)
    x = I.activations(M, K, 40 + M, outlier_row_frac=0.01).float()
    x[:, 17::128] = 1e-3                                             # tiny x under the spikes
    x = x.to(torch.float16).cuda()
    b = I.bias(N, 21, device="cuda")
    y, buf = guarded_empty(M, N)
    tq.w4g_gemm(x, qw, sc, b, y=y, path=path)
    torch.cuda.synchronize()
    check_canaries(buf, M, N, f"w4g path={path} M={M} K={K}")
    check_w4g_gemm(x, qw, sc, b, y, label=f"edge w4g path={path} M={M} K={K}")
