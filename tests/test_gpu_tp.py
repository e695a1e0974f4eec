"""Tensor-parallel shards through the CUDA kernels on one GPU: the ranks of a 2-way split are
run one after the other and combined on the host (concatenation for a row split, sum for a K
split), then compared with the unsharded oracle product ([TQ] §5.2, [VQ] §4.2)."""
import numpy as np
import pytest
import torch

import bit_weight_only_tq_b200 as tq
from bit_weight_only_tq_b200 import tp
import oracle as O
import tq_inputs as I
from gpu_util import bits, gpu, need_cuda

pytestmark = gpu


@pytest.mark.parametrize("fmt", [tq.FMT_TERNARY, tq.FMT_W4G128])
@pytest.mark.parametrize("mode", [tp.SHARD_ROWS, tp.SHARD_K])
@pytest.mark.parametrize("M", [1, 16, 300])
def test_two_way_split(fmt, mode, M):
    need_cuda()
    world, N, K = 2, 1000, 4096
    w = I.weights(N, K, 3, device="cuda")
    x = I.activations(M, K, 4, device="cuda")
    b = I.bias(N, 5, device="cuda")
    if fmt == tq.FMT_TERNARY:
        p, s = tq.tq_quantize_pack(w)
        z = None
    else:
        p, s, z, _ = tq.w4g_quantize_pack_ex(w, zero_point=True)
    parts = []
    for rank in range(world):
        xl = tp.shard_activations(x, fmt, mode, N, world, rank)
        if fmt == tq.FMT_TERNARY:
            pl, sl, _ = tp.shard_ternary(p, s, K, mode, world, rank)
            zl = None
        else:
            pl, sl, zl, _ = tp.shard_w4g(p, s, z, mode, world, rank)
        if mode == tp.SHARD_ROWS:
            sp = tp.shard_plan(fmt, mode, N, K, world, rank)
            bl = b[sp.row0:sp.row0 + sp.rows].contiguous()
        else:
            bl = b if rank == 0 else None
        y = tq.tq_gemm(xl, pl, sl, bl) if fmt == tq.FMT_TERNARY else tq.w4g_gemm_zp(xl, pl, sl, zl, bl)
        parts.append(y.float())
    y = torch.cat(parts, dim=1) if mode == tp.SHARD_ROWS else (parts[0] + parts[1])
    y = y.half().cpu().numpy().astype(np.float64)
    xn, bn = x.cpu().numpy(), b.cpu().numpy()
    if fmt == tq.FMT_TERNARY:
        yref, bound = O.tq_gemm(xn, p.cpu().numpy(), bits(s), bn, K)
    else:
        yref, bound = O.w4z_gemm(xn, p.cpu().numpy(), bits(s), z.cpu().numpy(), bn, K)
    slack = (world + 1) * 2.0 ** -11 * np.abs(yref)
    assert np.all(np.abs(y - yref) <= bound + slack)
