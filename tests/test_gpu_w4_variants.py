"""INT4 variants on the GPU against the oracle ([VQ] §5: zero-points, activation order).

Packing is bit-exact (qweight, scales, zeros, g_idx); GEMMs satisfy, element by element,
|y - y_ref| <= 1e-3 + 2e-3 * sum_k |x * What|, with canaries around every output."""
import numpy as np
import pytest
import torch

import bit_weight_only_tq_b200 as tq
import oracle as O
import tq_inputs as I
from gpu_util import bits, check_canaries, gpu, guarded_empty, need_cuda

pytestmark = gpu


def _edge_weights(N, K, seed, dtype=torch.float32):
    w = I.weights(N, K, seed, outlier_frac=0.001).float()
    g = torch.Generator().manual_seed(seed)
    v = w.view(N, K // 128, 128)
    v[0, 0] = 0.0                                         # zero group
    v[1, 0] = v[1, 0].abs()                               # one-sided groups
    v[2, 0] = -v[2, 0].abs()
    v[3, 0] = torch.randint(-12, 13, (128,), generator=g).float() * 2.0 ** -24   # subnormal scale
    v[4, 0, 5] = 3.0                                      # a spike
    return w.to(dtype)


def _check_pack(w, zero_point, perm):
    qw, sc, zp, gi = tq.w4g_quantize_pack_ex(w.cuda(), zero_point=zero_point,
                                             perm=None if perm is None else perm.cuda())
    torch.cuda.synchronize()
    wn = w.numpy()
    pn = None if perm is None else perm.numpy()
    if zero_point:
        rq, rs, rz, rg = O.w4z_quantize_pack(wn, pn)
        assert np.array_equal(zp.cpu().numpy(), rz), "zeros differ"
    elif pn is None:
        rq, rs = O.w4g_quantize_pack(wn)
        rg = np.arange(w.shape[1], dtype=np.int32) // 128
    else:
        rq, rs, rg = O.w4g_quantize_pack_actorder(wn, pn)
    assert np.array_equal(qw.cpu().numpy(), rq), "qweight differs"
    assert np.array_equal(bits(sc), rs), "scales differ"
    assert np.array_equal(gi.cpu().numpy(), rg), "g_idx differs"
    return qw, sc, zp, gi


@pytest.mark.parametrize("zero_point", [False, True])
@pytest.mark.parametrize("act_order", [False, True])
@pytest.mark.parametrize("dtype", [torch.float32, torch.float16])
def test_pack_bit_exact(zero_point, act_order, dtype):
    need_cuda()
    N, K = 40, 1024
    w = _edge_weights(N, K, 3, dtype)
    perm = torch.randperm(K, generator=torch.Generator().manual_seed(9)).to(torch.int32) if act_order else None
    _check_pack(w, zero_point, perm)


def _tie_weights(N, K, seed, np_dtype):
    """Groups whose weights sit exactly on the rounding ties (k + 1/2) s of their own scale s and
    on the representable values next to them: every group holds 7 s (so max|w| / 7 = s for the
    symmetric rule) and every other group also -8 s (so (hi - lo) / 15 = s for the zero-point
    rule, zero 8).  s ranges over fp16 normals and subnormals; for fp16 weights s = m 2^e with a
    5-bit m, so that every tie is itself an fp16 value."""
    rng = np.random.default_rng(seed)
    G = K // 128
    w = np.empty((N, G, 128), dtype=np_dtype)
    for n in range(N):
        for g in range(G):
            if np_dtype == np.float16:
                s0 = np.ldexp(float(rng.integers(1, 32)), int(rng.integers(-23, 6)))
            else:
                s0 = float(np.array([rng.integers(1, 0x5800)], dtype=np.uint16).view(np.float16)[0])
            tie = ((rng.integers(-7, 7, 128) + 0.5) * s0).astype(np_dtype)
            side = rng.integers(0, 3, 128)
            vals = np.where(side == 0, tie, np.where(side == 1, np.nextafter(tie, np_dtype(np.inf)),
                                                     np.nextafter(tie, np_dtype(-np.inf))))
            vals[0] = 7 * s0
            if (n + g) % 2:
                vals[1] = -8 * s0
            w[n, g] = vals
    return w.reshape(N, K)


# 37 x 384: 111 groups, so the last pass of the contiguous-group kernel (16 groups a warp) is ragged
@pytest.mark.parametrize("zero_point", [False, True])
@pytest.mark.parametrize("act_order", [False, True])
@pytest.mark.parametrize("np_dtype", [np.float32, np.float16])
def test_pack_rounding_ties(zero_point, act_order, np_dtype):
    need_cuda()
    N, K = 37, 384
    w = torch.from_numpy(_tie_weights(N, K, 17, np_dtype))
    perm = torch.randperm(K, generator=torch.Generator().manual_seed(5)).to(torch.int32) if act_order else None
    _check_pack(w, zero_point, perm)


def _zp_problem(M, N, K, seed, outlier_rows=0.0):
    w = _edge_weights(N, K, seed)
    qw, sc, zp, _ = tq.w4g_quantize_pack_ex(w.cuda(), zero_point=True)
    x = I.activations(M, K, seed + 1, device="cuda", outlier_row_frac=outlier_rows)
    b = I.bias(N, seed, device="cuda")
    return x, qw, sc, zp, b


def _check_zp(x, qw, sc, zp, b, y, g_idx=None, x_ref=None, cols=None, label=""):
    K = x.shape[1]
    xr = (x if x_ref is None else x_ref).cpu().numpy()
    q, s, z = qw.cpu().numpy(), bits(sc), zp.cpu().numpy()
    yt = y.cpu().numpy()
    bn = None if b is None else b.cpu().numpy()
    if cols is not None:
        q, s, z, yt = q[cols], s[cols], z[cols], yt[:, cols]
        bn = None if bn is None else bn[cols]
    yref, bound = O.w4z_gemm(xr, q, s, z, bn, K, g_idx=None if g_idx is None else g_idx.cpu().numpy())
    r = O.quant_check(yref, yt, bound=bound)
    assert r["ok"], (label, r)


@pytest.mark.parametrize("M,path", [(1, tq.PATH_DECODE), (7, tq.PATH_DECODE), (16, tq.PATH_DECODE),
                                    (40, tq.PATH_DECODE), (16, tq.PATH_PREFILL), (300, tq.PATH_PREFILL),
                                    (3, tq.PATH_GENERIC), (5, tq.PATH_AUTO), (600, tq.PATH_AUTO)])
@pytest.mark.parametrize("N,K", [(300, 1024), (4096, 4096)])
def test_zero_point_gemm(M, path, N, K):
    _zero_point_gemm(M, path, N, K)


# 150 row tiles at M = 256: the last two run in a second launch (their zero points, scales and
# bias from the row offset)
def test_zero_point_prefill_tail_launch():
    _zero_point_gemm(256, tq.PATH_PREFILL, 19150, 1024)


def _zero_point_gemm(M, path, N, K):
    need_cuda()
    x, qw, sc, zp, b = _zp_problem(M, N, K, 11 + M, outlier_rows=0.01)
    y, buf = guarded_empty(M, N)
    tq.w4g_gemm_zp(x, qw, sc, zp, b, y=y, path=path)
    torch.cuda.synchronize()
    check_canaries(buf, M, N, f"zp path={path} M={M}")
    _check_zp(x, qw, sc, zp, b, y, cols=None if N <= 1000 else np.arange(0, N, 7), label=f"zp M={M} path={path}")


@pytest.mark.parametrize("zero_point", [False, True])
@pytest.mark.parametrize("M", [1, 16, 256])
def test_act_order_end_to_end(zero_point, M):
    # pack in activation order (checkpoint layout), repack once, permute x per call, ordinary GEMM;
    # the oracle multiplies the original x by What[n, k] = s[n, g_idx[k]] (...) directly
    need_cuda()
    N, K = 512, 2048
    w = I.weights(N, K, 21, outlier_frac=0.001)
    perm = torch.randperm(K, generator=torch.Generator().manual_seed(5)).to(torch.int32).cuda()
    qw, sc, zp, g_idx = tq.w4g_quantize_pack_ex(w.cuda(), zero_point=zero_point, perm=perm)
    qw_p = tq.w4g_repack_act_order(qw, perm)
    x = I.activations(M, K, 22 + M, device="cuda")
    xp = tq.tq_permute_columns(x, perm)
    assert torch.equal(xp, x[:, perm.long()])
    y = tq.w4g_gemm_zp(xp, qw_p, sc, zp) if zero_point else tq.w4g_gemm(xp, qw_p, sc)
    torch.cuda.synchronize()
    xn, qn, sb, gn = x.cpu().numpy(), qw.cpu().numpy(), bits(sc), g_idx.cpu().numpy()
    if zero_point:
        yref, bound = O.w4z_gemm(xn, qn, sb, zp.cpu().numpy(), None, K, g_idx=gn)
    else:
        yref, bound = O.w4g_gemm_actorder(xn, qn, sb, gn, None, K)
    r = O.quant_check(yref, y.cpu().numpy(), bound=bound)
    assert r["ok"], r


def test_repack_moves_every_nibble():
    need_cuda()
    N, K = 8, 256
    u = torch.randint(0, 16, (N, K), generator=torch.Generator().manual_seed(2))
    qw = torch.from_numpy(O.pack_nibbles(u.numpy())).cuda()
    perm = torch.randperm(K, generator=torch.Generator().manual_seed(3)).to(torch.int32)
    out = tq.w4g_repack_act_order(qw, perm.cuda())
    got = O.unpack_nibbles(out.cpu().numpy())
    assert np.array_equal(got, u.numpy()[:, perm.numpy()])


@pytest.mark.parametrize("variant,M", [(tq.BATCH_MMA_SYNC, 1), (tq.BATCH_MMA_SYNC, 16), (tq.BATCH_TENSOR_CORE, 1),
                                       (tq.BATCH_TENSOR_CORE, 32)])
def test_zero_point_batch(variant, M):
    need_cuda()
    shapes = [(1000, 1152), (200, 4096), (4096, 4096)]
    probs = [_zp_problem(M, N, K, 31 + i) for i, (N, K) in enumerate(shapes)]
    ws = tq.batch_workspace()
    ys = tq.w4g_gemm_batch([p[0] for p in probs], [p[1] for p in probs], [p[2] for p in probs],
                           [p[4] for p in probs], workspace=ws, zeros_list=[p[3] for p in probs], variant=variant)
    torch.cuda.synchronize()
    for (x, qw, sc, zp, b), y, (N, K) in zip(probs, ys, shapes):
        _check_zp(x, qw, sc, zp, b, y, cols=None if N <= 1000 else np.arange(0, N, 7), label=f"zp batch {N}x{K}")
