"""Tensor-parallel sharding ([TQ] §5.2 scale broadcast, [VQ] §4.2 packed-factor shard rule),
checked on the CPU: the shard plan's arithmetic, and two gloo ranks that shard an oracle-packed
matrix, compute their partial products with the oracle and combine them with the library's
collectives.  The combined result must equal the unsharded oracle product within the stated
bound (plus the fp16 rounding of each rank's partial for a K split)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bit_weight_only_tq_b200 as tq
from bit_weight_only_tq_b200 import tp

import oracle as O
import tq_inputs as I


def test_plan_covers_every_row_and_column_once():
    for fmt, K in ((tq.FMT_TERNARY, 4096), (tq.FMT_W4G128, 4096), (tq.FMT_TERNARY, 1000)):
        for N in (1, 7, 4096, 14336):
            for world in (1, 2, 3, 4, 8):
                rows = []
                for r in range(world):
                    sp = tp.shard_plan(fmt, tp.SHARD_ROWS, N, K, world, r)
                    rows += list(range(sp.row0, sp.row0 + sp.rows))
                    assert sp.k0 == 0 and sp.cols == K and sp.scale_full == 0
                assert rows == list(range(N))
                if K % world == 0 and (K // world) % (128 if fmt == tq.FMT_W4G128 else 4) == 0:
                    pf = 8 if fmt == tq.FMT_W4G128 else 4
                    cols = []
                    for r in range(world):
                        sp = tp.shard_plan(fmt, tp.SHARD_K, N, K, world, r)
                        cols += list(range(sp.k0, sp.k0 + sp.cols))
                        assert sp.rows == N and sp.row0 == 0
                        # the packed-factor rule: offsets and sizes in packed units are the
                        # element offsets and sizes divided by the packed factor
                        assert sp.packed0 * pf == sp.k0 and sp.packed * pf == sp.cols
                        if fmt == tq.FMT_W4G128:
                            assert sp.group0 * 128 == sp.k0 and sp.groups * 128 == sp.cols
                        assert sp.scale_full == (1 if fmt == tq.FMT_TERNARY else 0)
                    assert cols == list(range(K))


def test_plan_rejects_splits_that_cut_a_packed_unit():
    with pytest.raises(tq.TQError):
        tp.shard_plan(tq.FMT_TERNARY, tp.SHARD_K, 64, 4096 + 4, 8, 0)    # 513 columns per rank: not whole bytes
    with pytest.raises(tq.TQError):
        tp.shard_plan(tq.FMT_W4G128, tp.SHARD_K, 64, 4096 + 128, 2, 0)  # 2112 columns: not whole groups
    with pytest.raises(tq.TQError):
        tp.shard_plan(tq.FMT_TERNARY, tp.SHARD_ROWS, 64, 4096, 2, 2)     # rank out of range
    with pytest.raises(tq.TQError):
        tp.shard_plan(7, tp.SHARD_ROWS, 64, 4096, 2, 0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        N, K, M = 37, 512, 3
        W = I.weights(N, K, 5).numpy()
        x = I.activations(M, K, 6)
        b = I.bias(N, 7)
        results = {}
        # ternary, both split modes
        p, s = O.tq_quantize_pack(W)
        pt, st = torch.from_numpy(p), torch.from_numpy(s.view(np.int16)).view(torch.float16)
        for mode in (tp.SHARD_ROWS, tp.SHARD_K):
            pl, sl, Kl = tp.shard_ternary(pt, st, K, mode, world, rank)
            xl = tp.shard_activations(x, tq.FMT_TERNARY, mode, N, world, rank)
            bl = None
            if mode == tp.SHARD_ROWS:
                sp = tp.shard_plan(tq.FMT_TERNARY, mode, N, K, world, rank)
                bl = b[sp.row0:sp.row0 + sp.rows].numpy()
            elif rank == 0:
                bl = b.numpy()
            yl, _ = O.tq_gemm(xl.numpy(), pl.numpy(), sl.view(torch.int16).numpy().view(np.uint16), bl, Kl)
            y = tp.combine(torch.from_numpy(yl.astype(np.float16)), mode, N, world)
            results[("tq", mode)] = y.numpy()
        # W4A16 with zero-points, both modes
        qw, sc, zp, _ = O.w4z_quantize_pack(W)
        qt, stw, zt = torch.from_numpy(qw), torch.from_numpy(sc.view(np.int16)).view(torch.float16), torch.from_numpy(zp)
        for mode in (tp.SHARD_ROWS, tp.SHARD_K):
            ql, sl, zl, Kl = tp.shard_w4g(qt, stw, zt, mode, world, rank)
            xl = tp.shard_activations(x, tq.FMT_W4G128, mode, N, world, rank)
            yl, _ = O.w4z_gemm(xl.numpy(), ql.numpy(), sl.view(torch.int16).numpy().view(np.uint16), zl.numpy(), None, Kl)
            y = tp.combine(torch.from_numpy(yl.astype(np.float16)), mode, N, world)
            results[("w4z", mode)] = y.numpy()
        # the row scale is broadcast from rank 0, not gathered
        sc_b = st.clone() if rank == 0 else torch.zeros_like(st)
        tp.broadcast_scale(sc_b)
        results["scale_equal"] = bool(torch.equal(sc_b.view(torch.int16), st.view(torch.int16)))
        out.put((rank, results))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_combine():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    res = dict(q.get(timeout=300) for _ in range(world))
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    N, K, M = 37, 512, 3
    W = I.weights(N, K, 5).numpy()
    x = I.activations(M, K, 6).numpy()
    b = I.bias(N, 7).numpy()
    p, s = O.tq_quantize_pack(W)
    yref_t, bound_t = O.tq_gemm(x, p, s, b, K)
    qw, sc, zp, _ = O.w4z_quantize_pack(W)
    yref_w, bound_w = O.w4z_gemm(x, qw, sc, zp, None, K)
    for rank in range(world):
        r = res[rank]
        assert r["scale_equal"]
        for key, yref, bound in ((("tq", tp.SHARD_ROWS), yref_t, bound_t), (("tq", tp.SHARD_K), yref_t, bound_t),
                                 (("w4z", tp.SHARD_ROWS), yref_w, bound_w), (("w4z", tp.SHARD_K), yref_w, bound_w)):
            y = r[key].astype(np.float64)
            # a K split sums fp16-rounded partials: allow their rounding on top of the bound
            slack = (world + 1) * 2.0 ** -11 * np.abs(yref) if key[1] == tp.SHARD_K else 2.0 ** -11 * np.abs(yref)
            assert np.all(np.abs(y - yref) <= bound + slack), key
