"""Tensor-parallel sharding of the packed linear layers ([TQ] §5.2, [VQ] §4.2).

Plumbing only: which part of a packed matrix a rank holds comes from the library's
``tq_shard_plan`` (the packed-factor rule of ``_adjust_shard_indexes_for_packing``); the GEMM on
the shard is the library's; the exchange is a ``torch.distributed`` collective (NCCL on GPUs).

  TQ_SHARD_ROWS  split the output rows N: a rank computes y[:, rows] with every column of x;
                 the ranks' outputs are concatenated (all-gather).
  TQ_SHARD_K     split the input columns K: a rank computes the partial sum over its columns;
                 the partials are summed (all-reduce).  The ternary row scale belongs to the
                 FULL row, so every rank keeps all N scales: they are broadcast from rank 0,
                 never gathered (gathering would concatenate world copies) nor recomputed from
                 a shard (a shard's mean |w| is a different number).
"""
from __future__ import annotations

import ctypes

import torch

from . import FMT_TERNARY, FMT_W4G128, TQError, lib, tq_gemm, w4g_gemm, w4g_gemm_zp

SHARD_ROWS, SHARD_K = 0, 1


class TqShard(ctypes.Structure):
    """struct tq_shard of include/tq.h."""
    _fields_ = [("row0", ctypes.c_int64), ("rows", ctypes.c_int64), ("k0", ctypes.c_int64),
                ("cols", ctypes.c_int64), ("packed0", ctypes.c_int64), ("packed", ctypes.c_int64),
                ("group0", ctypes.c_int64), ("groups", ctypes.c_int64), ("scale_full", ctypes.c_int)]


def shard_plan(fmt: int, mode: int, N: int, K: int, world: int, rank: int) -> TqShard:
    out = TqShard()
    st = lib.tq_shard_plan(int(fmt), int(mode), int(N), int(K), int(world), int(rank), ctypes.byref(out))
    if st != 0:
        raise TQError(st, "tq_shard_plan")
    return out


def shard_ternary(packed: torch.Tensor, scale: torch.Tensor, K: int, mode: int, world: int, rank: int):
    """This rank's (packed [rows, packed cols] contiguous, scale, K of the shard)."""
    sp = shard_plan(FMT_TERNARY, mode, packed.shape[0], K, world, rank)
    p = packed[sp.row0:sp.row0 + sp.rows, sp.packed0:sp.packed0 + sp.packed].contiguous()
    s = scale if sp.scale_full else scale[sp.row0:sp.row0 + sp.rows].contiguous()
    return p, s, sp.cols


def shard_w4g(qweight: torch.Tensor, scales: torch.Tensor, zeros, mode: int, world: int, rank: int):
    """This rank's (qweight, scales, zeros or None, K of the shard)."""
    K = qweight.shape[1] * 8
    sp = shard_plan(FMT_W4G128, mode, qweight.shape[0], K, world, rank)
    rows = slice(sp.row0, sp.row0 + sp.rows)
    q = qweight[rows, sp.packed0:sp.packed0 + sp.packed].contiguous()
    s = scales[rows, sp.group0:sp.group0 + sp.groups].contiguous()
    z = None if zeros is None else zeros[rows, sp.group0:sp.group0 + sp.groups].contiguous()
    return q, s, z, sp.cols


def shard_activations(x: torch.Tensor, fmt: int, mode: int, N: int, world: int, rank: int) -> torch.Tensor:
    """The columns of x this rank multiplies (all of them for a row split)."""
    sp = shard_plan(fmt, mode, N, x.shape[1], world, rank)
    return x if mode == SHARD_ROWS else x[:, sp.k0:sp.k0 + sp.cols].contiguous()


def broadcast_scale(scale: torch.Tensor, group=None) -> torch.Tensor:
    """Every rank receives rank 0's full scale vector ([TQ] §5.2: broadcast, not all-gather)."""
    import torch.distributed as dist

    dist.broadcast(scale, src=0, group=group)
    return scale


def combine(y_local: torch.Tensor, mode: int, N: int, world: int, group=None) -> torch.Tensor:
    """The full y from the ranks' outputs: concatenation along N (row split) or sum (K split)."""
    import torch.distributed as dist

    if world == 1:
        return y_local
    if mode == SHARD_K:
        dist.all_reduce(y_local, op=dist.ReduceOp.SUM, group=group)
        return y_local
    M = y_local.shape[0]
    rmax = -(-N // world)  # row counts differ by at most one: pad to the largest
    buf = torch.zeros(M, rmax, dtype=y_local.dtype, device=y_local.device)
    buf[:, :y_local.shape[1]] = y_local
    parts = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(parts, buf, group=group)
    cols = []
    for r in range(world):
        rows = N * (r + 1) // world - N * r // world
        cols.append(parts[r][:, :rows])
    return torch.cat(cols, dim=1)


def tp_gemm(x: torch.Tensor, packed_local, scale_local, bias, mode: int, N: int, world: int, rank: int,
            group=None, fmt: int = FMT_TERNARY, zeros_local=None) -> torch.Tensor:
    """One tensor-parallel linear: this rank's GEMM on its shard, then the collective.  x is the
    full activation [M, K]; the bias is added once (rank 0 for a K split)."""
    xl = shard_activations(x, fmt, mode, N, world, rank)
    if mode == SHARD_ROWS and bias is not None:
        sp = shard_plan(fmt, mode, N, x.shape[1], world, rank)
        b = bias[sp.row0:sp.row0 + sp.rows].contiguous()
    else:
        b = bias if rank == 0 else None
    if fmt == FMT_TERNARY:
        y = tq_gemm(xl, packed_local, scale_local, b)
    elif zeros_local is not None:
        y = w4g_gemm_zp(xl, packed_local, scale_local, zeros_local, b)
    else:
        y = w4g_gemm(xl, packed_local, scale_local, b)
    return combine(y, mode, N, world, group)
