"""Python binding of libtq.so (weight-only low-bit linear layer for B200, sm_100a).

Argument marshalling only: every step of the computation runs in the library's CUDA kernels.
PyTorch supplies device memory and the current stream.  There is no CPU fallback: importing
this package fails loudly if the shared library is missing and cannot be built.

Functions mirror the C ABI in include/tq.h:
    tq_quantize_pack, tq_gemm, w4g_quantize_pack, w4g_gemm, tq_validate_packed,
    tq_gemm_grouped, w4g_gemm_grouped, tq_gemm_batch, w4g_gemm_batch, tq_batch_workspace_size,
    tq_select_path, tq_device_status, tq_status_string
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

from . import build as _build

__all__ = [
    "TQError", "lib", "lib_path",
    "TQ_OK", "TQ_F32", "TQ_F16", "PATH_AUTO", "PATH_DECODE", "PATH_PREFILL", "PATH_GENERIC",
    "FMT_TERNARY", "FMT_W4G128",
    "tq_quantize_pack", "tq_gemm", "w4g_quantize_pack", "w4g_gemm", "tq_validate_packed",
    "tq_gemm_grouped", "w4g_gemm_grouped", "tq_gemm_batch", "w4g_gemm_batch", "batch_workspace",
    "tq_batch_workspace_size", "TqLinear", "w4g_quantize_pack_ex", "w4g_gemm_zp", "w4g_repack_act_order",
    "tq_permute_columns", "BATCH_AUTO", "BATCH_MMA_SYNC", "BATCH_TENSOR_CORE",
    "tq_select_path", "tq_device_status", "tq_status_string", "header_functions",
]

TQ_OK = 0
TQ_F32, TQ_F16 = 0, 1
PATH_AUTO, PATH_DECODE, PATH_PREFILL, PATH_GENERIC = 0, 1, 2, 3
FMT_TERNARY, FMT_W4G128 = 0, 1

_HERE = os.path.dirname(os.path.abspath(__file__))
HEADER = os.path.join(os.path.dirname(_HERE), "include", "tq.h")


def _load():
    path = _build.LIB
    if _build.needs_build():
        path = _build.build()
    if not os.path.exists(path):
        raise ImportError(f"libtq.so not found at {path} and could not be built")
    return ctypes.CDLL(path), path


lib, lib_path = _load()

_vp, _i64, _int = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int


class TqLinear(ctypes.Structure):
    """struct tq_linear of include/tq.h: one linear of a batch call (device pointers)."""
    _fields_ = [("x", ctypes.c_void_p), ("w", ctypes.c_void_p), ("scale", ctypes.c_void_p),
                ("bias", ctypes.c_void_p), ("y", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("zeros", ctypes.c_void_p)]


_SIGS = {
    "tq_quantize_pack": [_vp, _int, _vp, _vp, _i64, _i64, _vp],
    "tq_gemm": [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp],
    "tq_gemm_ex": [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _vp],
    "w4g_quantize_pack": [_vp, _int, _vp, _vp, _i64, _i64, _vp],
    "w4g_gemm": [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp],
    "w4g_gemm_ex": [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _vp],
    "tq_validate_packed": [_vp, _i64, _i64, _vp, _vp],
    "tq_gemm_grouped": [_vp, _int, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _vp],
    "w4g_gemm_grouped": [_vp, _int, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _vp],
    "tq_gemm_batch": [_vp, _int, _i64, _vp, ctypes.c_size_t, _vp],
    "tq_gemm_batch_next": [_vp, _int, _i64, _vp, ctypes.c_size_t, _int, _vp, _int, _i64, _vp],
    "w4g_gemm_batch_next": [_vp, _int, _i64, _vp, ctypes.c_size_t, _int, _vp, _int, _i64, _vp],
    "w4g_gemm_batch": [_vp, _int, _i64, _vp, ctypes.c_size_t, _vp],
    "tq_batch_workspace_size": [],
    "tq_gemm_batch_ex": [_vp, _int, _i64, _vp, ctypes.c_size_t, _int, _vp],
    "tq_gemm_batch_noalloc": [_vp, _int, _i64, _vp],
    "tq_interleave_packed": [_vp, _vp, _i64, _i64, _vp],
    "w4g_gemm_batch_ex": [_vp, _int, _i64, _vp, ctypes.c_size_t, _int, _vp],
    "tq_debug_set_wait_limit": [ctypes.c_longlong],
    "tq_debug_skip_activation_loads": [_int],
    "w4g_quantize_pack_ex": [_vp, _int, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _vp],
    "w4g_gemm_zp": [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp],
    "w4g_gemm_zp_ex": [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _vp],
    "w4g_repack_act_order": [_vp, _vp, _vp, _i64, _i64, _vp],
    "tq_permute_columns": [_vp, _vp, _vp, _i64, _i64, _vp],
    "tq_shard_plan": [_int, _int, _i64, _i64, _int, _int, _vp],
    "tq_select_path": [_int, _i64, _i64, _i64, _int],
    "tq_device_status": [],
    "tq_status_string": [_int],
    "tq_version": [],
}
for _name, _args in _SIGS.items():
    _f = getattr(lib, _name)
    _f.argtypes = _args
    _f.restype = {"tq_status_string": ctypes.c_char_p, "tq_batch_workspace_size": ctypes.c_size_t}.get(_name, ctypes.c_int)


def header_functions(path: str = HEADER):
    """Names of the functions declared in include/tq.h."""
    with open(path) as f:
        txt = f.read()
    return sorted(set(re.findall(r"^\s*TQ_API\s+(?:int|size_t|const char\*)\s+(\w+)\s*\(", txt, re.M)))


class TQError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {tq_status_string(status)} ({status})")


def tq_status_string(status: int) -> str:
    return lib.tq_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != TQ_OK:
        raise TQError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, dtype, name, ndim=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims")


def tq_quantize_pack(w: torch.Tensor, packed: torch.Tensor | None = None,
                     scale: torch.Tensor | None = None, stream=None):
    """Ternarise + pack W[N,K] (fp32/fp16) -> (packed uint8 [N, ceil(K/4)], scale fp16 [N])."""
    if w.dtype not in (torch.float32, torch.float16):
        raise ValueError("w must be float32 or float16")
    _need(w, w.dtype, "w", 2)
    N, K = w.shape
    if packed is None:
        packed = torch.empty(N, (K + 3) // 4, dtype=torch.uint8, device=w.device)
    if scale is None:
        scale = torch.empty(N, dtype=torch.float16, device=w.device)
    _need(packed, torch.uint8, "packed", 2)
    _need(scale, torch.float16, "scale", 1)
    dt = TQ_F16 if w.dtype == torch.float16 else TQ_F32
    _check(lib.tq_quantize_pack(_ptr(w), dt, _ptr(packed), _ptr(scale), N, K, _stream(stream)),
           "tq_quantize_pack")
    return packed, scale


def tq_gemm(x: torch.Tensor, packed: torch.Tensor, scale: torch.Tensor, bias=None, y=None,
            path: int = PATH_AUTO, stream=None) -> torch.Tensor:
    """y[M,N] = x[M,K] . What^T (+ bias) with ternary packed weights."""
    _need(x, torch.float16, "x", 2)
    _need(packed, torch.uint8, "packed", 2)
    _need(scale, torch.float16, "scale", 1)
    _need(bias, torch.float16, "bias", 1)
    M, K = x.shape
    N = packed.shape[0]
    if packed.shape[1] != (K + 3) // 4 or scale.shape[0] != N:
        raise ValueError("packed / scale shapes do not match x")
    if y is None:
        y = torch.empty(M, N, dtype=torch.float16, device=x.device)
    _need(y, torch.float16, "y", 2)
    _check(lib.tq_gemm_ex(_ptr(x), _ptr(packed), _ptr(scale), _ptr(bias), _ptr(y), M, N, K,
                          int(path), _stream(stream)), "tq_gemm")
    return y


def w4g_quantize_pack(w: torch.Tensor, qweight=None, scales=None, stream=None):
    """Symmetric INT4, group 128: W[N,K] -> (qweight int32 [N, K/8], scales fp16 [N, K/128])."""
    if w.dtype not in (torch.float32, torch.float16):
        raise ValueError("w must be float32 or float16")
    _need(w, w.dtype, "w", 2)
    N, K = w.shape
    if qweight is None:
        qweight = torch.empty(N, K // 8, dtype=torch.int32, device=w.device)
    if scales is None:
        scales = torch.empty(N, K // 128, dtype=torch.float16, device=w.device)
    dt = TQ_F16 if w.dtype == torch.float16 else TQ_F32
    _check(lib.w4g_quantize_pack(_ptr(w), dt, _ptr(qweight), _ptr(scales), N, K, _stream(stream)),
           "w4g_quantize_pack")
    return qweight, scales


def w4g_gemm(x: torch.Tensor, qweight: torch.Tensor, scales: torch.Tensor, bias=None, y=None,
             path: int = PATH_AUTO, stream=None) -> torch.Tensor:
    """y[M,N] = x[M,K] . What^T (+ bias) with W4A16 (group 128) weights."""
    _need(x, torch.float16, "x", 2)
    _need(qweight, torch.int32, "qweight", 2)
    _need(scales, torch.float16, "scales", 2)
    _need(bias, torch.float16, "bias", 1)
    M, K = x.shape
    N = qweight.shape[0]
    if qweight.shape[1] * 8 != K or tuple(scales.shape) != (N, K // 128):
        raise ValueError("qweight / scales shapes do not match x")
    if y is None:
        y = torch.empty(M, N, dtype=torch.float16, device=x.device)
    _need(y, torch.float16, "y", 2)
    _check(lib.w4g_gemm_ex(_ptr(x), _ptr(qweight), _ptr(scales), _ptr(bias), _ptr(y), M, N, K,
                           int(path), _stream(stream)), "w4g_gemm")
    return y


def w4g_quantize_pack_ex(w: torch.Tensor, zero_point: bool = False, perm: torch.Tensor | None = None,
                         stream=None):
    """General INT4 pack (group 128): symmetric or asymmetric (zero_point=True), in activation order
    when `perm` (int32 [K], the column processing order) is given.  Returns
    (qweight int32 [N, K/8] in the original column order, scales fp16 [N, K/128],
    zeros uint8 [N, K/128] or None, g_idx int32 [K])."""
    if w.dtype not in (torch.float32, torch.float16):
        raise ValueError("w must be float32 or float16")
    _need(w, w.dtype, "w", 2)
    _need(perm, torch.int32, "perm", 1)
    N, K = w.shape
    qweight = torch.empty(N, K // 8, dtype=torch.int32, device=w.device)
    scales = torch.empty(N, K // 128, dtype=torch.float16, device=w.device)
    zeros = torch.empty(N, K // 128, dtype=torch.uint8, device=w.device) if zero_point else None
    g_idx = torch.empty(K, dtype=torch.int32, device=w.device)
    dt = TQ_F16 if w.dtype == torch.float16 else TQ_F32
    _check(lib.w4g_quantize_pack_ex(_ptr(w), dt, _ptr(perm), _ptr(qweight), _ptr(scales), _ptr(zeros), _ptr(g_idx),
                                    N, K, _stream(stream)), "w4g_quantize_pack_ex")
    return qweight, scales, zeros, g_idx


def w4g_gemm_zp(x: torch.Tensor, qweight: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor, bias=None,
                y=None, path: int = PATH_AUTO, stream=None) -> torch.Tensor:
    """y = x . What^T (+ bias), What = scales[n, k/128] * (u - zeros[n, k/128])."""
    _need(x, torch.float16, "x", 2)
    _need(qweight, torch.int32, "qweight", 2)
    _need(scales, torch.float16, "scales", 2)
    _need(zeros, torch.uint8, "zeros", 2)
    _need(bias, torch.float16, "bias", 1)
    M, K = x.shape
    N = qweight.shape[0]
    if qweight.shape[1] * 8 != K or tuple(scales.shape) != (N, K // 128) or tuple(zeros.shape) != (N, K // 128):
        raise ValueError("qweight / scales / zeros shapes do not match x")
    if y is None:
        y = torch.empty(M, N, dtype=torch.float16, device=x.device)
    _need(y, torch.float16, "y", 2)
    _check(lib.w4g_gemm_zp_ex(_ptr(x), _ptr(qweight), _ptr(scales), _ptr(zeros), _ptr(bias), _ptr(y), M, N, K,
                              int(path), _stream(stream)), "w4g_gemm_zp")
    return y


def w4g_repack_act_order(qweight: torch.Tensor, perm: torch.Tensor, stream=None) -> torch.Tensor:
    """Columns reordered into the quantisation order: out[:, j] = qweight column perm[j]."""
    _need(qweight, torch.int32, "qweight", 2)
    _need(perm, torch.int32, "perm", 1)
    out = torch.empty_like(qweight)
    _check(lib.w4g_repack_act_order(_ptr(qweight), _ptr(perm), _ptr(out), qweight.shape[0], qweight.shape[1] * 8,
                                    _stream(stream)), "w4g_repack_act_order")
    return out


def tq_permute_columns(x: torch.Tensor, perm: torch.Tensor, out=None, stream=None) -> torch.Tensor:
    """out[m, j] = x[m, perm[j]] (fp16)."""
    _need(x, torch.float16, "x", 2)
    _need(perm, torch.int32, "perm", 1)
    if out is None:
        out = torch.empty_like(x)
    _need(out, torch.float16, "out", 2)
    _check(lib.tq_permute_columns(_ptr(x), _ptr(perm), _ptr(out), x.shape[0], x.shape[1], _stream(stream)),
           "tq_permute_columns")
    return out


def _ptr_array(ts):
    arr = (ctypes.c_void_p * len(ts))()
    for i, t in enumerate(ts):
        arr[i] = None if t is None else t.data_ptr()
    return arr


def _grouped(fn, x, weights, scales, biases, ys, wdtype, sdim, what, stream):
    _need(x, torch.float16, "x", 2)
    M, K = x.shape
    count = len(weights)
    if not (1 <= count <= 4) or len(scales) != count:
        raise ValueError("1..4 matrices with one scale tensor each")
    biases = [None] * count if biases is None else list(biases)
    Ns = []
    for w, s, b in zip(weights, scales, biases):
        _need(w, wdtype, "weights", 2)
        _need(s, torch.float16, "scales", sdim)
        _need(b, torch.float16, "bias", 1)
        Ns.append(w.shape[0])
    if ys is None:
        ys = [torch.empty(M, n, dtype=torch.float16, device=x.device) for n in Ns]
    for yv, n in zip(ys, Ns):
        _need(yv, torch.float16, "y", 2)
        if tuple(yv.shape) != (M, n):
            raise ValueError("y shape mismatch")
    nar = (ctypes.c_int64 * count)(*Ns)
    has_bias = any(b is not None for b in biases)
    _check(fn(_ptr(x), count, _ptr_array(weights), _ptr_array(scales),
              _ptr_array(biases) if has_bias else None, _ptr_array(ys), nar, M, K, _stream(stream)), what)
    return ys


def tq_gemm_grouped(x, packed_list, scale_list, bias_list=None, y_list=None, stream=None):
    """Several ternary linears sharing x (e.g. q, k, v) in one launch: returns [y_g]."""
    return _grouped(lib.tq_gemm_grouped, x, packed_list, scale_list, bias_list, y_list, torch.uint8, 1,
                    "tq_gemm_grouped", stream)


def w4g_gemm_grouped(x, qweight_list, scales_list, bias_list=None, y_list=None, stream=None):
    """Several W4A16 linears sharing x in one launch: returns [y_g]."""
    return _grouped(lib.w4g_gemm_grouped, x, qweight_list, scales_list, bias_list, y_list, torch.int32, 2,
                    "w4g_gemm_grouped", stream)


def tq_batch_workspace_size() -> int:
    """Bytes of workspace the batch calls need on the current device."""
    return int(lib.tq_batch_workspace_size())


def batch_workspace(device=None) -> torch.Tensor:
    """A zero-filled workspace for tq_gemm_batch / w4g_gemm_batch on `device` (default: the
    current device).  Zero it again only after a call that failed."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        n = tq_batch_workspace_size()
    return torch.zeros(n, dtype=torch.uint8, device=dev)


BATCH_AUTO, BATCH_MMA_SYNC, BATCH_TENSOR_CORE, BATCH_INTERLEAVED = 0, 1, 2, 16


def tq_interleave_packed(packed: torch.Tensor, out: torch.Tensor = None, stream=None) -> torch.Tensor:
    """Relayout packed ternary rows [N, K/4] (K % 16 == 0) into the pair-interleaved layout that
    tq_gemm_batch(..., interleaved=True) reads; `out` may be `packed` itself."""
    _need(packed, torch.uint8, "packed", 2)
    out = torch.empty_like(packed) if out is None else out
    _need(out, torch.uint8, "out", 2)
    if tuple(out.shape) != tuple(packed.shape):
        raise ValueError("out shape mismatch")
    N, K = packed.shape[0], packed.shape[1] * 4
    _check(lib.tq_interleave_packed(_ptr(packed), _ptr(out), N, K, _stream(stream)), "tq_interleave_packed")
    return out


def _batch(fn, xs, weights, scales, biases, ys, workspace, wdtype, sdim, what, stream, zeros=None, variant=0,
           next_fn=None, next_weights=None, next_M=0, k_per_col=4):
    count = len(weights)
    if not (1 <= count <= 8) or len(scales) != count or len(xs) != count:
        raise ValueError("1..8 linears, each with its x, weights and scales")
    biases = [None] * count if biases is None else list(biases)
    M = xs[0].shape[0]
    items = (TqLinear * count)()
    out = []
    for i, (x, w, s, b) in enumerate(zip(xs, weights, scales, biases)):
        _need(x, torch.float16, "x", 2)
        _need(w, wdtype, "weights", 2)
        _need(s, torch.float16, "scales", sdim)
        _need(b, torch.float16, "bias", 1)
        if x.shape[0] != M:
            raise ValueError("every x of a batch has the same number of tokens M")
        N, K = w.shape[0], x.shape[1]
        y = torch.empty(M, N, dtype=torch.float16, device=x.device) if ys is None else ys[i]
        _need(y, torch.float16, "y", 2)
        if tuple(y.shape) != (M, N):
            raise ValueError("y shape mismatch")
        z = None if zeros is None else zeros[i]
        _need(z, torch.uint8, "zeros", 2)
        items[i] = TqLinear(x.data_ptr(), w.data_ptr(), s.data_ptr(), None if b is None else b.data_ptr(),
                            y.data_ptr(), N, K, None if z is None else z.data_ptr())
        out.append(y)
    if workspace is None:
        raise ValueError("a workspace from batch_workspace() is required")
    _need(workspace, torch.uint8, "workspace", 1)
    if next_weights:
        nxt = (TqLinear * len(next_weights))()
        for i, w in enumerate(next_weights):
            _need(w, wdtype, "next weights", 2)
            nxt[i] = TqLinear(None, w.data_ptr(), None, None, None, w.shape[0], w.shape[1] * k_per_col, None)
        _check(next_fn(items, count, M, _ptr(workspace), workspace.numel(), int(variant), nxt, len(next_weights),
                       int(next_M), _stream(stream)), what)
        return out
    _check(fn(items, count, M, _ptr(workspace), workspace.numel(), int(variant), _stream(stream)), what)
    return out


def tq_gemm_batch(xs, packed_list, scale_list, bias_list=None, y_list=None, workspace=None, stream=None,
                  variant=BATCH_AUTO, interleaved=False, next_packed=None, next_M=0):
    """Independent ternary linears sharing M (each with its own x) in one persistent launch.
    interleaved=True: the packed weights come from tq_interleave_packed.  next_packed / next_M:
    the packed weights and token count of the batch call that follows on this stream (its first
    tiles are prefetched into L2 during this one; tq_gemm_batch_next)."""
    v = int(variant) | (BATCH_INTERLEAVED if interleaved else 0)
    return _batch(lib.tq_gemm_batch_ex, xs, packed_list, scale_list, bias_list, y_list, workspace, torch.uint8, 1,
                  "tq_gemm_batch", stream, variant=v, next_fn=lib.tq_gemm_batch_next if next_packed else None,
                  next_weights=next_packed,
                  next_M=next_M, k_per_col=4)


def w4g_gemm_batch(xs, qweight_list, scales_list, bias_list=None, y_list=None, workspace=None, stream=None,
                   zeros_list=None, variant=BATCH_AUTO, next_qweight=None, next_M=0):
    """Independent W4A16 linears sharing M in one persistent launch (zero-points optional);
    next_qweight / next_M name the batch call that follows (w4g_gemm_batch_next)."""
    return _batch(lib.w4g_gemm_batch_ex, xs, qweight_list, scales_list, bias_list, y_list, workspace, torch.int32, 2,
                  "w4g_gemm_batch", stream, zeros=zeros_list, variant=variant,
                  next_fn=lib.w4g_gemm_batch_next if next_qweight else None, next_weights=next_qweight,
                  next_M=next_M, k_per_col=8)


def tq_gemm_batch_noalloc(xs, packed_list, scale_list, bias_list=None, y_list=None, stream=None):
    """tq_gemm_batch with the library's own static scratch: no workspace argument, nothing
    allocated by the library (the outputs are allocated here only when y_list is None).  Calls
    that may overlap on one device share that scratch and must be serialised."""
    count = len(packed_list)
    if not (1 <= count <= 8) or len(scale_list) != count or len(xs) != count:
        raise ValueError("1..8 linears, each with its x, weights and scales")
    biases = [None] * count if bias_list is None else list(bias_list)
    M = xs[0].shape[0]
    items = (TqLinear * count)()
    out = []
    for i, (x, w, s, b) in enumerate(zip(xs, packed_list, scale_list, biases)):
        _need(x, torch.float16, "x", 2)
        _need(w, torch.uint8, "packed", 2)
        _need(s, torch.float16, "scale", 1)
        _need(b, torch.float16, "bias", 1)
        if x.shape[0] != M:
            raise ValueError("every x of a batch has the same number of tokens M")
        N, K = w.shape[0], x.shape[1]
        y = torch.empty(M, N, dtype=torch.float16, device=x.device) if y_list is None else y_list[i]
        _need(y, torch.float16, "y", 2)
        if tuple(y.shape) != (M, N):
            raise ValueError("y shape mismatch")
        items[i] = TqLinear(x.data_ptr(), w.data_ptr(), s.data_ptr(), None if b is None else b.data_ptr(),
                            y.data_ptr(), N, K, None)
        out.append(y)
    _check(lib.tq_gemm_batch_noalloc(items, count, M, _stream(stream)), "tq_gemm_batch_noalloc")
    return out


def tq_validate_packed(packed: torch.Tensor, K: int, stream=None) -> int:
    """Number of bytes of `packed` holding the invalid code 0b11 among the first K codes."""
    _need(packed, torch.uint8, "packed", 2)
    bad = torch.empty(1, dtype=torch.int32, device=packed.device)
    _check(lib.tq_validate_packed(_ptr(packed), packed.shape[0], K, _ptr(bad), _stream(stream)),
           "tq_validate_packed")
    return int(bad.item())


def tq_select_path(fmt: int, M: int, N: int, K: int, aligned: bool = True) -> int:
    return int(lib.tq_select_path(int(fmt), int(M), int(N), int(K), 1 if aligned else 0))


def tq_device_status() -> int:
    return int(lib.tq_device_status())
