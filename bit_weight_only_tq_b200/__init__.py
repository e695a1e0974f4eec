"""Python binding of libtq.so (weight-only low-bit linear layer for B200, sm_100a).

Argument marshalling only: every step of the computation runs in the library's CUDA kernels.
PyTorch supplies device memory and the current stream.  There is no CPU fallback: importing
this package fails loudly if the shared library is missing and cannot be built.

Functions mirror the C ABI in include/tq.h:
    tq_quantize_pack, tq_gemm, w4g_quantize_pack, w4g_gemm, tq_validate_packed,
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
    "tq_gemm_grouped", "w4g_gemm_grouped",
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
    "tq_select_path": [_int, _i64, _i64, _i64, _int],
    "tq_device_status": [],
    "tq_status_string": [_int],
    "tq_version": [],
}
for _name, _args in _SIGS.items():
    _f = getattr(lib, _name)
    _f.argtypes = _args
    _f.restype = ctypes.c_char_p if _name == "tq_status_string" else ctypes.c_int


def header_functions(path: str = HEADER):
    """Names of the functions declared in include/tq.h."""
    with open(path) as f:
        txt = f.read()
    return sorted(set(re.findall(r"^\s*TQ_API\s+(?:int|const char\*)\s+(\w+)\s*\(", txt, re.M)))


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
