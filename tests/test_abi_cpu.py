"""Host-side checks of the C ABI that need no GPU: the library loads, exports every function
declared in include/tq.h, validates arguments before touching the device, and applies the
documented dispatch rule."""
import ctypes
import os

import pytest
import torch

import bit_weight_only_tq_b200 as tq


def test_library_exports_every_header_function():
    names = tq.header_functions()
    assert len(names) == 30
    for n in names:
        assert hasattr(tq.lib, n), n
    for n in ("tq_quantize_pack", "tq_gemm", "w4g_quantize_pack", "w4g_gemm", "tq_validate_packed",
              "tq_select_path", "tq_device_status", "tq_status_string", "tq_gemm_batch", "w4g_gemm_batch",
              "tq_batch_workspace_size"):
        assert n in names


def test_status_strings():
    assert tq.tq_status_string(0) == "ok"
    for s in range(-8, 0):
        assert tq.tq_status_string(s) != "unknown status"
    assert tq.tq_status_string(-99) == "unknown status"
    assert tq.lib.tq_version() >> 16 == 1


NULL = None


@pytest.mark.parametrize("N,K,expect", [(-1, 8, -2), (4, 0, -2), (4, -3, -2), (4, 2 ** 29, -2)])
def test_pack_rejects_bad_shapes(N, K, expect):
    assert tq.lib.tq_quantize_pack(ctypes.c_void_p(16), 0, ctypes.c_void_p(16), ctypes.c_void_p(16),
                                   N, K, NULL) == expect


def test_pack_rejects_dtype_and_null():
    assert tq.lib.tq_quantize_pack(ctypes.c_void_p(16), 7, ctypes.c_void_p(16), ctypes.c_void_p(16), 4, 8, NULL) == -4
    assert tq.lib.tq_quantize_pack(NULL, 0, ctypes.c_void_p(16), ctypes.c_void_p(16), 4, 8, NULL) == -1
    assert tq.lib.w4g_quantize_pack(ctypes.c_void_p(16), 0, ctypes.c_void_p(16), ctypes.c_void_p(16), 4, 100, NULL) == -2
    # empty problem: nothing to do, no pointer needed
    assert tq.lib.tq_quantize_pack(NULL, 0, NULL, NULL, 0, 8, NULL) == 0


def test_gemm_argument_errors_without_gpu():
    p = ctypes.c_void_p(4096)
    assert tq.lib.tq_gemm(p, p, p, NULL, p, -1, 4, 8, NULL) == -2
    assert tq.lib.tq_gemm(p, p, p, NULL, p, 1, 4, 0, NULL) == -2
    assert tq.lib.tq_gemm(NULL, p, p, NULL, p, 1, 4, 8, NULL) == -1
    assert tq.lib.tq_gemm(p, p, NULL, NULL, p, 1, 4, 8, NULL) == -1
    assert tq.lib.tq_gemm(NULL, NULL, NULL, NULL, NULL, 0, 4, 8, NULL) == 0   # empty
    assert tq.lib.tq_gemm(NULL, NULL, NULL, NULL, NULL, 3, 0, 8, NULL) == 0   # empty
    assert tq.lib.tq_gemm_ex(p, p, p, NULL, p, 1, 4, 64, 9, NULL) == -8       # unknown path
    assert tq.lib.w4g_gemm(p, p, p, NULL, p, 1, 4, 100, NULL) == -2           # K % 128
    # forced fast paths refuse shapes they cannot take / misaligned pointers
    assert tq.lib.tq_gemm_ex(p, p, p, NULL, p, 65, 4, 64, 1, NULL) == -8      # decode needs M<=64
    assert tq.lib.tq_gemm_ex(p, p, p, NULL, p, 1, 4, 100, 1, NULL) == -8      # decode needs K%64
    assert tq.lib.tq_gemm_ex(p, p, p, NULL, p, 256, 4, 100, 2, NULL) == -8    # prefill needs K%64
    q = ctypes.c_void_p(4098)
    assert tq.lib.tq_gemm_ex(q, p, p, NULL, p, 1, 4, 64, 1, NULL) == -3       # misaligned x
    assert tq.lib.w4g_gemm_ex(p, p, q, NULL, p, 300, 4, 128, 2, NULL) == -3   # misaligned scales


def test_validate_argument_errors():
    assert tq.lib.tq_validate_packed(ctypes.c_void_p(16), 4, 0, ctypes.c_void_p(16), NULL) == -2
    assert tq.lib.tq_validate_packed(ctypes.c_void_p(16), 4, 8, NULL, NULL) == -1


def test_dispatch_rule():
    T, W = tq.FMT_TERNARY, tq.FMT_W4G128
    # decode for skinny M on shapes the decode kernel takes
    for M in (1, 2, 4, 8, 9, 16):
        assert tq.tq_select_path(T, M, 4096, 4096) == tq.PATH_DECODE
        assert tq.tq_select_path(W, M, 4096, 14336) == tq.PATH_DECODE
    assert tq.tq_select_path(T, 1, 4096, 14336) == tq.PATH_DECODE
    assert tq.tq_select_path(T, 1, 3584, 18944) == tq.PATH_DECODE
    assert tq.tq_select_path(T, 16, 37888, 3584) == tq.PATH_DECODE
    # measured crossover (Qwen2-7B shapes): decode up to M = 16 for both formats (a second
    # 16-token chunk costs more than the tensor-core path); the tensor-core path above
    for M in (17, 24, 32, 33, 40, 48, 64, 512, 2048, 8192):
        assert tq.tq_select_path(T, M, 4096, 4096) == tq.PATH_PREFILL
    for M in (17, 24, 32, 512, 2048, 8192):
        assert tq.tq_select_path(W, M, 14336, 4096) == tq.PATH_PREFILL
    # shapes / alignment the fast kernels do not take
    assert tq.tq_select_path(T, 1, 4096, 4100) == tq.PATH_GENERIC
    assert tq.tq_select_path(T, 1, 4096, 4096, aligned=False) == tq.PATH_GENERIC
    assert tq.tq_select_path(T, 512, 4096, 4095) == tq.PATH_GENERIC
    assert tq.tq_select_path(W, 1, 4096, 4000) == -2
    assert tq.tq_select_path(T, 1, 4096, 0) == -2
    assert tq.tq_select_path(5, 1, 4096, 4096) == -8


def test_grouped_argument_errors_without_gpu():
    p = ctypes.c_void_p(4096)
    arr = (ctypes.c_void_p * 3)(4096, 4096, 4096)
    ns = (ctypes.c_int64 * 3)(64, 64, 64)
    assert tq.lib.tq_gemm_grouped(p, 0, arr, arr, None, arr, ns, 1, 64, None) == -2   # count
    assert tq.lib.tq_gemm_grouped(p, 5, arr, arr, None, arr, ns, 1, 64, None) == -2
    assert tq.lib.tq_gemm_grouped(p, 3, None, arr, None, arr, ns, 1, 64, None) == -1  # null array
    bad = (ctypes.c_int64 * 3)(64, -1, 64)
    assert tq.lib.tq_gemm_grouped(p, 3, arr, arr, None, arr, bad, 1, 64, None) == -2
    assert tq.lib.w4g_gemm_grouped(p, 3, arr, arr, None, arr, ns, 1, 100, None) == -2  # K % 128
    assert tq.lib.tq_gemm_grouped(p, 3, arr, arr, None, arr, ns, 0, 64, None) == 0    # M = 0


def _items(*specs):
    arr = (tq.TqLinear * len(specs))()
    for i, (x, w, sc, y, N, K) in enumerate(specs):
        arr[i] = tq.TqLinear(x, w, sc, None, y, N, K)
    return arr


def test_batch_argument_errors_without_gpu():
    a, q = 4096, 4098  # a 16-byte aligned and a misaligned fake device address
    ws, big = ctypes.c_void_p(1 << 20), 1 << 40
    ok = _items((a, a, a, a, 64, 128))
    assert tq.lib.tq_gemm_batch(ok, 0, 1, ws, big, None) == -2                 # count
    assert tq.lib.tq_gemm_batch(ok, 9, 1, ws, big, None) == -2
    assert tq.lib.tq_gemm_batch(ok, 1, 33, ws, big, None) == -2                # M > 32
    assert tq.lib.tq_gemm_batch_ex(ok, 1, 17, ws, big, tq.BATCH_MMA_SYNC, None) == -8   # mma.sync: M <= 16
    assert tq.lib.tq_gemm_batch_ex(ok, 1, 4, ws, big, 7, None) == -8                     # unknown variant
    assert tq.lib.tq_gemm_batch(ok, 1, -1, ws, big, None) == -2
    assert tq.lib.tq_gemm_batch(None, 1, 1, ws, big, None) == -1
    assert tq.lib.tq_gemm_batch(_items((a, a, a, a, 64, 100)), 1, 1, ws, big, None) == -2   # K % 64
    assert tq.lib.w4g_gemm_batch(_items((a, a, a, a, 64, 192)), 1, 1, ws, big, None) == -2  # K % 128
    assert tq.lib.tq_gemm_batch(_items((a, a, a, a, -1, 128)), 1, 1, ws, big, None) == -2
    assert tq.lib.tq_gemm_batch(_items((0, a, a, a, 64, 128)), 1, 1, ws, big, None) == -1   # null x
    assert tq.lib.tq_gemm_batch(_items((q, a, a, a, 64, 128)), 1, 1, ws, big, None) == -3   # misaligned x
    assert tq.lib.tq_gemm_batch(_items((a, q, a, a, 64, 128)), 1, 1, ws, big, None) == -3   # misaligned w
    assert tq.lib.tq_gemm_batch(ok, 1, 1, None, big, None) == -1                # no workspace
    # the interleaved-layout flag: ternary items on the mma.sync kernel only
    assert tq.lib.tq_gemm_batch_ex(ok, 1, 4, ws, big, tq.BATCH_TENSOR_CORE | tq.BATCH_INTERLEAVED, None) == -8
    assert tq.lib.tq_gemm_batch_ex(ok, 1, 17, ws, big, tq.BATCH_AUTO | tq.BATCH_INTERLEAVED, None) == -8
    assert tq.lib.w4g_gemm_batch_ex(ok, 1, 4, ws, big, tq.BATCH_MMA_SYNC | tq.BATCH_INTERLEAVED, None) == -8
    assert tq.lib.tq_gemm_batch_ex(ok, 1, 4, ws, big, 3 | tq.BATCH_INTERLEAVED, None) == -8
    # the call-with-next entry: the next items' count, token count, pointers and shapes are
    # checked before anything else
    nxt = _items((0, a, 0, 0, 64, 128))
    assert tq.lib.tq_gemm_batch_next(ok, 1, 1, ws, big, 0, nxt, 9, 1, None) == -2   # next count
    assert tq.lib.tq_gemm_batch_next(ok, 1, 1, ws, big, 0, nxt, -1, 1, None) == -2
    assert tq.lib.tq_gemm_batch_next(ok, 1, 1, ws, big, 0, nxt, 1, 33, None) == -2  # next M
    assert tq.lib.tq_gemm_batch_next(ok, 1, 1, ws, big, 0, None, 1, 1, None) == -1  # null next
    assert tq.lib.tq_gemm_batch_next(ok, 1, 1, ws, big, 0, _items((0, 0, 0, 0, 64, 128)), 1, 1, None) == -1
    assert tq.lib.tq_gemm_batch_next(ok, 1, 1, ws, big, 0, _items((0, q, 0, 0, 64, 128)), 1, 1, None) == -3
    assert tq.lib.tq_gemm_batch_next(ok, 1, 1, ws, big, 0, _items((0, a, 0, 0, 64, 100)), 1, 1, None) == -2
    assert tq.lib.w4g_gemm_batch_next(ok, 1, 1, ws, big, 0, _items((0, a, 0, 0, 64, 192)), 1, 1, None) == -2
    assert tq.lib.tq_gemm_batch_next(ok, 0, 1, ws, big, 0, nxt, 1, 1, None) == -2   # this call's count
    # the allocation-free variant checks the same arguments before any device work
    assert tq.lib.tq_gemm_batch_noalloc(ok, 0, 1, None) == -2
    assert tq.lib.tq_gemm_batch_noalloc(ok, 9, 1, None) == -2
    assert tq.lib.tq_gemm_batch_noalloc(ok, 1, 33, None) == -2
    assert tq.lib.tq_gemm_batch_noalloc(ok, 1, -1, None) == -2
    assert tq.lib.tq_gemm_batch_noalloc(None, 1, 1, None) == -1
    assert tq.lib.tq_gemm_batch_noalloc(ok, 1, 0, None) == 0
    assert tq.lib.tq_gemm_batch(ok, 1, 1, ctypes.c_void_p(1 << 20 | 4), big, None) == -3
    need = tq.tq_batch_workspace_size()
    assert need > 0
    assert tq.lib.tq_gemm_batch(ok, 1, 1, ws, need - 1, None) == -2            # workspace too small
    # nothing to do: no launch, no workspace needed
    assert tq.lib.tq_gemm_batch(ok, 1, 0, None, 0, None) == 0                   # M = 0
    assert tq.lib.tq_gemm_batch(_items((0, 0, 0, 0, 0, 128)), 1, 4, None, 0, None) == 0  # N = 0


def test_no_cpu_fallback_for_host_tensors():
    # the product path runs only in the CUDA library: host tensors are refused, never computed
    x = torch.zeros(1, 64, dtype=torch.float16)
    p = torch.full((8, 16), 0x55, dtype=torch.uint8)
    s = torch.zeros(8, dtype=torch.float16)
    with pytest.raises(ValueError):
        tq.tq_gemm(x, p, s)
    with pytest.raises(ValueError):
        tq.tq_quantize_pack(torch.zeros(8, 64))


def test_import_fails_loudly_without_the_library(tmp_path):
    # a copy of the package with no libtq.so and no compiler: importing it must fail
    import shutil
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    shutil.copytree(os.path.join(root, "bit_weight_only_tq_b200"), tmp_path / "bit_weight_only_tq_b200",
                    ignore=shutil.ignore_patterns("*.so", "*.so.tmp", "__pycache__"))
    shutil.copytree(os.path.join(root, "include"), tmp_path / "include")
    env = dict(os.environ, NVCC=str(tmp_path / "no-such-nvcc"))
    r = subprocess.run([sys.executable, "-c", "import bit_weight_only_tq_b200"], cwd=tmp_path, env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert not (tmp_path / "bit_weight_only_tq_b200" / "libtq.so").exists()


def test_interleave_argument_errors_without_gpu():
    a = ctypes.c_void_p(1 << 20)
    q = ctypes.c_void_p((1 << 20) + 2)
    assert tq.lib.tq_interleave_packed(a, a, 8, 24, None) == -2      # K % 16
    assert tq.lib.tq_interleave_packed(a, a, -1, 64, None) == -2
    assert tq.lib.tq_interleave_packed(a, a, 0, 64, None) == 0       # empty
    assert tq.lib.tq_interleave_packed(None, a, 8, 64, None) == -1
    assert tq.lib.tq_interleave_packed(q, a, 8, 64, None) == -3      # misaligned
